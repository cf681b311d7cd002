// Host-side internals of libw4b200 shared between its translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <cstring>

#include "w4.h"

namespace w4dev {
struct ErrorWord;
}

namespace w4host {

struct DeviceInfo {
  int dev = -1;
  int sms = 0;
  int major = 0;
  int minor = 0;
  size_t smem_optin = 0;
  w4dev::ErrorWord* err = nullptr;  // device address of this device's error word
};

// Current device's cached properties (W4_ERR_DEVICE unless it is sm_100).
w4_status current_device(const DeviceInfo** out);

// Record a one-line reason for the calling thread and return `s`.
w4_status fail(w4_status s, const char* fmt, ...);
w4_status cuda_fail(cudaError_t e, const char* what);
uint64_t wait_timeout_ns();

// Tensor maps of one packed weight's nibbles [K rows][N/2 bytes]: boxes of
// 128 and 16 rows x 256 B (wide tiles), 256 and 32 rows x 128 B (narrow
// tiles). Cached per (pointer, K, N).
w4_status encode_w4_maps(CUtensorMap* wide_full, CUtensorMap* wide_unit, CUtensorMap* narrow_full,
                         CUtensorMap* narrow_unit, const uint8_t* qw, int64_t K, int64_t N);

// ---- body kernels
bool gemv_eligible(const w4_desc& d, const char** why);
size_t gemv_workspace_bytes(const w4_desc* d, int count, int sms);
w4_status launch_gemv(const w4_desc* d, int count, void* ws, size_t ws_size, cudaStream_t st,
                      const DeviceInfo& di);
w4_status launch_generic(const w4_desc& d, cudaStream_t st, const DeviceInfo& di);
// tcgen05 3xTF32 tile GEMM for M above kTcMinM (no workspace)
constexpr int64_t kTcMinM = 16;
bool tc_eligible(const w4_desc& d, const char** why);
w4_status launch_tc(const w4_desc* d, int count, cudaStream_t st, const DeviceInfo& di);
// y = 0 for K = 0; with epi_of, through that descriptor's fused epilogue.
w4_status launch_zero_fill(float* y, int64_t ldy, int64_t M, int64_t N, cudaStream_t st,
                           const w4_desc* epi_of = nullptr);

// ---- head kernels
struct HeadArgs {
  const float* h;
  int64_t ldh;
  const int8_t* table;
  int64_t ldt;
  const float* scales;
  float* logits;
  int64_t ldl;
  int64_t M, K, V;
};
size_t head_workspace_bytes(int64_t M, int64_t K, int64_t V, int sms);
w4_status launch_head(const HeadArgs& a, void* ws, size_t ws_size, cudaStream_t st, const DeviceInfo& di);
w4_status launch_head_generic(const HeadArgs& a, cudaStream_t st, const DeviceInfo& di);
// greedy decoding: the rows kernel folds its logits into 64-bit keys (M <= 2
// and h fits its shared memory); otherwise logits are written and reduced
bool head_rows_path(int64_t M, int64_t K);
w4_status launch_head_keys(const HeadArgs& a, unsigned long long* keys, cudaStream_t st, const DeviceInfo& di);
w4_status launch_argmax_rows(const float* logits, int64_t ldl, int64_t M, int64_t V, unsigned long long* keys,
                             cudaStream_t st);
w4_status launch_argmax_finish(const unsigned long long* keys, int64_t M, int32_t* tokens, float* best,
                               cudaStream_t st);

// ---- the head's streaming layout (i8r.cu), also read by the fused decode step
constexpr int kStreamHeadRound = 4096;  // table bytes of a round
constexpr int kStreamHeadKCap = 8192;   // rows of h the head kernel holds
struct StreamHeadGeom {
  int32_t nb, gsl, A, ngroups;  // 16-row blocks, log2 strips per group, rounds per group, groups
  int64_t group_bytes;          // A rounds of table bytes, then 8 * 2^gsl scales
  int64_t bytes;
};
bool stream_head_geom(int64_t K, int64_t V, StreamHeadGeom* g);
w4_status check_stream_head(const float* h, const void* tr, int64_t K, int64_t V);
w4_status launch_stream_head(const float* h, const void* tr, int64_t K, int64_t V, float* logits, cudaStream_t st,
                             const DeviceInfo& di);

// ---- diagnostics
w4_status launch_debug_wait(uint64_t timeout_ns, cudaStream_t st, const DeviceInfo& di);

}  // namespace w4host
