// w4_matmul_noalloc: w4_matmul for callers that cannot allocate device
// memory, with the split-K scratch held in a fixed array of this library.
//
// Who needs it: code that must not call cudaMalloc at the point where it
// multiplies, for example a plugin running inside another framework that owns
// every device allocation, a process that reserves all of its device memory
// up front and forbids allocation afterwards, or a latency-critical path that
// cannot afford the allocator's locking and possible device synchronisation.
// Such a caller still passes its inputs and outputs; only the scratch is
// provided here.
//
// The scratch is one file-scope __device__ array of W4_NOALLOC_SCRATCH_BYTES.
// Every GPU that loads the library holds it until the process exits, and all
// calls share it: each call that needs scratch first clears the split-K
// counters at its start (they must start at zero), and calls whose work
// overlaps on the GPU (different streams, or different host threads on one
// device) race on it. A call that the tensor-core or plain kernel takes needs
// no scratch at all.
#include <cuda_runtime.h>

#include <mutex>

#include "w4_internal.h"

static __device__ __align__(256) unsigned char g_w4_noalloc_scratch[W4_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevNoAlloc = 64;
constexpr size_t kCounterBytes = 4096;  // the GEMV's split-K counter block at the start of its workspace
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevNoAlloc] = {};

// Device address of the scratch array on the current device. In host code the
// array's name is only a host-side stand-in, so the address is asked from the
// runtime, once per device, with that device current.
w4_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return w4host::fail(W4_ERR_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevNoAlloc) return w4host::fail(W4_ERR_DEVICE, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_w4_noalloc_scratch);
    if (e != cudaSuccess) return w4host::cuda_fail(e, "cudaGetSymbolAddress(noalloc scratch)");
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return W4_OK;
}

}  // namespace

extern "C" w4_status w4_matmul_noalloc(const float* x, int64_t ldx, const uint8_t* qw, const float* scales,
                                       const uint8_t* zp, float* y, int64_t ldy, int64_t M, int64_t K, int64_t N,
                                       void* stream) {
  if (M < 0 || K < 0 || N < 0) return w4host::fail(W4_ERR_SHAPE, "negative size");
  if (M == 0 || N == 0) return W4_OK;
  const w4host::DeviceInfo* di = nullptr;
  w4_status rc = w4host::current_device(&di);
  if (rc != W4_OK) return rc;
  // The split-K scratch is the GEMV's; a call that goes to the tensor-core
  // kernel (M above 16) or to the plain kernel needs none.
  w4_desc d = {};
  d.x = x;
  d.ldx = ldx;
  d.qw = qw;
  d.scales = scales;
  d.zp = zp;
  d.y = y;
  d.ldy = ldy;
  d.M = M;
  d.K = K;
  d.N = N;
  const char* why = "";
  const bool gemv = M <= w4host::kTcMinM && w4host::gemv_eligible(d, &why);  // the choice w4_matmul makes
  const size_t need = gemv ? w4_matmul_workspace_size(M, K, N) : 0;
  if (need > static_cast<size_t>(W4_NOALLOC_SCRATCH_BYTES))
    return w4host::fail(W4_ERR_WORKSPACE,
                        "w4_matmul_noalloc: this shape needs %zu bytes of scratch, more than the %u bytes it holds "
                        "(M = %lld); use w4_matmul with a workspace",
                        need, static_cast<unsigned>(W4_NOALLOC_SCRATCH_BYTES), static_cast<long long>(M));
  void* scratch = nullptr;
  rc = scratch_address(&scratch);
  if (rc != W4_OK) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (need > 0) {
    // only the split-K counters must start at zero (the partial sums are
    // written before they are read); clearing them on every call also resets
    // a block that a call which timed out left non-zero
    const cudaError_t e = cudaMemsetAsync(scratch, 0, need < kCounterBytes ? need : kCounterBytes, st);
    if (e != cudaSuccess) return w4host::cuda_fail(e, "clear noalloc scratch counters");
  }
  return w4_matmul(x, ldx, qw, scales, zp, y, ldy, M, K, N, need > 0 ? scratch : nullptr, need, stream);
}
