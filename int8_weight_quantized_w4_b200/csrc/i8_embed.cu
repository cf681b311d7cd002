// i8_embed_lookup: the token lookup on the tied int8 table of "ONNX export,
// quantization and the browser runtime", section "Quantization
// (train/quantize.py)", step 3: the table is stored once as [K, V] int8 with
// one scale per token, and the lookup is Gather(axis=1) + Transpose on it,
// dequantized: out[i, k] = T[k, tokens[i]] * s[tokens[i]].
//
// One CTA per (token, 256 rows): each thread reads one byte of the token's
// column (rows are ldt bytes apart) and writes one fp32. The lookup touches
// K bytes per token, so it is latency-bound; no staging is worth it.
#include <cuda_runtime.h>

#include "w4_device.cuh"
#include "w4_internal.h"

namespace {

using namespace w4dev;

constexpr int ET = 256;

__global__ void __launch_bounds__(ET) i8_embed_kernel(const int8_t* __restrict__ table, int64_t ldt,
                                                      const float* __restrict__ scales,
                                                      const int32_t* __restrict__ tokens, float* __restrict__ out,
                                                      int64_t ldo, int32_t K, int32_t V, ErrorWord* err) {
  const int64_t i = blockIdx.x;
  const int k = blockIdx.y * ET + threadIdx.x;
  const int32_t v = __ldg(tokens + i);
  const bool valid = v >= 0 && v < V;
  if (!valid && threadIdx.x == 0 && blockIdx.y == 0) record_error(err, W4_ERR_VALUE, K_EMBED, v);
  if (k >= K) return;
  float e = 0.f;
  if (valid) e = static_cast<float>(__ldg(table + static_cast<int64_t>(k) * ldt + v)) * __ldg(scales + v);
  out[i * ldo + k] = e;
}

}  // namespace

extern "C" w4_status i8_embed_lookup(const int8_t* table, int64_t ldt, const float* scales, const int32_t* tokens,
                                     int64_t ntok, float* out, int64_t ldo, int64_t K, int64_t V, void* stream) {
  using namespace w4host;
  if (ntok < 0 || K < 0 || V < 0) return fail(W4_ERR_SHAPE, "negative size");
  if (ntok == 0 || K == 0) return W4_OK;
  if (V == 0) return fail(W4_ERR_SHAPE, "V == 0: no token is valid");
  if (table == nullptr || scales == nullptr || tokens == nullptr || out == nullptr)
    return fail(W4_ERR_NULL, "table, scales, tokens and out must not be NULL");
  if (ldt < V) return fail(W4_ERR_SHAPE, "ldt < V");
  if (ldo < K) return fail(W4_ERR_SHAPE, "ldo < K");
  if (K > 0x7fffffff || V > 0x7fffffff || ntok > 0x7fffffff)
    return fail(W4_ERR_SHAPE, "sizes must be below 2^31");
  if ((reinterpret_cast<uintptr_t>(scales) & 3) != 0 || (reinterpret_cast<uintptr_t>(out) & 3) != 0 ||
      (reinterpret_cast<uintptr_t>(tokens) & 3) != 0)
    return fail(W4_ERR_ALIGN, "scales, tokens and out must be 4-byte aligned");
  const DeviceInfo* di = nullptr;
  const w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  const dim3 grid(static_cast<unsigned>(ntok), static_cast<unsigned>((K + ET - 1) / ET));
  if (grid.y > 65535) return fail(W4_ERR_SHAPE, "K too large for the lookup grid");
  i8_embed_kernel<<<grid, ET, 0, static_cast<cudaStream_t>(stream)>>>(
      table, ldt, scales, tokens, out, ldo, static_cast<int32_t>(K), static_cast<int32_t>(V), di->err);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch i8_embed");
}
