// w4_quantize / i8_quantize_head: the export's quantisers on the GPU.
// "ONNX export, quantization and the browser runtime", section
// "Quantization (train/quantize.py)":
//  * step 2 (dq4): 4-bit asymmetric, blocks along K (32 shipped; 64 is the
//    group size of the page's MLX comparison), one scale and one uint4 zero
//    point per (block, column); scales fp32, or fp16 (the "fp16 scales" row
//    of the page's measurements);
//  * step 3 (embedding_int8): int8 with one scale per token (column of the
//    [K, V] head table).
// The page gives no formula. The min/max reading, every step in fp64 (the
// differences of fp32 values are exact there and each division rounds once),
// so that the integer codes follow from the definition and not from an
// evaluation order:
//   lo = min(min w, 0), hi = max(max w, 0); s = (hi - lo) / 15 rounded once
//   to the stored type; a stored s of 0 (an all-zero block, or a range below
//   the type's smallest value) becomes s = 1, zp = 0; zp = rint(-lo / s),
//   q = rint(w / s) + zp, both clamped to 0..15 (rint: half to even).
//   int8: s = max|w| / 127 rounded once to fp32 (0 -> 1), q = rint(w / s)
//   clamped to -127..127.
// Inputs must be finite.
//
// One thread per (K-block, column pair) for dq4: the two columns of a packed
// byte; loads of neighbouring threads are neighbouring 8 bytes of a row. One
// thread per column for the int8 table. Both passes over a block re-read it
// (the second from L1/L2). Memory-bound, one launch each.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "w4_device.cuh"
#include "w4_internal.h"

namespace {

constexpr int QT = 128;

struct Q4 {
  double s;  // stored scale, widened
  int zp;
};

__device__ __forceinline__ Q4 q4_params(double lo, double hi, bool f16, float* s32, __half* s16) {
  const double s64 = (hi - lo) / 15.0;
  double s;
  if (f16) {
    const __half h = __double2half(s64);
    s = static_cast<double>(__half2float(h));
    *s16 = s == 0.0 ? __float2half(1.f) : h;
  } else {
    const float f = __double2float_rn(s64);
    s = static_cast<double>(f);
    *s32 = s == 0.0 ? 1.f : f;
  }
  if (s == 0.0) return {1.0, 0};
  const double z = rint(-lo / s);
  return {s, static_cast<int>(fmin(fmax(z, 0.0), 15.0))};
}

__device__ __forceinline__ int q4_code(float w, const Q4& p) {
  const double q = rint(static_cast<double>(w) / p.s) + p.zp;
  return static_cast<int>(fmin(fmax(q, 0.0), 15.0));
}

template <int B>
__global__ void __launch_bounds__(QT) w4_quant_kernel(const float* __restrict__ w, int64_t ldw, int64_t N, int f16,
                                                      uint8_t* __restrict__ qw, void* __restrict__ scales,
                                                      uint8_t* __restrict__ zp) {
  const int64_t p = static_cast<int64_t>(blockIdx.x) * QT + threadIdx.x;  // column pair
  const int64_t b = blockIdx.y;                                            // K-block
  if (p >= N / 2) return;
  const float* src = w + b * B * ldw + 2 * p;
  double lo0 = 0.0, hi0 = 0.0, lo1 = 0.0, hi1 = 0.0;
#pragma unroll 8
  for (int r = 0; r < B; ++r) {
    const double a = src[r * ldw], c = src[r * ldw + 1];
    lo0 = fmin(lo0, a);
    hi0 = fmax(hi0, a);
    lo1 = fmin(lo1, c);
    hi1 = fmax(hi1, c);
  }
  float s32[2] = {0.f, 0.f};
  __half s16[2];
  const Q4 p0 = q4_params(lo0, hi0, f16 != 0, &s32[0], &s16[0]);
  const Q4 p1 = q4_params(lo1, hi1, f16 != 0, &s32[1], &s16[1]);
  if (f16) {
    __half* sc = static_cast<__half*>(scales) + b * N + 2 * p;
    sc[0] = s16[0];
    sc[1] = s16[1];
  } else {
    float* sc = static_cast<float*>(scales) + b * N + 2 * p;
    sc[0] = s32[0];
    sc[1] = s32[1];
  }
  zp[b * (N / 2) + p] = static_cast<uint8_t>(p0.zp | (p1.zp << 4));
  uint8_t* dst = qw + b * B * (N / 2) + p;
#pragma unroll 8
  for (int r = 0; r < B; ++r)
    dst[r * (N / 2)] = static_cast<uint8_t>(q4_code(src[r * ldw], p0) | (q4_code(src[r * ldw + 1], p1) << 4));
}

__global__ void __launch_bounds__(QT) i8_quant_kernel(const float* __restrict__ w, int64_t ldw, int64_t K, int64_t V,
                                                      int8_t* __restrict__ table, int64_t ldt,
                                                      float* __restrict__ scales) {
  const int64_t v = static_cast<int64_t>(blockIdx.x) * QT + threadIdx.x;
  if (v >= V) return;
  double amax = 0.0;
  for (int64_t k = 0; k < K; ++k) amax = fmax(amax, fabs(static_cast<double>(w[k * ldw + v])));
  float s = __double2float_rn(amax / 127.0);
  if (s == 0.f) s = 1.f;
  scales[v] = s;
  const double sd = static_cast<double>(s);
  for (int64_t k = 0; k < K; ++k) {
    const double q = rint(static_cast<double>(w[k * ldw + v]) / sd);
    table[k * ldt + v] = static_cast<int8_t>(fmin(fmax(q, -127.0), 127.0));
  }
}

}  // namespace

extern "C" w4_status w4_quantize(const float* w, int64_t ldw, int64_t K, int64_t N, int32_t block,
                                 int32_t scale_type, uint8_t* qw, void* scales, uint8_t* zp, void* stream) {
  using namespace w4host;
  if (K < 0 || N < 0) return fail(W4_ERR_SHAPE, "negative size");
  if (block != 32 && block != 64) return fail(W4_ERR_VALUE, "block must be 32 or 64, not %d", int(block));
  if (scale_type != W4_SCALE_F32 && scale_type != W4_SCALE_F16)
    return fail(W4_ERR_VALUE, "unknown scale type %d", int(scale_type));
  if (K % block != 0) return fail(W4_ERR_SHAPE, "K=%lld is not a multiple of %d", (long long)K, int(block));
  if (N % 2 != 0) return fail(W4_ERR_SHAPE, "N=%lld is odd", (long long)N);
  if (K == 0 || N == 0) return W4_OK;
  if (ldw < N) return fail(W4_ERR_SHAPE, "ldw=%lld < N=%lld", (long long)ldw, (long long)N);
  if (w == nullptr || qw == nullptr || scales == nullptr || zp == nullptr)
    return fail(W4_ERR_NULL, "w, qw, scales and zp must not be NULL");
  if ((reinterpret_cast<uintptr_t>(w) & 3) != 0) return fail(W4_ERR_ALIGN, "w must be 4-byte aligned");
  const uintptr_t sa = scale_type == W4_SCALE_F16 ? 1 : 3;
  if ((reinterpret_cast<uintptr_t>(scales) & sa) != 0)
    return fail(W4_ERR_ALIGN, "scales must be aligned to their element size");
  if (K / block > 65535) return fail(W4_ERR_SHAPE, "K / block must be at most 65535");
  const DeviceInfo* di = nullptr;
  const w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  const dim3 grid(static_cast<unsigned>((N / 2 + QT - 1) / QT), static_cast<unsigned>(K / block));
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int f16 = scale_type == W4_SCALE_F16 ? 1 : 0;
  if (block == 32)
    w4_quant_kernel<32><<<grid, QT, 0, st>>>(w, ldw, N, f16, qw, scales, zp);
  else
    w4_quant_kernel<64><<<grid, QT, 0, st>>>(w, ldw, N, f16, qw, scales, zp);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch w4_quant");
}

extern "C" w4_status i8_quantize_head(const float* w, int64_t ldw, int64_t K, int64_t V, int8_t* table, int64_t ldt,
                                      float* scales, void* stream) {
  using namespace w4host;
  if (K < 0 || V < 0) return fail(W4_ERR_SHAPE, "negative size");
  if (V == 0) return W4_OK;
  if (ldw < V || ldt < V) return fail(W4_ERR_SHAPE, "ldw and ldt must be at least V");
  if (scales == nullptr) return fail(W4_ERR_NULL, "scales must not be NULL");
  if (K > 0 && (w == nullptr || table == nullptr)) return fail(W4_ERR_NULL, "w and table must not be NULL");
  if ((reinterpret_cast<uintptr_t>(w) & 3) != 0 || (reinterpret_cast<uintptr_t>(scales) & 3) != 0)
    return fail(W4_ERR_ALIGN, "w and scales must be 4-byte aligned");
  const DeviceInfo* di = nullptr;
  const w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  i8_quant_kernel<<<static_cast<unsigned>((V + QT - 1) / QT), QT, 0, static_cast<cudaStream_t>(stream)>>>(
      w, ldw, K, V, table, ldt, scales);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch i8_quant");
}
