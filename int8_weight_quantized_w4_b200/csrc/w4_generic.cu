// Plain-load kernels for the shapes and alignments the TMA GEMV cannot take
// (N % 32 != 0, x rows not 16-byte aligned), the zero fill for K = 0, the
// plain head kernel, and the bounded-wait self test.
//
// Same arithmetic as the fast kernels' definition: w = (q - zp) * s with
// (q - zp) exact and one fp32 multiply ("ONNX export, quantization and the
// browser runtime", section "Quantization (train/quantize.py)", step 2), or
// w = q * s for the int8 head (step 3); fp32 accumulation in three levels
// (32 rows, 16 blocks, the rest) so the rounding error stays far below the
// 1e-5 * sum|x*w| tolerance even at K = 8192.
#include <cuda_runtime.h>

#include "w4_device.cuh"
#include "w4_internal.h"

namespace {

using namespace w4dev;

constexpr int GEN_MT = 8;  // rows of x per thread

// One thread per (column pair, group of 8 rows of x).
__global__ void __launch_bounds__(128) w4_generic_kernel(const float* __restrict__ x, int64_t ldx,
                                                         const uint8_t* __restrict__ qw,
                                                         const float* __restrict__ scales,
                                                         const uint8_t* __restrict__ zp, float* __restrict__ y,
                                                         int64_t ldy, int64_t M, int64_t K, int64_t N, Epi epi) {
  const int64_t pcol = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // column pair
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * GEN_MT;
  const int64_t half = N / 2;
  if (pcol >= half) return;
  const int mrows = static_cast<int>(min(static_cast<int64_t>(GEN_MT), M - m0));
  const int64_t nb = K / 32;
  float tot0[GEN_MT], tot1[GEN_MT];
#pragma unroll
  for (int m = 0; m < GEN_MT; ++m) tot0[m] = tot1[m] = 0.f;
  for (int64_t g0 = 0; g0 < nb; g0 += 16) {
    float grp0[GEN_MT], grp1[GEN_MT];
#pragma unroll
    for (int m = 0; m < GEN_MT; ++m) grp0[m] = grp1[m] = 0.f;
    const int64_t g1 = min(nb, g0 + 16);
    for (int64_t b = g0; b < g1; ++b) {
      const uint8_t zb = zp[b * half + pcol];
      const int z0 = zb & 15, z1 = zb >> 4;
      const float s0 = scales[b * N + 2 * pcol], s1 = scales[b * N + 2 * pcol + 1];
      float blk0[GEN_MT], blk1[GEN_MT];
#pragma unroll
      for (int m = 0; m < GEN_MT; ++m) blk0[m] = blk1[m] = 0.f;
      for (int kk = 0; kk < 32; ++kk) {
        const int64_t k = b * 32 + kk;
        const uint8_t qb = qw[k * half + pcol];
        const float w0 = static_cast<float>(static_cast<int>(qb & 15) - z0) * s0;
        const float w1 = static_cast<float>(static_cast<int>(qb >> 4) - z1) * s1;
#pragma unroll
        for (int m = 0; m < GEN_MT; ++m) {
          if (m < mrows) {
            const float xv = x[(m0 + m) * ldx + k];
            blk0[m] = fmaf(xv, w0, blk0[m]);
            blk1[m] = fmaf(xv, w1, blk1[m]);
          }
        }
      }
#pragma unroll
      for (int m = 0; m < GEN_MT; ++m) {
        grp0[m] += blk0[m];
        grp1[m] += blk1[m];
      }
    }
#pragma unroll
    for (int m = 0; m < GEN_MT; ++m) {
      tot0[m] += grp0[m];
      tot1[m] += grp1[m];
    }
  }
#pragma unroll
  for (int m = 0; m < GEN_MT; ++m) {
    if (m < mrows) {
      y[(m0 + m) * ldy + 2 * pcol] = epi_apply(tot0[m], epi, m0 + m, 2 * pcol);
      y[(m0 + m) * ldy + 2 * pcol + 1] = epi_apply(tot1[m], epi, m0 + m, 2 * pcol + 1);
    }
  }
}

// y = 0 (K = 0), through the epilogue when one is given.
__global__ void zero_fill_kernel(float* y, int64_t ldy, int64_t M, int64_t N, Epi epi) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t m = blockIdx.y;
  if (n < N && m < M) y[m * ldy + n] = epi_apply(0.f, epi, m, n);
}

// One thread per (token column, group of 8 rows of h).
__global__ void __launch_bounds__(128) head_generic_kernel(const float* __restrict__ h, int64_t ldh,
                                                           const int8_t* __restrict__ table, int64_t ldt,
                                                           const float* __restrict__ scales,
                                                           float* __restrict__ logits, int64_t ldl, int64_t M,
                                                           int64_t K, int64_t V) {
  const int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * GEN_MT;
  if (v >= V) return;
  const int mrows = static_cast<int>(min(static_cast<int64_t>(GEN_MT), M - m0));
  const float s = scales[v];
  float tot[GEN_MT], grp[GEN_MT], blk[GEN_MT];
#pragma unroll
  for (int m = 0; m < GEN_MT; ++m) tot[m] = grp[m] = blk[m] = 0.f;
  for (int64_t k = 0; k < K; ++k) {
    const float w = static_cast<float>(table[k * ldt + v]) * s;
#pragma unroll
    for (int m = 0; m < GEN_MT; ++m)
      if (m < mrows) blk[m] = fmaf(h[(m0 + m) * ldh + k], w, blk[m]);
    if ((k & 31) == 31 || k == K - 1) {
#pragma unroll
      for (int m = 0; m < GEN_MT; ++m) {
        grp[m] += blk[m];
        blk[m] = 0.f;
      }
      if ((k & 511) == 511 || k == K - 1) {
#pragma unroll
        for (int m = 0; m < GEN_MT; ++m) {
          tot[m] += grp[m];
          grp[m] = 0.f;
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < GEN_MT; ++m)
    if (m < mrows) logits[(m0 + m) * ldl + v] = tot[m];
}

// Waits on a shared-memory barrier that nothing completes, through the same
// bounded wait the matmul kernels use; records W4_ERR_TIMEOUT and returns.
__global__ void debug_wait_kernel(ErrorWord* err, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, timeout_ns, &abort_flag, err, K_DEBUG, 77);
}

}  // namespace

namespace w4host {

w4_status launch_generic(const w4_desc& d, cudaStream_t st, const DeviceInfo&) {
  const int64_t half = d.N / 2;
  const dim3 grid(static_cast<unsigned>((half + 127) / 128), static_cast<unsigned>((d.M + GEN_MT - 1) / GEN_MT));
  if (grid.y > 65535) return fail(W4_ERR_SHAPE, "M too large for the generic kernel");
  w4_generic_kernel<<<grid, 128, 0, st>>>(d.x, d.ldx, d.qw, d.scales, d.zp, d.y, d.ldy, d.M, d.K, d.N,
                                          Epi{d.bias, d.residual, d.ldr, d.act, 0});
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch w4_generic");
}

w4_status launch_zero_fill(float* y, int64_t ldy, int64_t M, int64_t N, cudaStream_t st, const w4_desc* epi_of) {
  if (M > 65535) return fail(W4_ERR_SHAPE, "M too large for the zero fill");
  const dim3 grid(static_cast<unsigned>((N + 255) / 256), static_cast<unsigned>(M));
  const Epi epi = epi_of == nullptr ? Epi{nullptr, nullptr, 0, W4_ACT_NONE, 0}
                                    : Epi{epi_of->bias, epi_of->residual, epi_of->ldr, epi_of->act, 0};
  zero_fill_kernel<<<grid, 256, 0, st>>>(y, ldy, M, N, epi);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch zero_fill");
}

w4_status launch_head_generic(const HeadArgs& a, cudaStream_t st, const DeviceInfo&) {
  const dim3 grid(static_cast<unsigned>((a.V + 127) / 128), static_cast<unsigned>((a.M + GEN_MT - 1) / GEN_MT));
  if (grid.y > 65535) return fail(W4_ERR_SHAPE, "M too large for the generic head kernel");
  head_generic_kernel<<<grid, 128, 0, st>>>(a.h, a.ldh, a.table, a.ldt, a.scales, a.logits, a.ldl, a.M, a.K, a.V);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch head_generic");
}

w4_status launch_debug_wait(uint64_t timeout_ns, cudaStream_t st, const DeviceInfo& di) {
  debug_wait_kernel<<<1, 32, 0, st>>>(di.err, timeout_ns);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch debug_wait");
}

}  // namespace w4host
