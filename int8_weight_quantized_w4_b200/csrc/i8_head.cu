// i8_head: logits[m, v] = s_v * sum_k h[m, k] * T[k, v] for the int8 tied
// LM head of "ONNX export, quantization and the browser runtime", section
// "Quantization (train/quantize.py)", steps 3 (embedding_int8: int8, one
// scale per token, [768, V] layout) and 4 (last_token_logits: only the last
// position's rows h are multiplied).
//
// Design (sm_100a):
//  * Row k of T starts at byte k*ldt, which is not aligned when ldt is odd
//    (V = 50257). With T 16-byte aligned, (k*ldt) mod 16 depends only on
//    k mod 16, so a warp that takes the rows k = k0 + w + 16 i (w = warp)
//    sees ONE misalignment r_w for all its rows. Each lane then loads
//    aligned CB-byte chunks (LDG.128 for CB = 16) and the warp's 32 lanes
//    cover the byte window that starts r_w bytes before the tile's first
//    column: no realignment in registers at all. The CTA's reduction across
//    warps undoes the per-warp shift (column c of the tile sits at window
//    position c + r_w of warp w). A tile is 31 chunks wide, so every warp's
//    32-chunk window covers it whatever r_w is.
//  * int8 -> fp32 exactly with one PRMT per element: the byte, biased by
//    0x80, is placed in the mantissa of 2^23 (0x4B0000uu), then one packed
//    f32x2 add removes 2^23 + 128. The per-token scale is applied once per
//    column after the sum.
//  * K is split over a thread-block cluster of KS CTAs (grid.y); each CTA
//    reduces its warps in shared memory, then CTA r of the cluster adds the
//    KS partials of its share of the columns through distributed shared
//    memory, in rank order (deterministic, no workspace, no atomics).
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "w4_device.cuh"
#include "w4_internal.h"

namespace cg = cooperative_groups;

namespace {

using namespace w4dev;

constexpr int NW = 16;  // warps per CTA; row stride of a warp

template <int MT>
struct HCfg {
  static constexpr int CB = MT <= 2 ? 16 : (MT == 4 ? 8 : 4);  // bytes per lane chunk
  static constexpr int WIN = 32 * CB;                          // window columns per warp
  static constexpr int TV = 31 * CB;                           // tile columns
  static constexpr int D = MT == 8 ? 2 : 4;  // rows in flight per warp batch
  static constexpr int RED_FLOATS = NW * MT * WIN;
  static constexpr int PART_FLOATS = MT * TV;
  static constexpr int SMEM = (RED_FLOATS + PART_FLOATS) * 4 + 64 * 4;
};

__device__ __forceinline__ float byte_magic(uint32_t biased_word, int j) {
  // bytes of the result: [biased byte j, 0x00, 0x00, 0x4B]
  return __uint_as_float(__byte_perm(biased_word, 0x4B000000u, 0x7540u + j));
}

template <int CB>
struct Chunk {
  uint32_t w[CB / 4];
};

template <int CB>
__device__ __forceinline__ Chunk<CB> load_chunk(const int8_t* p) {
  Chunk<CB> c;
  if constexpr (CB == 16) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    c.w[0] = v.x; c.w[1] = v.y; c.w[2] = v.z; c.w[3] = v.w;
  } else if constexpr (CB == 8) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    c.w[0] = v.x; c.w[1] = v.y;
  } else {
    c.w[0] = __ldg(reinterpret_cast<const unsigned int*>(p));
  }
  return c;
}

// Bytes of a chunk that straddles the end of the table: read the ones before
// `end`, zero the rest (their columns are never written).
template <int CB>
__device__ __forceinline__ Chunk<CB> load_chunk_clipped(const int8_t* p, const int8_t* end) {
  Chunk<CB> c;
#pragma unroll
  for (int i = 0; i < CB / 4; ++i) {
    uint32_t v = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int8_t* q = p + 4 * i + b;
      const uint32_t byte = (q < end) ? static_cast<uint32_t>(static_cast<uint8_t>(*q)) : 0u;
      v |= byte << (8 * b);
    }
    c.w[i] = v;
  }
  return c;
}

template <int MT>
__global__ void __launch_bounds__(NW * 32, MT == 1 ? 2 : 1) i8_head_kernel(const float* __restrict__ h, int64_t ldh,
                                                             const int8_t* __restrict__ table, int64_t ldt,
                                                             const float* __restrict__ scales,
                                                             float* __restrict__ logits, int64_t ldl, int32_t M,
                                                             int32_t K, int32_t V, int32_t KR) {
  using C = HCfg<MT>;
  constexpr int CB = C::CB;
  extern __shared__ __align__(16) float hsm[];
  float* red = hsm;                       // [NW][MT][WIN]
  float* part = hsm + C::RED_FLOATS;      // [MT][TV]
  int* shift = reinterpret_cast<int*>(part + C::PART_FLOATS);  // [NW]

  cg::cluster_group cluster = cg::this_cluster();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t v0 = static_cast<int64_t>(blockIdx.x) * C::TV;
  const int32_t kbeg = blockIdx.y * KR;
  const int32_t kend = min(K, kbeg + KR);
  const int32_t m0 = blockIdx.z * MT;
  const int mrows = min(MT, M - m0);
  const int8_t* table_end = table + (static_cast<int64_t>(K) - 1) * ldt + V;

  // window of this warp: starts r bytes before column v0 of each of its rows
  const int64_t first_row = kbeg + warp;
  const int r = static_cast<int>(reinterpret_cast<uintptr_t>(table + first_row * ldt + v0) & (CB - 1));
  if (lane == 0) shift[warp] = r;

  // acc[mm * CB/2 + pp] = columns {2pp, 2pp+1} of the lane's chunk, row mm
  float2 acc[MT * CB / 2];
#pragma unroll
  for (int i = 0; i < MT * CB / 2; ++i) acc[i] = make_float2(0.f, 0.f);
  const float2 bias = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)

  for (int32_t k0 = kbeg + warp; k0 < kend; k0 += NW * C::D) {
    Chunk<CB> ch[C::D];
    float hv[C::D][MT];
#pragma unroll
    for (int j = 0; j < C::D; ++j) {
      const int32_t k = k0 + j * NW;
      if (k < kend) {
        const int8_t* p = table + static_cast<int64_t>(k) * ldt + v0 - r + lane * CB;
        ch[j] = (p + CB <= table_end) ? load_chunk<CB>(p) : load_chunk_clipped<CB>(p, table_end);
#pragma unroll
        for (int mm = 0; mm < MT; ++mm)
          hv[j][mm] = (mm < mrows) ? __ldg(h + static_cast<int64_t>(m0 + mm) * ldh + k) : 0.f;
      } else {
#pragma unroll
        for (int i = 0; i < CB / 4; ++i) ch[j].w[i] = 0u;  // q = 0
#pragma unroll
        for (int mm = 0; mm < MT; ++mm) hv[j][mm] = 0.f;
      }
    }
#pragma unroll
    for (int j = 0; j < C::D; ++j) {
#pragma unroll
      for (int i = 0; i < CB / 4; ++i) {
        const uint32_t bw = ch[j].w[i] ^ 0x80808080u;
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
          const float2 e = make_float2(byte_magic(bw, 2 * pr), byte_magic(bw, 2 * pr + 1));
          const float2 q = __fadd2_rn(e, bias);  // exact int8 values
#pragma unroll
          for (int mm = 0; mm < MT; ++mm) {
            const float2 hh = make_float2(hv[j][mm], hv[j][mm]);
            acc[mm * (CB / 2) + i * 2 + pr] = __ffma2_rn(hh, q, acc[mm * (CB / 2) + i * 2 + pr]);
          }
        }
      }
    }
  }

  // ---- CTA reduction across warps (undo the per-warp window shift)
#pragma unroll
  for (int mm = 0; mm < MT; ++mm) {
    float* dst = red + (warp * MT + mm) * C::WIN + lane * CB;
#pragma unroll
    for (int pp = 0; pp < CB / 2; ++pp) {
      dst[2 * pp] = acc[mm * (CB / 2) + pp].x;
      dst[2 * pp + 1] = acc[mm * (CB / 2) + pp].y;
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < MT * C::TV; idx += NW * 32) {
    const int mm = idx / C::TV;
    const int c = idx - mm * C::TV;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) v += red[(w * MT + mm) * C::WIN + c + shift[w]];
    part[idx] = v;
  }
  // ---- cluster reduction across the K-split, through distributed shared memory
  cluster.sync();
  const int ks = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int per = (C::TV + ks - 1) / ks;
  const int c_lo = rank * per;
  const int c_hi = min(C::TV, c_lo + per);
  for (int idx = threadIdx.x; idx < MT * per; idx += NW * 32) {
    const int mm = idx / per;
    const int c = c_lo + (idx - mm * per);
    if (c >= c_hi) continue;
    float v = 0.f;
    for (int q = 0; q < ks; ++q) v += cluster.map_shared_rank(part, q)[mm * C::TV + c];
    const int64_t col = v0 + c;
    if (mm < mrows && col < V) logits[static_cast<int64_t>(m0 + mm) * ldl + col] = v * __ldg(scales + col);
  }
  cluster.sync();  // keep this CTA's shared memory alive until every peer has read it
}

template <int MT>
w4_status launch_head_mt(const w4host::HeadArgs& a, cudaStream_t st, const w4host::DeviceInfo& di) {
  using C = HCfg<MT>;
  static int configured[64] = {};
  if (di.dev < 64 && !configured[di.dev]) {
    cudaError_t e = cudaFuncSetAttribute(i8_head_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return w4host::cuda_fail(e, "cudaFuncSetAttribute(i8_head)");
    configured[di.dev] = 1;
  }
  const int64_t ntiles = (a.V + C::TV - 1) / C::TV;
  const int64_t nmc = (a.M + MT - 1) / MT;
  // K-split: enough CTAs for two per SM, at most 8 (portable cluster size),
  // at least 16 rows (one per warp) per CTA.
  int ks = static_cast<int>((2 * di.sms + ntiles * nmc - 1) / (ntiles * nmc));
  ks = std::max(1, std::min({ks, 8, static_cast<int>((a.K + NW - 1) / NW)}));
  const int32_t KR = static_cast<int32_t>(((a.K + ks - 1) / ks + NW - 1) / NW * NW);
  ks = static_cast<int>((a.K + KR - 1) / KR);
  if (ntiles > 0x7fffffff || nmc > 65535) return w4host::fail(W4_ERR_SHAPE, "head grid too large");

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ntiles), static_cast<unsigned>(ks), static_cast<unsigned>(nmc));
  cfg.blockDim = dim3(NW * 32, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(ks);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, i8_head_kernel<MT>, a.h, a.ldh, a.table, a.ldt, a.scales, a.logits, a.ldl,
                                     static_cast<int32_t>(a.M), static_cast<int32_t>(a.K), static_cast<int32_t>(a.V),
                                     KR);
  if (e != cudaSuccess) return w4host::cuda_fail(e, "launch i8_head");
  return W4_OK;
}

}  // namespace

namespace w4host {

w4_status launch_head(const HeadArgs& a, cudaStream_t st, const DeviceInfo& di) {
  if (a.K > 0x7fffffff || a.V > 0x7fffffff || a.M > 0x7fffffff)
    return fail(W4_ERR_SHAPE, "head sizes must be below 2^31 on the fast path");
  if (a.M <= 1) return launch_head_mt<1>(a, st, di);
  if (a.M <= 2) return launch_head_mt<2>(a, st, di);
  if (a.M <= 4) return launch_head_mt<4>(a, st, di);
  return launch_head_mt<8>(a, st, di);
}

}  // namespace w4host
