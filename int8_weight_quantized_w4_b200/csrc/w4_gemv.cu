// w4_gemv: y = x . W for small M (decode), W in the 4-bit blocked format of
// "ONNX export, quantization and the browser runtime", section
// "Quantization (train/quantize.py)", step 2 (dq4): blocks of 32 along K,
// fp32 scale and uint4 zero point per (block, column), w = (q - zp) * scale.
//
// Design (sm_100a):
//  * Persistent: one CTA per SM. The work of all matrices of a launch is one
//    flat space of "block-tiles" (one 32-row K-block of one 256-column tile
//    of one group of MT rows of x); CTA i takes the contiguous range
//    [i*W/G, (i+1)*W/G), so every SM streams the same number of weight bytes
//    (stream-K). A tile whose K-range straddles CTAs is finished by the last
//    CTA to arrive: each writes its partial sums to the workspace, bumps the
//    tile's counter, and the last one adds the partials in CTA order (a fixed
//    order: the result does not depend on arrival order) and resets the
//    counter to zero. A CTA is the first contributor of at most one split
//    tile, so counters are indexed by that CTA and live in a fixed region at
//    the start of the workspace: whatever shapes earlier calls had, the
//    counter region is all zeros between calls.
//  * Warp-specialised: warp 0 is the producer. Stages hold 8 K-blocks and
//    are aligned to the tile's 8-block grid, so a full stage is four copies,
//    issued by four lanes at once: 2-D tensor copies of the nibbles
//    (256 rows x 128 B), the scales (8 x 256 fp32) and the zero points
//    (8 x 128 B), and an untiled bulk copy per row of x. A partial stage (at
//    the ends of a CTA's range) issues per-block copies, one lane per block.
//    The stages form a ring guarded by mbarriers (no multicast anywhere).
//    The consumer warps dequantise in registers and accumulate.
//  * Dequantisation uses the exponent trick of w4_device.cuh: one LOP3 per
//    weight builds 2^23 + q*16^j, one packed f32x2 add subtracts the matching
//    zero-point float, packed f32x2 FMAs accumulate. Lane l owns 8 columns
//    (one 32-bit word of nibbles per row).
//  * MT = 1: two rows are processed as one f32x2 lane pair ({x_k, x_k+1}),
//    the scale is applied once per warp's row slice of a block.
//    MT >= 2: the weight is dequantised to fp32 exactly as the oracle does
//    ((q - zp) * s, one rounding) and reused for the MT rows of x.
//  * Accumulation is two-level (per stage slice, then across stages, then
//    across warps, then across CTAs), all fp32, fixed order.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>

#include "w4_device.cuh"
#include "w4_internal.h"

namespace {

using namespace w4dev;

constexpr int TILE_N = 256;         // columns per tile: 128 bytes of nibbles per row
constexpr int SB = 8;               // K-blocks per pipeline stage (256 rows)
constexpr int QW_STAGE = SB * 32 * (TILE_N / 2);  // 32 KB
constexpr int SC_STAGE = SB * TILE_N * 4;         // 8 KB
constexpr int ZP_STAGE = SB * (TILE_N / 2);       // 1 KB

// Per-matrix fields the kernel reads while walking its range. They are copied
// from the parameter block into shared memory once per CTA: dynamically
// indexed reads of a large parameter block miss the constant cache.
struct MatScalars {
  const float* x;
  const float* scales;
  const uint8_t* zp;
  float* y;
  int64_t ldx;
  int64_t ldy;
  int64_t bt_off;  // first flat block-tile of this matrix
  int32_t M, K, N, nb;
  int32_t ntn;  // column tiles
  int32_t nmc;  // groups of MT rows
};
static_assert(sizeof(MatScalars) % 8 == 0, "copied as 8-byte words");

struct MatParams {
  CUtensorMap qw_full;  // [K rows][N/2 bytes], box 256 rows x 128 bytes
  CUtensorMap qw_blk;   // same tensor, box 32 rows x 128 bytes
  CUtensorMap sc_full;  // [K/32][N] fp32, box 8 x 256
  CUtensorMap zp_full;  // [K/32][N/2 bytes], box 8 x 128
  MatScalars s;
};

struct GemvParams {
  MatParams mat[W4_GROUP_MAX];
  int64_t W;  // total block-tiles
  float* ws_partials;
  int32_t* ws_counters;
  ErrorWord* err;
  uint64_t timeout_ns;
  int32_t count;
  int32_t total_tiles;
};

template <int MT>
struct Cfg {
  static constexpr int NCW = (MT >= 4) ? 8 : 16;  // consumer warps
  static constexpr int NTHREADS = (NCW + 1) * 32;
  static constexpr int ROWS_PER_WARP = SB * 32 / NCW;  // 16 or 32
  static constexpr bool SMEM_ACC = MT >= 4;          // cross-stage accumulator in shared memory
  static constexpr int X_STAGE = MT * SB * 32 * 4;
  static constexpr int STAGE_BYTES = QW_STAGE + SC_STAGE + ZP_STAGE + X_STAGE;
  static constexpr int NSTAGES = (MT >= 8) ? 3 : 4;
  // per-warp column sums: [NCW][TILE_N] reused per row (register accumulator)
  // or [NCW][MT][TILE_N] holding the accumulator itself (SMEM_ACC)
  static constexpr int RED_BYTES = NCW * (SMEM_ACC ? MT : 1) * TILE_N * 4;
  static constexpr int SCAL_OFF = NSTAGES * STAGE_BYTES + RED_BYTES;
  static constexpr int BAR_OFF = SCAL_OFF + W4_GROUP_MAX * static_cast<int>(sizeof(MatScalars));
  static constexpr int SMEM_BYTES = BAR_OFF + 2 * NSTAGES * 8 + 64;
};

// Flat block-tile f -> (matrix, tile within matrix, block within tile).
struct Pos {
  int g;
  int64_t tile_l;
  int32_t blk;
};

__device__ __forceinline__ Pos locate(const MatScalars* ms, int count, int64_t f, int g_hint) {
  int g = g_hint;
#pragma unroll 1
  while (g + 1 < count && ms[g + 1].bt_off <= f) ++g;
  const MatScalars& m = ms[g];
  const int64_t local = f - m.bt_off;
  Pos r;
  r.g = g;
  r.tile_l = local / m.nb;
  r.blk = static_cast<int32_t>(local - r.tile_l * m.nb);
  return r;
}

// CTA whose range holds flat index f (ranges are [floor(i W / G), floor((i+1) W / G))).
__device__ __forceinline__ int64_t cta_of(int64_t f, int64_t W, int64_t G) { return ((f + 1) * G + W - 1) / W - 1; }

__device__ __forceinline__ int64_t range_lo(int64_t i, int64_t W, int64_t G) { return (i * W) / G; }

template <int MT>
__global__ void __launch_bounds__(Cfg<MT>::NTHREADS, 1) w4_gemv_kernel(const __grid_constant__ GemvParams p) {
  using C = Cfg<MT>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + C::NSTAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + C::NSTAGES);
  int* bcast = reinterpret_cast<int*>(empty + C::NSTAGES) + 4;
  float* red = reinterpret_cast<float*>(smem + C::NSTAGES * C::STAGE_BYTES);
  MatScalars* ms = reinterpret_cast<MatScalars*>(smem + C::SCAL_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t lo = range_lo(blockIdx.x, p.W, G);
  const int64_t hi = range_lo(blockIdx.x + 1, p.W, G);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::NCW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  {
    constexpr int WORDS = sizeof(MatScalars) / 8;
    for (int i = threadIdx.x; i < p.count * WORDS; i += blockDim.x) {
      const int g = i / WORDS, j = i - g * WORDS;
      reinterpret_cast<uint64_t*>(ms + g)[j] = reinterpret_cast<const uint64_t*>(&p.mat[g].s)[j];
    }
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lo < hi) {
      const int g_first = locate(ms, p.count, lo, 0).g;
      const int g_last = locate(ms, p.count, hi - 1, g_first).g;
      for (int g = g_first + (lane >> 2); g <= g_last; g += 8) {
        const CUtensorMap* mp = (lane & 3) == 0 ? &p.mat[g].qw_full
                               : (lane & 3) == 1 ? &p.mat[g].qw_blk
                               : (lane & 3) == 2 ? &p.mat[g].sc_full : &p.mat[g].zp_full;
        prefetch_tensormap(mp);
      }
    }
    int it = 0;
    int g_hint = 0;
    bool ok = true;
    int64_t f = lo;
    while (f < hi && ok) {
      const Pos ps = locate(ms, p.count, f, g_hint);
      g_hint = ps.g;
      const MatScalars& m = ms[ps.g];
      const MatParams& mp = p.mat[ps.g];
      const int64_t seg_end = min(hi, f + (m.nb - ps.blk));
      const int32_t t = static_cast<int32_t>(ps.tile_l / m.nmc);
      const int32_t mc = static_cast<int32_t>(ps.tile_l - static_cast<int64_t>(t) * m.nmc);
      const int32_t ncols = min(TILE_N, m.N - t * TILE_N);
      const int32_t mrows = min(MT, m.M - mc * MT);
      const float* xrow0 = m.x + static_cast<int64_t>(mc) * MT * m.ldx;
      const float* scol = m.scales + static_cast<int64_t>(t) * TILE_N;
      const uint8_t* zcol = m.zp + static_cast<int64_t>(t) * (TILE_N / 2);
      int32_t blk = ps.blk;
      const int32_t blk_end = blk + static_cast<int32_t>(seg_end - f);
      while (blk < blk_end) {
        const int32_t nblk = min(SB - (blk % SB), blk_end - blk);  // stay on the 8-block grid
        const bool full_stage = (nblk == SB);
        const int s = it % C::NSTAGES;
        const uint32_t round = it / C::NSTAGES;
        if (round > 0 && lane == 0)
          ok = mbar_wait_bounded(&empty[s], (round - 1) & 1, p.timeout_ns, abort_flag, p.err, K_GEMV, 1);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        uint8_t* st = smem + s * C::STAGE_BYTES;
        if (lane == 0) {
          const uint32_t wbytes = full_stage ? static_cast<uint32_t>(QW_STAGE + SC_STAGE + ZP_STAGE)
                                             : static_cast<uint32_t>(nblk) * (32 * (TILE_N / 2) + ncols * 4 + ncols / 2);
          mbar_arrive_expect_tx(&full[s], wbytes + static_cast<uint32_t>(mrows) * nblk * 128);
        }
        __syncwarp();
        if (full_stage) {
          if (lane == 0) tma_g2s_2d(st, &mp.qw_full, t * (TILE_N / 2), blk * 32, &full[s]);
          if (lane == 1) tma_g2s_2d(st + QW_STAGE, &mp.sc_full, t * TILE_N, blk, &full[s]);
          if (lane == 2) tma_g2s_2d(st + QW_STAGE + SC_STAGE, &mp.zp_full, t * (TILE_N / 2), blk, &full[s]);
        } else if (lane < nblk) {
          const int64_t b = blk + lane;
          tma_g2s_2d(st + lane * 32 * (TILE_N / 2), &mp.qw_blk, t * (TILE_N / 2), static_cast<int32_t>(b * 32),
                     &full[s]);
          bulk_g2s(st + QW_STAGE + lane * TILE_N * 4, scol + b * m.N, ncols * 4, &full[s]);
          bulk_g2s(st + QW_STAGE + SC_STAGE + lane * (TILE_N / 2), zcol + b * (m.N / 2), ncols / 2, &full[s]);
        }
        if (lane >= 8 && lane < 8 + mrows)
          bulk_g2s(st + QW_STAGE + SC_STAGE + ZP_STAGE + (lane - 8) * SB * 32 * 4,
                   xrow0 + static_cast<int64_t>(lane - 8) * m.ldx + static_cast<int64_t>(blk) * 32, nblk * 128,
                   &full[s]);
        ++it;
        blk += nblk;
      }
      f = seg_end;
    }
    // Copies still in flight must land before this CTA may exit: wait (bounded)
    // for the last fill of every stage. In a normal run the consumers have
    // already waited for all of them. Stage s was filled ceil((it - s) / NSTAGES)
    // times.
    if (lane == 0)
      for (int s = 0; s < C::NSTAGES; ++s) {
        const int fills_s = it > s ? (it - s + C::NSTAGES - 1) / C::NSTAGES : 0;
        if (fills_s > 0) mbar_wait_bounded(&full[s], (fills_s - 1) & 1, p.timeout_ns, nullptr, p.err, K_GEMV, 2);
      }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int cw = warp - 1;  // 0 .. NCW-1
  const int ctid = threadIdx.x - 32;
  constexpr int WPB = 32 / C::ROWS_PER_WARP;  // warps per K-block (2 or 1)
  const int jblk = cw / WPB;
  const int r0 = (cw % WPB) * C::ROWS_PER_WARP;
  int it = 0;
  bool ok = true;

  int64_t f = lo;
  int g_hint = 0;
  while (f < hi) {
    const Pos ps = locate(ms, p.count, f, g_hint);
    g_hint = ps.g;
    const MatScalars& m = ms[ps.g];
    const int64_t seg_end = min(hi, f + (m.nb - ps.blk));
    const int32_t t = static_cast<int32_t>(ps.tile_l / m.nmc);
    const int32_t mc = static_cast<int32_t>(ps.tile_l - static_cast<int64_t>(t) * m.nmc);

    // accumulators: MT == 1 -> acc[i] = {even rows, odd rows} of column i
    //               MT == 2 -> acc[mm*4 + pp] = columns {2pp, 2pp+1} of row mm
    //               MT >= 4 -> this warp's slice red[cw][mm][TILE_N] in shared memory
    constexpr int NACC = C::SMEM_ACC ? 1 : (MT == 1 ? 8 : MT * 4);
    float2 acc[NACC];
#pragma unroll
    for (int i = 0; i < NACC; ++i) acc[i] = make_float2(0.f, 0.f);
    float* wacc = red + cw * (C::SMEM_ACC ? MT : 1) * TILE_N + lane * 8;
    if constexpr (C::SMEM_ACC) {
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) {
        reinterpret_cast<float4*>(wacc + mm * TILE_N)[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4*>(wacc + mm * TILE_N)[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }

    int32_t blk = ps.blk;
    const int32_t blk_end = blk + static_cast<int32_t>(seg_end - f);
    while (blk < blk_end) {
      const int32_t nblk = min(SB - (blk % SB), blk_end - blk);  // same grid as the producer
      const int s = it % C::NSTAGES;
      const uint32_t round = it / C::NSTAGES;
      if (ok) ok = mbar_wait_bounded(&full[s], round & 1, p.timeout_ns, abort_flag, p.err, K_GEMV, 3);
      if (ok && jblk < nblk) {
        const uint8_t* st = smem + s * C::STAGE_BYTES;
        const uint32_t* q32 = reinterpret_cast<const uint32_t*>(st) + (jblk * 32 + r0) * 32 + lane;
        const uint32_t zw = reinterpret_cast<const uint32_t*>(st + QW_STAGE + SC_STAGE)[jblk * 32 + lane];
        const float4* sc4 = reinterpret_cast<const float4*>(st + QW_STAGE) + jblk * (TILE_N / 4) + lane * 2;
        const float4 sa = sc4[0], sb = sc4[1];
        const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
        const float* xs = reinterpret_cast<const float*>(st + QW_STAGE + SC_STAGE + ZP_STAGE) + jblk * 32 + r0;
        float ncz[8], sp[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          ncz[i] = -magic_nib(i < 4 ? zw : (zw >> 16), i & 3);
          sp[i] = sv[i] * inv_slot_scale(i & 3);
        }
        if constexpr (MT == 1) {
          float2 P[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) P[i] = make_float2(0.f, 0.f);
#pragma unroll
          for (int r = 0; r < C::ROWS_PER_WARP; r += 2) {
            const float2 xx = *reinterpret_cast<const float2*>(xs + r);
            const uint32_t a0 = q32[r * 32], a1 = q32[(r + 1) * 32];
            const uint32_t b0 = a0 >> 16, b1 = a1 >> 16;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 e = make_float2(magic_nib(i < 4 ? a0 : b0, i & 3), magic_nib(i < 4 ? a1 : b1, i & 3));
              const float2 d = __fadd2_rn(e, make_float2(ncz[i], ncz[i]));
              P[i] = __ffma2_rn(xx, d, P[i]);
            }
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = __ffma2_rn(P[i], make_float2(sp[i], sp[i]), acc[i]);
        } else {
          float2 P[MT * 4];
#pragma unroll
          for (int i = 0; i < MT * 4; ++i) P[i] = make_float2(0.f, 0.f);
#pragma unroll 4
          for (int r = 0; r < C::ROWS_PER_WARP; ++r) {
            const uint32_t a = q32[r * 32];
            const uint32_t b = a >> 16;
            float2 wv[4];
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
              const int i0 = 2 * pp, i1 = 2 * pp + 1;
              const float2 e = make_float2(magic_nib(i0 < 4 ? a : b, i0 & 3), magic_nib(i1 < 4 ? a : b, i1 & 3));
              const float2 d = __fadd2_rn(e, make_float2(ncz[i0], ncz[i1]));
              wv[pp] = __fmul2_rn(d, make_float2(sp[i0], sp[i1]));
            }
#pragma unroll
            for (int mm = 0; mm < MT; ++mm) {
              const float xv = xs[mm * SB * 32 + r];
              const float2 xx = make_float2(xv, xv);
#pragma unroll
              for (int pp = 0; pp < 4; ++pp) P[mm * 4 + pp] = __ffma2_rn(xx, wv[pp], P[mm * 4 + pp]);
            }
          }
          if constexpr (C::SMEM_ACC) {
#pragma unroll
            for (int mm = 0; mm < MT; ++mm) {
              float4* a4 = reinterpret_cast<float4*>(wacc + mm * TILE_N);
              float4 u = a4[0], v = a4[1];
              u.x += P[mm * 4 + 0].x; u.y += P[mm * 4 + 0].y; u.z += P[mm * 4 + 1].x; u.w += P[mm * 4 + 1].y;
              v.x += P[mm * 4 + 2].x; v.y += P[mm * 4 + 2].y; v.z += P[mm * 4 + 3].x; v.w += P[mm * 4 + 3].y;
              a4[0] = u;
              a4[1] = v;
            }
          } else {
#pragma unroll
            for (int i = 0; i < MT * 4; ++i) acc[i] = __fadd2_rn(acc[i], P[i]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      ++it;
      blk += nblk;
    }

    // ---- segment done: reduce the NCW warps' partials, then write or fix up
    const int64_t t_start = f - ps.blk;
    const int64_t t_end = t_start + m.nb;
    const int64_t c_first = cta_of(t_start, p.W, G);
    const int64_t c_last = cta_of(t_end - 1, p.W, G);
    const bool split = c_first != c_last;
    const int slot = (split && static_cast<int64_t>(blockIdx.x) == c_first && lo < t_start) ? 1 : 0;
    const int col = ctid;  // threads 0..255 own one column each in the reduction
    const int64_t gcol = static_cast<int64_t>(t) * TILE_N + col;
#pragma unroll
    for (int mm = 0; mm < MT; ++mm) {
      if constexpr (!C::SMEM_ACC) {
        float4 lo4, hi4;
        if constexpr (MT == 1) {
          lo4 = make_float4(acc[0].x + acc[0].y, acc[1].x + acc[1].y, acc[2].x + acc[2].y, acc[3].x + acc[3].y);
          hi4 = make_float4(acc[4].x + acc[4].y, acc[5].x + acc[5].y, acc[6].x + acc[6].y, acc[7].x + acc[7].y);
        } else {
          lo4 = make_float4(acc[mm * 4 + 0].x, acc[mm * 4 + 0].y, acc[mm * 4 + 1].x, acc[mm * 4 + 1].y);
          hi4 = make_float4(acc[mm * 4 + 2].x, acc[mm * 4 + 2].y, acc[mm * 4 + 3].x, acc[mm * 4 + 3].y);
        }
        float4* dst = reinterpret_cast<float4*>(wacc);
        dst[0] = lo4;
        dst[1] = hi4;
      }
      named_bar_sync(1, C::NCW * 32);
      if (col < TILE_N) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < C::NCW; ++w)
          v += red[(w * (C::SMEM_ACC ? MT : 1) + (C::SMEM_ACC ? mm : 0)) * TILE_N + col];
        const int32_t row = mc * MT + mm;
        if (!split) {
          if (ok && row < m.M && gcol < m.N) m.y[static_cast<int64_t>(row) * m.ldy + gcol] = v;
        } else {
          p.ws_partials[((static_cast<int64_t>(blockIdx.x) * 2 + slot) * MT + mm) * TILE_N + col] = v;
        }
      }
      named_bar_sync(1, C::NCW * 32);
    }
    if (split) {
      __threadfence();
      named_bar_sync(1, C::NCW * 32);
      if (ctid == 0) bcast[0] = ok ? atomicAdd(&p.ws_counters[c_first], 1) : -1;
      named_bar_sync(1, C::NCW * 32);
      const int prev = bcast[0];
      if (prev == static_cast<int>(c_last - c_first)) {
        __threadfence();
        if (col < TILE_N) {
          for (int mm = 0; mm < MT; ++mm) {
            float v = 0.f;
            for (int64_t c = c_first; c <= c_last; ++c) {
              const int sl = (c == c_first && range_lo(c, p.W, G) < t_start) ? 1 : 0;
              v += __ldcg(&p.ws_partials[((c * 2 + sl) * MT + mm) * TILE_N + col]);
            }
            const int32_t row = mc * MT + mm;
            if (row < m.M && gcol < m.N) m.y[static_cast<int64_t>(row) * m.ldy + gcol] = v;
          }
        }
        if (ctid == 0) p.ws_counters[c_first] = 0;
      }
      named_bar_sync(1, C::NCW * 32);
    }
    f = seg_end;
  }
}

template <int MT>
w4_status launch_mt(const GemvParams& prm, int grid, cudaStream_t st, const w4host::DeviceInfo& di) {
  using C = Cfg<MT>;
  static int configured_dev[64] = {};
  if (di.dev < 64 && !configured_dev[di.dev]) {
    cudaError_t e = cudaFuncSetAttribute(w4_gemv_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return w4host::cuda_fail(e, "cudaFuncSetAttribute(w4_gemv)");
    configured_dev[di.dev] = 1;
  }
  w4_gemv_kernel<MT><<<grid, C::NTHREADS, C::SMEM_BYTES, st>>>(prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return w4host::cuda_fail(e, "launch w4_gemv");
  return W4_OK;
}

int pick_mt(const w4_desc* d, int count) {
  int64_t mx = 0;
  for (int i = 0; i < count; ++i) mx = std::max(mx, d[i].M);
  return mx <= 1 ? 1 : mx <= 2 ? 2 : mx <= 4 ? 4 : 8;
}

struct Plan {
  int mt = 1;
  int64_t W = 0;
  int32_t total_tiles = 0;
  int grid = 0;
};

Plan make_plan(const w4_desc* d, int count, int sms) {
  Plan pl;
  pl.mt = pick_mt(d, count);
  for (int i = 0; i < count; ++i) {
    if (d[i].M == 0 || d[i].N == 0 || d[i].K == 0) continue;
    const int64_t ntn = (d[i].N + TILE_N - 1) / TILE_N;
    const int64_t nmc = (d[i].M + pl.mt - 1) / pl.mt;
    pl.total_tiles += static_cast<int32_t>(ntn * nmc);
    pl.W += ntn * nmc * (d[i].K / 32);
  }
  pl.grid = static_cast<int>(std::min<int64_t>(std::min(sms, 1024), pl.W));
  return pl;
}

// Workspace: [COUNTER_SLOTS int32 counters][grid][2][MT][TILE_N] fp32 partials.
constexpr int COUNTER_SLOTS = 1024;  // >= grid (one per CTA)
constexpr size_t COUNTER_BYTES = COUNTER_SLOTS * sizeof(int32_t);

size_t ws_bytes(const Plan& pl) {
  if (pl.W == 0) return 0;
  return COUNTER_BYTES + static_cast<size_t>(pl.grid) * 2 * pl.mt * TILE_N * sizeof(float);
}

}  // namespace

namespace w4host {

bool gemv_eligible(const w4_desc& d, const char** why) {
  if (d.N % 32 != 0) {
    *why = "the GEMV path needs N % 32 == 0";
    return false;
  }
  if ((reinterpret_cast<uintptr_t>(d.x) & 15) != 0 || (d.ldx % 4) != 0) {
    *why = "the GEMV path needs x 16-byte aligned and ldx % 4 == 0";
    return false;
  }
  if (d.K > (int64_t(1) << 31) - 32 || d.N > (int64_t(1) << 31) - 256) {
    *why = "the GEMV path needs K and N below 2^31";
    return false;
  }
  return true;
}

size_t gemv_workspace_bytes(const w4_desc* d, int count, int sms) { return ws_bytes(make_plan(d, count, sms)); }

w4_status launch_gemv(const w4_desc* d, int count, void* ws, size_t ws_size, cudaStream_t st, const DeviceInfo& di) {
  if (count > W4_GROUP_MAX) return fail(W4_ERR_SHAPE, "at most %d matrices per GEMV launch", W4_GROUP_MAX);
  const Plan pl = make_plan(d, count, di.sms);
  if (pl.W == 0) return W4_OK;
  const size_t need = ws_bytes(pl);
  if (ws == nullptr || ws_size < need)
    return fail(W4_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws == nullptr ? size_t(0) : ws_size);
  if ((reinterpret_cast<uintptr_t>(ws) & 15) != 0) return fail(W4_ERR_WORKSPACE, "workspace must be 16-byte aligned");

  static_assert(sizeof(GemvParams) <= 32000, "kernel parameters must fit the 32 KB limit");
  static thread_local GemvParams prm;  // ~31 KB: kept off the host stack
  std::memset(&prm, 0, sizeof(prm));
  int g = 0;
  int64_t bt = 0;
  int32_t tiles = 0;
  for (int i = 0; i < count; ++i) {
    const w4_desc& s = d[i];
    if (s.M == 0 || s.N == 0 || s.K == 0) continue;
    MatParams& mpar = prm.mat[g];
    w4_status rc = encode_w4_maps(&mpar.qw_full, &mpar.qw_blk, &mpar.sc_full, &mpar.zp_full, s.qw, s.scales, s.zp,
                                  s.K, s.N);
    if (rc != W4_OK) return rc;
    MatScalars& m = mpar.s;
    m.x = s.x;
    m.scales = s.scales;
    m.zp = s.zp;
    m.y = s.y;
    m.ldx = s.ldx;
    m.ldy = s.ldy;
    m.M = static_cast<int32_t>(s.M);
    m.K = static_cast<int32_t>(s.K);
    m.N = static_cast<int32_t>(s.N);
    m.nb = static_cast<int32_t>(s.K / 32);
    m.ntn = static_cast<int32_t>((s.N + TILE_N - 1) / TILE_N);
    m.nmc = static_cast<int32_t>((s.M + pl.mt - 1) / pl.mt);
    m.bt_off = bt;
    tiles += m.ntn * m.nmc;
    bt += static_cast<int64_t>(m.ntn) * m.nmc * m.nb;
    ++g;
  }
  prm.count = g;
  prm.W = bt;
  prm.total_tiles = tiles;
  prm.ws_counters = static_cast<int32_t*>(ws);
  prm.ws_partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + COUNTER_BYTES);
  prm.err = di.err;
  prm.timeout_ns = wait_timeout_ns();
  switch (pl.mt) {
    case 1: return launch_mt<1>(prm, pl.grid, st, di);
    case 2: return launch_mt<2>(prm, pl.grid, st, di);
    case 4: return launch_mt<4>(prm, pl.grid, st, di);
    default: return launch_mt<8>(prm, pl.grid, st, di);
  }
}

}  // namespace w4host
