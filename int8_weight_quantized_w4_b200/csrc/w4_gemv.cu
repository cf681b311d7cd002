// w4_gemv: y = x . W for small M (decode), W in the 4-bit blocked format of
// "ONNX export, quantization and the browser runtime", section
// "Quantization (train/quantize.py)", step 2 (dq4): blocks of 32 along K,
// fp32 scale and uint4 zero point per (block, column), w = (q - zp) * scale.
//
// Design (sm_100a):
//  * Column tiles are 512 columns wide (256-byte row pieces, which stream at
//    full HBM speed where 128-byte pieces do not); the last 256 or fewer
//    columns of a weight may form a narrow 256-column tile instead.
//  * Work is counted in units of 4 KB of nibbles: 16 rows of a wide tile or
//    32 rows (one K-block) of a narrow one. All matrices of a launch form one
//    flat range of units; CTA i (one per SM, persistent) takes
//    [i*W/G, (i+1)*W/G), so every SM streams the same bytes (stream-K). A
//    tile whose K-range straddles CTAs is finished by the last CTA to arrive:
//    each writes its partial sums to the workspace, bumps a counter, and the
//    last one adds the partials in CTA order (a fixed order: the result does
//    not depend on arrival order) and resets the counter to zero. A CTA is
//    the first contributor of at most one split tile, so the counters are
//    indexed by that CTA and live in a fixed block at the workspace start.
//  * Warp-specialised: warp 0 is the producer. A stage holds 8 units and is
//    aligned to the tile's 8-unit grid; a full stage is one 2-D tensor copy of
//    the nibbles (128 rows x 256 B or 256 rows x 128 B), one bulk copy per
//    K-block of scales and of zero points, and one per row of x, issued by
//    several lanes at once. A partial stage (at the ends of a CTA's range)
//    copies unit by unit. Stages form a ring guarded by mbarriers; no copy
//    uses multicast. Consumer warps dequantise in registers: each takes
//    16 rows x 256 columns of a stage, a lane owning 8 columns.
//  * Dequantisation uses the exponent trick of w4_device.cuh: one LOP3 per
//    weight builds 2^23 + q*16^j, one FADD subtracts the matching zero-point
//    float, one FFMA accumulates (scalar fp32: the packed f32x2 forms cost
//    more instructions here than they save).
//  * MT = 1: the scale is applied once per warp's 16-row slice of a block
//    (s * sum x (q - zp)).
//    MT >= 2: the weight is dequantised to fp32 exactly as the oracle does
//    ((q - zp) * s, one rounding) and reused for the MT rows of x.
//  * Accumulation is two-level (per 16-row slice, then across stages), then
//    across warps, then across CTAs: all fp32, all in a fixed order.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>

#include "w4_device.cuh"
#include "w4_internal.h"

namespace {

using namespace w4dev;

constexpr int WIDE_N = 512;    // columns of a wide tile (256-byte rows)
constexpr int NARROW_N = 256;  // columns of a narrow remainder tile (128-byte rows)
constexpr int SU = 8;          // units per pipeline stage
constexpr int QW_STAGE = SU * 4096;  // 32 KB of nibbles
constexpr int SC_STAGE = 8192;       // 4 blocks x 512 fp32 (wide) or 8 x 256 (narrow)
constexpr int ZP_STAGE = 1024;       // 4 x 256 B or 8 x 128 B
constexpr int X_ROWS = 256;          // rows of x per stage, at most

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
  int64_t u_off;   // first flat unit of this matrix
  int64_t u_wide;  // units of its wide tiles (all groups of MT rows)
  int32_t M, K, N, nb;
  int32_t ntw;     // wide tiles (the last may be partial)
  int32_t narrow;  // 1 when the last <= 256 columns form a narrow tile
  int32_t nmc;     // groups of MT rows
  int32_t pad;
};
static_assert(sizeof(MatScalars) % 8 == 0, "copied as 8-byte words");

struct MatParams {
  CUtensorMap qw_wide_full;    // [K rows][N/2 bytes], box 128 rows x 256 B
  CUtensorMap qw_wide_unit;    // box 16 rows x 256 B
  CUtensorMap qw_narrow_full;  // box 256 rows x 128 B
  CUtensorMap qw_narrow_unit;  // box 32 rows x 128 B
  MatScalars s;
};

struct GemvParams {
  MatParams mat[W4_GROUP_MAX];
  int64_t W;  // total units
  float* ws_partials;
  int32_t* ws_counters;
  ErrorWord* err;
  uint64_t timeout_ns;
  int32_t count;
  int32_t pad;
};

template <int MT>
struct Cfg {
  static constexpr int NCW = 8;                   // consumer warps (two 16-row items each per stage)
  static constexpr int IPW = 16 / NCW;            // 16-row items per warp per stage
  static constexpr int NTHREADS = (NCW + 1) * 32;
  static constexpr bool SMEM_ACC = MT >= 4;       // cross-stage accumulator in shared memory
  static constexpr int X_STAGE = MT * X_ROWS * 4;
  static constexpr int STAGE_BYTES = QW_STAGE + SC_STAGE + ZP_STAGE + X_STAGE;
  static constexpr int NSTAGES = (MT >= 8) ? 3 : 4;
  // per-warp column sums: [NCW][256] reused per row of x (register
  // accumulator) or [NCW][MT][256] holding the accumulator itself (SMEM_ACC)
  static constexpr int RED_BYTES = NCW * (SMEM_ACC ? MT : 1) * 256 * 4;
  static constexpr int SCAL_OFF = NSTAGES * STAGE_BYTES + RED_BYTES;
  static constexpr int BAR_OFF = SCAL_OFF + W4_GROUP_MAX * static_cast<int>(sizeof(MatScalars));
  static constexpr int SMEM_BYTES = BAR_OFF + 2 * NSTAGES * 8 + 64;
};

// Flat unit f -> (matrix, tile, group of rows, unit within the tile).
struct Pos {
  int g;
  bool wide;
  int32_t tile;       // column tile index (wide tiles first, then the narrow one)
  int32_t mc;         // group of MT rows of x
  int32_t unit;       // unit within the tile
  int32_t tile_units; // 2*nb (wide) or nb (narrow)
};

__device__ __forceinline__ Pos locate(const MatScalars* ms, int count, int64_t f, int g_hint) {
  int g = g_hint;
#pragma unroll 1
  while (g + 1 < count && ms[g + 1].u_off <= f) ++g;
  const MatScalars& m = ms[g];
  const int64_t local = f - m.u_off;
  Pos r;
  r.g = g;
  if (local < m.u_wide) {
    r.wide = true;
    r.tile_units = 2 * m.nb;
    const int64_t tl = local / r.tile_units;
    r.unit = static_cast<int32_t>(local - tl * r.tile_units);
    r.tile = static_cast<int32_t>(tl / m.nmc);
    r.mc = static_cast<int32_t>(tl - static_cast<int64_t>(r.tile) * m.nmc);
  } else {
    r.wide = false;
    r.tile_units = m.nb;
    const int64_t l2 = local - m.u_wide;
    r.mc = static_cast<int32_t>(l2 / m.nb);
    r.unit = static_cast<int32_t>(l2 - static_cast<int64_t>(r.mc) * m.nb);
    r.tile = m.ntw;
  }
  return r;
}

// CTA whose range holds flat index f (ranges are [floor(i W / G), floor((i+1) W / G))).
__device__ __forceinline__ int64_t cta_of(int64_t f, int64_t W, int64_t G) { return ((f + 1) * G + W - 1) / W - 1; }

__device__ __forceinline__ int64_t range_lo(int64_t i, int64_t W, int64_t G) { return (i * W) / G; }

// One 16-row x 256-column item of a stage, for a consumer warp.
struct Item {
  const uint32_t* q32;  // this lane's word of the item's first row
  int qstride;          // words between rows
  uint32_t zw;          // zero-point word (8 columns)
  const float* sc;      // this lane's 8 scales
  const float* xs;      // x of the item's first row (row stride X_ROWS)
};

__device__ __forceinline__ Item make_item(const uint8_t* st, bool wide, int u0, int j, int sub, int lane) {
  Item it;
  const uint32_t* q = reinterpret_cast<const uint32_t*>(st);
  const float* scs = reinterpret_cast<const float*>(st + QW_STAGE);
  const uint32_t* zps = reinterpret_cast<const uint32_t*>(st + QW_STAGE + SC_STAGE);
  const float* xst = reinterpret_cast<const float*>(st + QW_STAGE + SC_STAGE + ZP_STAGE);
  if (wide) {
    const int slot = ((u0 + j) >> 1) - (u0 >> 1);  // K-block slot in the stage
    it.qstride = 64;
    it.q32 = q + (j * 16) * 64 + sub * 32 + lane;
    it.zw = zps[slot * 64 + sub * 32 + lane];
    it.sc = scs + slot * 512 + sub * 256 + lane * 8;
    it.xs = xst + j * 16;
  } else {
    it.qstride = 32;
    it.q32 = q + (j * 32 + sub * 16) * 32 + lane;
    it.zw = zps[j * 32 + lane];
    it.sc = scs + j * 256 + lane * 8;
    it.xs = xst + j * 32 + sub * 16;
  }
  return it;
}

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
        const CUtensorMap* mp = (lane & 3) == 0   ? &p.mat[g].qw_wide_full
                                : (lane & 3) == 1 ? &p.mat[g].qw_wide_unit
                                : (lane & 3) == 2 ? &p.mat[g].qw_narrow_full
                                                  : &p.mat[g].qw_narrow_unit;
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
      const int64_t seg_end = min(hi, f + (ps.tile_units - ps.unit));
      const int32_t col0 = ps.tile * WIDE_N;
      const int32_t ncols = min(ps.wide ? WIDE_N : NARROW_N, m.N - col0);
      const int32_t mrows = min(MT, m.M - ps.mc * MT);
      const float* xrow0 = m.x + static_cast<int64_t>(ps.mc) * MT * m.ldx;
      int32_t u = ps.unit;
      const int32_t u_end = u + static_cast<int32_t>(seg_end - f);
      while (u < u_end) {
        const int32_t n = min(SU - (u % SU), u_end - u);  // stay on the 8-unit grid
        const bool full_stage = (n == SU);
        const int s = it % C::NSTAGES;
        const uint32_t round = it / C::NSTAGES;
        if (round > 0 && lane == 0)
          ok = mbar_wait_bounded(&empty[s], (round - 1) & 1, p.timeout_ns, abort_flag, p.err, K_GEMV, 1);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        uint8_t* st = smem + s * C::STAGE_BYTES;
        // K-blocks the stage touches and rows of x it needs
        const int32_t b0 = ps.wide ? (u >> 1) : u;
        const int32_t nblk = ps.wide ? (((u + n - 1) >> 1) - b0 + 1) : n;
        const int32_t xrows = ps.wide ? n * 16 : n * 32;
        const int32_t row0 = ps.wide ? u * 16 : u * 32;
        if (lane == 0) {
          const uint32_t bytes = static_cast<uint32_t>(n) * 4096u +
                                 static_cast<uint32_t>(nblk) * static_cast<uint32_t>(ncols * 4 + ncols / 2) +
                                 static_cast<uint32_t>(mrows * xrows * 4);
          mbar_arrive_expect_tx(&full[s], bytes);
        }
        __syncwarp();
        if (full_stage) {
          if (lane == 0)
            tma_g2s_2d(st, ps.wide ? &mp.qw_wide_full : &mp.qw_narrow_full, col0 / 2, row0, &full[s]);
        } else if (lane < n) {
          if (ps.wide)
            tma_g2s_2d(st + lane * 4096, &mp.qw_wide_unit, col0 / 2, (u + lane) * 16, &full[s]);
          else
            tma_g2s_2d(st + lane * 4096, &mp.qw_narrow_unit, col0 / 2, (u + lane) * 32, &full[s]);
        }
        if (lane >= 8 && lane < 8 + nblk) {
          const int32_t sl = lane - 8;
          const int64_t b = b0 + sl;
          const int bsz = ps.wide ? 512 : 256;  // floats per block slot
          bulk_g2s(st + QW_STAGE + sl * bsz * 4, m.scales + b * m.N + col0, ncols * 4, &full[s]);
          bulk_g2s(st + QW_STAGE + SC_STAGE + sl * (bsz / 2), m.zp + (b * m.N + col0) / 2, ncols / 2, &full[s]);
        }
        if (lane >= 16 && lane < 16 + mrows)
          bulk_g2s(st + QW_STAGE + SC_STAGE + ZP_STAGE + (lane - 16) * X_ROWS * 4,
                   xrow0 + static_cast<int64_t>(lane - 16) * m.ldx + row0, xrows * 4, &full[s]);
        ++it;
        u += n;
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
  const int sub = cw & 1;   // column half (wide tiles) or row half (narrow tiles)
  uint32_t kMagic;          // 0x4B000000 (the bits of 2^23) held in a register
  asm("mov.b32 %0, 0x4B000000;" : "=r"(kMagic));
  int it = 0;
  bool ok = true;
  int g_hint = 0;

  int64_t f = lo;
  while (f < hi) {
    const Pos ps = locate(ms, p.count, f, g_hint);
    g_hint = ps.g;
    const MatScalars& m = ms[ps.g];
    const int64_t seg_end = min(hi, f + (ps.tile_units - ps.unit));

    // accumulators: MT <= 2 -> acc[mm*4 + pp] = columns {2pp, 2pp+1} of row mm
    //               MT >= 4 -> this warp's slice red[cw][mm][256] in shared memory
    constexpr int NACC = C::SMEM_ACC ? 1 : MT * 4;
    float2 acc[NACC];
#pragma unroll
    for (int i = 0; i < NACC; ++i) acc[i] = make_float2(0.f, 0.f);
    float* wacc = red + cw * (C::SMEM_ACC ? MT : 1) * 256 + lane * 8;
    if constexpr (C::SMEM_ACC) {
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) {
        reinterpret_cast<float4*>(wacc + mm * 256)[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4*>(wacc + mm * 256)[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }

    int32_t u = ps.unit;
    const int32_t u_end = u + static_cast<int32_t>(seg_end - f);
    while (u < u_end) {
      const int32_t n = min(SU - (u % SU), u_end - u);  // same grid as the producer
      const int s = it % C::NSTAGES;
      const uint32_t round = it / C::NSTAGES;
      if (ok) ok = mbar_wait_bounded(&full[s], round & 1, p.timeout_ns, abort_flag, p.err, K_GEMV, 3);
#pragma unroll
      for (int ii = 0; ii < C::IPW; ++ii) {
        const int j = (cw >> 1) + ii * (C::NCW >> 1);  // unit of the stage for this item
        if (!(ok && j < n)) continue;
        const Item item = make_item(smem + s * C::STAGE_BYTES, ps.wide, u, j, sub, lane);
        const float4 sa = reinterpret_cast<const float4*>(item.sc)[0];
        const float4 sb = reinterpret_cast<const float4*>(item.sc)[1];
        const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
        float ncz[8], sp[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          ncz[i] = -magic_nib(i < 4 ? item.zw : (item.zw >> 16), i & 3);
          sp[i] = sv[i] * inv_slot_scale(i & 3);
        }
        if constexpr (MT == 1) {
          // scalar fp32: per weight one LOP3 (ALU pipe), one FADD and one FFMA
          float P[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) P[i] = 0.f;
#pragma unroll
          for (int r4 = 0; r4 < 16; r4 += 4) {
            const float4 x4 = *reinterpret_cast<const float4*>(item.xs + r4);
            const float xr[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
              const uint32_t a = item.q32[(r4 + rr) * item.qstride];
              const uint32_t b = a >> 16;
#pragma unroll
              for (int i = 0; i < 8; ++i) P[i] = fmaf(xr[rr], magic_nib_r(i < 4 ? a : b, kMagic, i & 3) + ncz[i], P[i]);
            }
          }
#pragma unroll
          for (int pp = 0; pp < 4; ++pp) {
            acc[pp].x = fmaf(P[2 * pp], sp[2 * pp], acc[pp].x);
            acc[pp].y = fmaf(P[2 * pp + 1], sp[2 * pp + 1], acc[pp].y);
          }
        } else {
          float2 P[MT * 4];
#pragma unroll
          for (int i = 0; i < MT * 4; ++i) P[i] = make_float2(0.f, 0.f);
#pragma unroll 4
          for (int r = 0; r < 16; ++r) {
            const uint32_t a = item.q32[r * item.qstride];
            const uint32_t b = a >> 16;
            float wv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) wv[i] = (magic_nib_r(i < 4 ? a : b, kMagic, i & 3) + ncz[i]) * sp[i];
#pragma unroll
            for (int mm = 0; mm < MT; ++mm) {
              const float xv = item.xs[mm * X_ROWS + r];
#pragma unroll
              for (int pp = 0; pp < 4; ++pp) {
                P[mm * 4 + pp].x = fmaf(xv, wv[2 * pp], P[mm * 4 + pp].x);
                P[mm * 4 + pp].y = fmaf(xv, wv[2 * pp + 1], P[mm * 4 + pp].y);
              }
            }
          }
          if constexpr (C::SMEM_ACC) {
#pragma unroll
            for (int mm = 0; mm < MT; ++mm) {
              float4* a4 = reinterpret_cast<float4*>(wacc + mm * 256);
              float4 va = a4[0], vb = a4[1];
              va.x += P[mm * 4 + 0].x; va.y += P[mm * 4 + 0].y; va.z += P[mm * 4 + 1].x; va.w += P[mm * 4 + 1].y;
              vb.x += P[mm * 4 + 2].x; vb.y += P[mm * 4 + 2].y; vb.z += P[mm * 4 + 3].x; vb.w += P[mm * 4 + 3].y;
              a4[0] = va;
              a4[1] = vb;
            }
          } else {
#pragma unroll
            for (int i = 0; i < MT * 4; ++i) {
              acc[i].x += P[i].x;
              acc[i].y += P[i].y;
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      ++it;
      u += n;
    }

    // ---- segment done: reduce the warps' partials, then write or fix up
    const int32_t col0 = ps.tile * WIDE_N;
    const int32_t wt = ps.wide ? WIDE_N : NARROW_N;
    const int32_t mc = ps.mc;
    const int64_t t_start = f - ps.unit;
    const int64_t c_first = cta_of(t_start, p.W, G);
    const int64_t c_last = cta_of(t_start + ps.tile_units - 1, p.W, G);
    const bool split = c_first != c_last;
    const int slot = (split && static_cast<int64_t>(blockIdx.x) == c_first && lo < t_start) ? 1 : 0;
#pragma unroll
    for (int mm = 0; mm < MT; ++mm) {
      if constexpr (!C::SMEM_ACC) {
        float4* dst = reinterpret_cast<float4*>(wacc);
        dst[0] = make_float4(acc[mm * 4 + 0].x, acc[mm * 4 + 0].y, acc[mm * 4 + 1].x, acc[mm * 4 + 1].y);
        dst[1] = make_float4(acc[mm * 4 + 2].x, acc[mm * 4 + 2].y, acc[mm * 4 + 3].x, acc[mm * 4 + 3].y);
      }
      named_bar_sync(1, C::NCW * 32);
      for (int c = ctid; c < wt; c += C::NCW * 32) {
        const int cg = ps.wide ? (c >> 8) : -1;  // column half that owns column c (wide tiles)
        const int cc = c & 255;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < C::NCW; ++w)
          if (cg < 0 || (w & 1) == cg)
            v += red[(w * (C::SMEM_ACC ? MT : 1) + (C::SMEM_ACC ? mm : 0)) * 256 + cc];
        const int32_t row = mc * MT + mm;
        const int64_t gcol = static_cast<int64_t>(col0) + c;
        if (!split) {
          if (ok && row < m.M && gcol < m.N) m.y[static_cast<int64_t>(row) * m.ldy + gcol] = v;
        } else {
          p.ws_partials[((static_cast<int64_t>(blockIdx.x) * 2 + slot) * MT + mm) * WIDE_N + c] = v;
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
        for (int mm = 0; mm < MT; ++mm) {
          for (int c = ctid; c < wt; c += C::NCW * 32) {
            float v = 0.f;
            for (int64_t cc = c_first; cc <= c_last; ++cc) {
              const int sl = (cc == c_first && range_lo(cc, p.W, G) < t_start) ? 1 : 0;
              v += __ldcg(&p.ws_partials[((cc * 2 + sl) * MT + mm) * WIDE_N + c]);
            }
            const int32_t row = mc * MT + mm;
            const int64_t gcol = static_cast<int64_t>(col0) + c;
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

// Column tiling of one weight: ntw wide tiles (the last possibly partial) and
// an optional narrow tile for a remainder of at most 256 columns.
void tiling(int64_t N, int32_t* ntw, int32_t* narrow) {
  int64_t w = N / WIDE_N;
  const int64_t rem = N - w * WIDE_N;
  int32_t nar = 0;
  if (rem > NARROW_N) ++w;
  else if (rem > 0) nar = 1;
  *ntw = static_cast<int32_t>(w);
  *narrow = nar;
}

struct Plan {
  int mt = 1;
  int64_t W = 0;
  int grid = 0;
};

// Workspace: [COUNTER_SLOTS int32 counters][grid][2][MT][WIDE_N] fp32 partials.
constexpr int COUNTER_SLOTS = 1024;  // >= grid (one per CTA)
constexpr size_t COUNTER_BYTES = COUNTER_SLOTS * sizeof(int32_t);

Plan make_plan(const w4_desc* d, int count, int sms) {
  Plan pl;
  pl.mt = pick_mt(d, count);
  for (int i = 0; i < count; ++i) {
    if (d[i].M == 0 || d[i].N == 0 || d[i].K == 0) continue;
    int32_t ntw, nar;
    tiling(d[i].N, &ntw, &nar);
    const int64_t nmc = (d[i].M + pl.mt - 1) / pl.mt;
    const int64_t nb = d[i].K / 32;
    pl.W += nmc * (static_cast<int64_t>(ntw) * 2 * nb + nar * nb);
  }
  pl.grid = static_cast<int>(std::min<int64_t>(std::min(sms, COUNTER_SLOTS), pl.W));
  return pl;
}

size_t ws_bytes(const Plan& pl) {
  if (pl.W == 0) return 0;
  return COUNTER_BYTES + static_cast<size_t>(pl.grid) * 2 * pl.mt * WIDE_N * sizeof(float);
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
  if (d.K > (int64_t(1) << 30) || d.N > (int64_t(1) << 30)) {
    *why = "the GEMV path needs K and N below 2^30";
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
  int64_t uoff = 0;
  for (int i = 0; i < count; ++i) {
    const w4_desc& s = d[i];
    if (s.M == 0 || s.N == 0 || s.K == 0) continue;
    MatParams& mpar = prm.mat[g];
    w4_status rc = encode_w4_maps(&mpar.qw_wide_full, &mpar.qw_wide_unit, &mpar.qw_narrow_full, &mpar.qw_narrow_unit,
                                  s.qw, s.K, s.N);
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
    tiling(s.N, &m.ntw, &m.narrow);
    m.nmc = static_cast<int32_t>((s.M + pl.mt - 1) / pl.mt);
    m.u_off = uoff;
    m.u_wide = static_cast<int64_t>(m.ntw) * m.nmc * 2 * m.nb;
    uoff += m.u_wide + static_cast<int64_t>(m.narrow) * m.nmc * m.nb;
    ++g;
  }
  prm.count = g;
  prm.W = uoff;
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
