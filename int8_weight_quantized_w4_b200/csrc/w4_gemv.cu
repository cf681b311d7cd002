// w4_gemv: y = x . W for small M (decode), W in the 4-bit blocked format of
// "ONNX export, quantization and the browser runtime", section
// "Quantization (train/quantize.py)", step 2 (dq4): blocks of 32 along K,
// fp32 scale and uint4 zero point per (block, column), w = (q - zp) * scale.
//
// Design (sm_100a):
//  * Column tiles are 512 columns wide (256-byte row pieces, which stream at
//    full HBM speed where 128-byte pieces do not); the last 256 or fewer
//    columns of a weight may form a narrow 256-column tile instead. A weight
//    whose wide tiles would be taller than about two CTAs' shares is cut into
//    narrow tiles only, so that no tile holds more than one CTA's whole range.
//  * Work is counted in units of 4 KB of nibbles: 16 rows of a wide tile or
//    32 rows (one K-block) of a narrow one. All matrices of a launch form one
//    flat range of units; CTA i (one per SM, persistent) takes
//    [i*W/G, (i+1)*W/G), so every SM streams the same bytes (stream-K).
//  * A tile whose K-range straddles CTAs is finished by one of them, chosen on
//    the host (a CTA whose whole range lies inside the tile, if any; else one
//    of the two, so that no CTA publishes more than about half of its range).
//    Every other
//    contributor writes its partial sums to one of its two workspace slots and
//    bumps a counter (indexed by the tile's first CTA); the finisher waits
//    (bounded) until the count is complete, adds the others' partials in CTA
//    order to its own and resets the counter to zero. The launch is
//    cooperative, so all CTAs are resident and the finisher's wait ends.
//  * A CTA walks its range as segments (one tile each): the pieces it
//    publishes first, then its whole tiles, then the pieces it finishes. Partials are therefore published
//    early, and the finisher's epilogue warp
//    collects them before it needs them: a round trip to global memory while
//    every SM streams takes microseconds, and none is left on the finisher's
//    path at the end.
//  * Warp-specialised: warp 0 is the producer. A stage holds 8 units and is
//    aligned to the tile's 8-unit grid; a full stage is one 2-D tensor copy of
//    the nibbles (128 rows x 256 B or 256 rows x 128 B), one bulk copy per
//    K-block of scales and of zero points, and one per row of x, issued by
//    several lanes at once. A partial stage (at the ends of a segment)
//    copies unit by unit. Stages form a ring of three guarded by mbarriers; no copy
//    uses multicast. Eight consumer warps dequantise in registers: each takes
//    16 rows x 256 columns of a stage, a lane owning 8 columns.
//  * M <= 2: two epilogue warps finish segments (sum over the consumer warps,
//    write y or publish a partial and take part in the fix-up) while the
//    consumers go on with the next segment; the consumers hand their sums
//    over in one of two shared-memory buffers, guarded by mbarriers.
//    M >= 4: accumulators live in shared memory and the consumers finish
//    each segment themselves.
//  * Dequantisation uses the exponent trick of w4_device.cuh: one LOP3 per
//    weight builds 2^23 + q*16^j, a subtraction of the matching zero-point
//    float gives (q - zp)*16^j exactly, one FMA accumulates.
//  * MT = 1: rows are taken in pairs (k, k+1) so that the subtraction and the
//    FMA are packed f32x2 instructions (FADD2, FFMA2) with x[k], x[k+1] as
//    one operand; the two halves are added at the end of a 16-row slice and
//    the scale is applied once per slice (s * sum x (q - zp)).
//    MT >= 2: the weight is dequantised to fp32 exactly as the oracle does
//    ((q - zp) * s, one rounding) and reused for the MT rows of x.
//  * The walk over segments (locate, seg_init, seg_next, seg_info) is inlined
//    into each warp role: at kernel start a call into not-yet-fetched code
//    costs about a microsecond of instruction fetch, and these calls sit on
//    the producer's path to its first copy.
//  * Accumulation is per 16-row slice, then across stages, then across
//    warps, then across CTAs: all fp32, all in a fixed order.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <memory>
#include <vector>

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
constexpr int GRID_MAX = 256;        // CTAs per launch, at most

// Per-matrix fields the kernel reads while walking its range. Each CTA copies
// those of the matrices its range touches from the parameter block into
// shared memory once: dynamically indexed reads of a large parameter block
// miss the constant cache.
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
  int32_t nnar;    // narrow tiles after them (the last may be partial)
  int32_t nmc;     // groups of MT rows
  int32_t pad;
  Epi epi;         // fused epilogue of the final store
};
static_assert(sizeof(MatScalars) % 8 == 0, "copied as 8-byte words");
constexpr int MS_WORDS = sizeof(MatScalars) / 8;
static_assert(MS_WORDS <= 32, "one lane per word");

struct MatParams {
  CUtensorMap qw_wide_full;    // [K rows][N/2 bytes], box 128 rows x 256 B
  CUtensorMap qw_wide_unit;    // box 16 rows x 256 B
  CUtensorMap qw_narrow_full;  // box 256 rows x 128 B
  CUtensorMap qw_narrow_unit;  // box 32 rows x 128 B
  MatScalars s;
};

struct GemvParams {
  MatParams mat[W4_GROUP_MAX];
  uint8_t cta_g[GRID_MAX][2];  // first and last matrix that each CTA's range touches
  // Split-tile roles of each CTA: bit 0 set when it finishes the tile holding
  // its first unit, bit 1 the tile holding its last unit (only meaningful
  // when that tile straddles CTAs). Chosen on the host, see cta_roles().
  uint8_t cta_fin[GRID_MAX];
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
  static constexpr bool ASYNC = MT <= 2;          // epilogue warps finish segments
  static constexpr int NEPI = ASYNC ? 2 : 0;      // epilogue warps
  static constexpr int NTHREADS = (1 + NCW + NEPI) * 32;
  static constexpr int X_STAGE = MT * X_ROWS * 4;
  static constexpr int STAGE_BYTES = QW_STAGE + SC_STAGE + ZP_STAGE + X_STAGE;
  static constexpr int NSTAGES = 3;  // measured best for the GPT-2 body (3 vs 4 stages)
  // per-warp column sums [NCW][MT][256]: handed to the epilogue warps (two
  // buffers, M <= 2) or the accumulators themselves (one buffer, M >= 4)
  static constexpr int RED_FLOATS = NCW * MT * 256;
  static constexpr int NRED = ASYNC ? 2 : 1;
  static constexpr int RED_OFF = NSTAGES * STAGE_BYTES;
  // owner's gathered sums [NEPI][MT][512] (epilogue warps only)
  static constexpr int OWN_OFF = RED_OFF + NRED * RED_FLOATS * 4;
  static constexpr int SCAL_OFF = OWN_OFF + NEPI * MT * WIDE_N * 4;
  static constexpr int BAR_OFF = SCAL_OFF + W4_GROUP_MAX * static_cast<int>(sizeof(MatScalars));
  static constexpr int NBARS = 2 * NSTAGES + 4;  // full, empty, red_full[2], red_empty[2]
  static constexpr int SMEM_BYTES = BAR_OFF + NBARS * 8 + 64;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory of one CTA");
};

// Flat unit f -> (matrix, tile, group of rows, unit within the tile).
struct Pos {
  int g;
  bool wide;
  int32_t col0;       // first column of the tile (wide tiles first, then narrow ones)
  int32_t mc;         // group of MT rows of x
  int32_t unit;       // unit within the tile
  int32_t tile_units; // 2*nb (wide) or nb (narrow)
};

// g is a matrix at or before the one holding f; g_hi the last this CTA touches.
__device__ __forceinline__ Pos locate(const MatScalars* ms, int g_hi, int64_t f, int g) {
#pragma unroll 1
  while (g < g_hi && ms[g + 1].u_off <= f) ++g;
  const MatScalars& m = ms[g];
  const int64_t local = f - m.u_off;
  Pos r;
  r.g = g;
  if (local < m.u_wide) {
    r.wide = true;
    r.tile_units = 2 * m.nb;
    const int64_t tl = static_cast<uint32_t>(local) / static_cast<uint32_t>(r.tile_units);
    r.unit = static_cast<int32_t>(local - tl * r.tile_units);
    const int32_t tile = static_cast<int32_t>(static_cast<uint32_t>(tl) / static_cast<uint32_t>(m.nmc));
    r.mc = static_cast<int32_t>(tl - static_cast<int64_t>(tile) * m.nmc);
    r.col0 = tile * WIDE_N;
  } else {
    r.wide = false;
    r.tile_units = m.nb;
    const int64_t l2 = local - m.u_wide;
    const int64_t tl = static_cast<uint32_t>(l2) / static_cast<uint32_t>(m.nb);
    r.unit = static_cast<int32_t>(l2 - tl * m.nb);
    const int32_t tile = static_cast<int32_t>(static_cast<uint32_t>(tl) / static_cast<uint32_t>(m.nmc));
    r.mc = static_cast<int32_t>(tl - static_cast<int64_t>(tile) * m.nmc);
    r.col0 = m.ntw * WIDE_N + tile * NARROW_N;
  }
  return r;
}

// CTA whose range holds flat index f (ranges are [floor(i W / G), floor((i+1) W / G))).
// The host guarantees W * G < 2^32, so every product here fits 32 bits and the
// divisions are 32-bit ones (a 64-bit division is a long subroutine, and these
// sit on the path to a CTA's first copy).
__device__ __forceinline__ int64_t cta_of(int64_t f, int64_t W, int64_t G) {
  return static_cast<uint32_t>((f + 1) * G + W - 1) / static_cast<uint32_t>(W) - 1;
}

__device__ __forceinline__ int64_t range_lo(int64_t i, int64_t W, int64_t G) {
  return static_cast<uint32_t>(i * W) / static_cast<uint32_t>(G);
}

// The segments of a CTA's range [lo, hi), in processing order. The piece at
// the start (up to the end of the tile holding lo) and the piece at the end
// (from the start of the tile holding hi-1) each go first when this CTA
// publishes them and last when it finishes their tile; the whole tiles in
// between go in the middle. A range inside one tile is a single segment.
// Producer, consumers and epilogue warps walk the same sequence.
struct SegIter {
  int64_t lo, hi;
  int64_t hd_end;    // end of the first piece
  int64_t tl_start;  // start of the last piece (hi when there is none)
  int64_t f;         // cursor over the whole tiles between
  int k;             // 0 head-early, 1 tail-early, 2 middle, 3 head-late, 4 tail-late, 5 done
  bool head_late, tail_late;
  int g1, gm;        // last matrix of the range; cursor hint
};

__device__ __forceinline__ void seg_init(SegIter& it, const MatScalars* ms, int g0, int g1, int64_t lo, int64_t hi,
                                      int fin) {
  it.lo = lo;
  it.hi = hi;
  it.k = 0;
  it.g1 = g1;
  it.head_late = false;
  it.tail_late = false;
  const Pos a = locate(ms, g1, lo, g0);
  it.gm = a.g;
  it.hd_end = min(hi, lo - a.unit + a.tile_units);
  if (it.hd_end == hi) {
    it.tl_start = hi;
  } else {
    if (a.unit > 0) it.head_late = (fin & 1) != 0;
    const Pos b = locate(ms, g1, hi - 1, a.g);
    it.tl_start = hi - 1 - b.unit;
    // a last piece that is a whole tile waits for nobody: it may as well go last
    it.tail_late = it.tl_start + b.tile_units == hi || (fin & 2) != 0;
  }
  it.f = it.hd_end;
}

__device__ __forceinline__ bool seg_next(SegIter& it, const MatScalars* ms, int64_t& a, int64_t& b) {
  if (it.hd_end == it.hi) {  // a single segment
    if (it.k++ > 0) return false;
    a = it.lo;
    b = it.hi;
    return true;
  }
  while (it.k < 5) {
    switch (it.k) {
      case 0:
        it.k = 1;
        if (!it.head_late) {
          a = it.lo;
          b = it.hd_end;
          return true;
        }
        break;
      case 1:
        it.k = 2;
        if (!it.tail_late) {
          a = it.tl_start;
          b = it.hi;
          return true;
        }
        break;
      case 2:
        if (it.f < it.tl_start) {
          const Pos p = locate(ms, it.g1, it.f, it.gm);
          it.gm = p.g;
          a = it.f;
          b = it.f + p.tile_units;  // f is at a tile start
          it.f = b;
          return true;
        }
        it.k = 3;
        break;
      case 3:
        it.k = 4;
        if (it.head_late) {
          a = it.lo;
          b = it.hd_end;
          return true;
        }
        break;
      default:
        it.k = 5;
        if (it.tail_late) {
          a = it.tl_start;
          b = it.hi;
          return true;
        }
        break;
    }
  }
  return false;
}

// One 16-row x 256-column item of a stage, for a consumer warp. Rows of a
// wide stage are 64 words apart, of a narrow one 32.
struct Item {
  const uint32_t* q32;  // this lane's word of the item's first row
  uint32_t zw;          // zero-point word (8 columns)
  const float* sc;      // this lane's 8 scales
  const float* xs;      // x of the item's first row (row stride X_ROWS)
};

template <bool WIDE>
__device__ __forceinline__ Item make_item(const uint8_t* st, int u0, int j, int sub, int lane) {
  Item it;
  const uint32_t* q = reinterpret_cast<const uint32_t*>(st);
  const float* scs = reinterpret_cast<const float*>(st + QW_STAGE);
  const uint32_t* zps = reinterpret_cast<const uint32_t*>(st + QW_STAGE + SC_STAGE);
  const float* xst = reinterpret_cast<const float*>(st + QW_STAGE + SC_STAGE + ZP_STAGE);
  if (WIDE) {
    const int slot = ((u0 + j) >> 1) - (u0 >> 1);  // K-block slot in the stage
    it.q32 = q + (j * 16) * 64 + sub * 32 + lane;
    it.zw = zps[slot * 64 + sub * 32 + lane];
    it.sc = scs + slot * 512 + sub * 256 + lane * 8;
    it.xs = xst + j * 16;
  } else {
    it.q32 = q + (j * 32 + sub * 16) * 32 + lane;
    it.zw = zps[j * 32 + lane];
    it.sc = scs + j * 256 + lane * 8;
    it.xs = xst + j * 32 + sub * 16;
  }
  return it;
}

// The items of one stage for consumer warp cw: MT <= 2 accumulates into
// acc[mm*4 + pp] (columns {2pp, 2pp+1} of row mm), MT >= 4 into the warp's
// shared-memory slice wacc[mm*256 + 0..7].
template <int MT, bool WIDE, int NCW, int IPW>
__device__ __forceinline__ void stage_items(const uint8_t* st, int u, int n, int cw, int sub, int lane,
                                            uint32_t kMagic, float2* acc, float* wacc) {
  constexpr int QS = WIDE ? 64 : 32;
#pragma unroll
  for (int ii = 0; ii < IPW; ++ii) {
    const int j = (cw >> 1) + ii * (NCW >> 1);  // unit of the stage for this item
    if (j >= n) continue;
    const Item item = make_item<WIDE>(st, u, j, sub, lane);
    const float4 sa4 = reinterpret_cast<const float4*>(item.sc)[0];
    const float4 sb4 = reinterpret_cast<const float4*>(item.sc)[1];
    const float sv[8] = {sa4.x, sa4.y, sa4.z, sa4.w, sb4.x, sb4.y, sb4.z, sb4.w};
    float sp[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) sp[i] = sv[i] * inv_slot_scale(i & 3);
    if constexpr (MT == 1) {
      // rows in pairs: per weight one LOP3, half an FADD2, half an FFMA2
      float2 nz[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float z = -magic_nib(i < 4 ? item.zw : (item.zw >> 16), i & 3);
        nz[i] = make_float2(z, z);
      }
      float2 P[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) P[i] = make_float2(0.f, 0.f);
#pragma unroll
      for (int r = 0; r < 16; r += 4) {
        const float4 x4 = *reinterpret_cast<const float4*>(item.xs + r);
        const float2 xa = make_float2(x4.x, x4.y);
        const float2 xb = make_float2(x4.z, x4.w);
        uint32_t wl[4], wh[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          wl[t] = item.q32[(r + t) * QS];
          wh[t] = __umulhi(wl[t], 65536u);  // = wl >> 16, issued on the FMA pipe, not the integer ALU
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int sl = i & 3;
          const float2 m01 = make_float2(magic_nib_r(i < 4 ? wl[0] : wh[0], kMagic, sl),
                                         magic_nib_r(i < 4 ? wl[1] : wh[1], kMagic, sl));
          const float2 m23 = make_float2(magic_nib_r(i < 4 ? wl[2] : wh[2], kMagic, sl),
                                         magic_nib_r(i < 4 ? wl[3] : wh[3], kMagic, sl));
          P[i] = __ffma2_rn(xa, __fadd2_rn(m01, nz[i]), P[i]);
          P[i] = __ffma2_rn(xb, __fadd2_rn(m23, nz[i]), P[i]);
        }
      }
#pragma unroll
      for (int pp = 0; pp < 4; ++pp) {
        acc[pp].x = fmaf(P[2 * pp].x + P[2 * pp].y, sp[2 * pp], acc[pp].x);
        acc[pp].y = fmaf(P[2 * pp + 1].x + P[2 * pp + 1].y, sp[2 * pp + 1], acc[pp].y);
      }
    } else {
      // columns in pairs: the packed f32x2 add, multiply and FMA do per
      // element exactly what the scalar ones do, in half the instructions
      float2 ncz[4], sp2[4];
#pragma unroll
      for (int pp = 0; pp < 4; ++pp) {
        const int i0 = 2 * pp, i1 = 2 * pp + 1;
        ncz[pp] = make_float2(-magic_nib(i0 < 4 ? item.zw : (item.zw >> 16), i0 & 3),
                              -magic_nib(i1 < 4 ? item.zw : (item.zw >> 16), i1 & 3));
        sp2[pp] = make_float2(sp[i0], sp[i1]);
      }
      float2 P[MT * 4];
#pragma unroll
      for (int i = 0; i < MT * 4; ++i) P[i] = make_float2(0.f, 0.f);
#pragma unroll 4
      for (int r = 0; r < 16; ++r) {
        const uint32_t a = item.q32[r * QS];
        const uint32_t b = a >> 16;
        float2 wv[4];  // (q - zp) * s of columns 2pp, 2pp + 1: one rounding, as the page's w
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          const int i0 = 2 * pp, i1 = 2 * pp + 1;
          const float2 m = make_float2(magic_nib_r(i0 < 4 ? a : b, kMagic, i0 & 3),
                                       magic_nib_r(i1 < 4 ? a : b, kMagic, i1 & 3));
          wv[pp] = __fmul2_rn(__fadd2_rn(m, ncz[pp]), sp2[pp]);
        }
#pragma unroll
        for (int mm = 0; mm < MT; ++mm) {
          const float xv = item.xs[mm * X_ROWS + r];
          const float2 x2 = make_float2(xv, xv);
#pragma unroll
          for (int pp = 0; pp < 4; ++pp) P[mm * 4 + pp] = __ffma2_rn(x2, wv[pp], P[mm * 4 + pp]);
        }
      }
      if constexpr (MT >= 4) {
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
}

__device__ __forceinline__ int ld_acquire_gpu(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// What the finishing threads need to know about a segment.
struct SegInfo {
  const MatScalars* m;
  int32_t col0;  // first column of the tile
  int32_t wt;    // columns of the tile (512 or 256)
  int32_t mc;
  bool wide;
  bool split;    // the tile straddles CTAs
  bool owner;    // ... and this CTA finishes it
  int64_t c_first, c_last;
};

// a: first unit of the segment; lo: first unit of this CTA's range; fin: its role bits.
__device__ __forceinline__ SegInfo seg_info(const MatScalars* ms, const Pos& ps, int64_t a, int64_t lo, int fin,
                                         int64_t W, int64_t G) {
  SegInfo s;
  s.m = &ms[ps.g];
  s.col0 = ps.col0;
  s.wt = ps.wide ? WIDE_N : NARROW_N;
  s.mc = ps.mc;
  s.wide = ps.wide;
  const int64_t t_start = a - ps.unit;
  s.c_first = cta_of(t_start, W, G);
  s.c_last = cta_of(t_start + ps.tile_units - 1, W, G);
  s.split = s.c_first != s.c_last;
  s.owner = s.split && (fin & (a == lo ? 1 : 2)) != 0;
  return s;
}

// Partial of contributor cta to a tile whose first CTA is c_first: slot 1 for
// the piece at the end of cta's range (cta == c_first), slot 0 for the piece
// at its start or a range inside the tile.
__device__ __forceinline__ float* partial_at(const GemvParams& p, int64_t cta, int64_t c_first, int mt, int mm, int c) {
  return p.ws_partials + ((cta * 2 + (cta == c_first ? 1 : 0)) * mt + mm) * WIDE_N + c;
}

// Owner of a split tile: wait (bounded) until every other contributor has
// published (thread 0 polls; the result goes to all NT threads). Returns
// false on timeout or abort.
template <int NT, class Sync, class Bcast>
__device__ __forceinline__ bool owner_wait(const SegInfo& s, int tid, const GemvParams& p, volatile int* abort,
                                           Sync sync, Bcast bcast) {
  int32_t* ctr = p.ws_counters + s.c_first;
  const int need = static_cast<int>(s.c_last - s.c_first);
  int okv = 1;
  if (tid == 0) {
    const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
    while (ld_acquire_gpu(ctr) != need) {
      if (*abort) {
        okv = 0;
        break;
      }
      if (globaltimer_ns() - t0 > p.timeout_ns) {
        *abort = 1;
        record_error(p.err, W4_ERR_TIMEOUT, K_GEMV, 6);
        okv = 0;
        break;
      }
      __nanosleep(200);
    }
  }
  okv = bcast(okv);
  sync();  // orders the other threads' reads after thread 0's acquire
  return okv != 0;
}

// Sum of the other contributors' partials of row mm, columns tid + i*NT, in
// CTA order (skipping this CTA, the finisher): one contributor at a time, all of its columns in flight at once.
template <int MT, int NT>
__device__ __forceinline__ void gather_row(const SegInfo& s, int tid, const GemvParams& p, int mm,
                                           float (&t)[WIDE_N / NT]) {
  constexpr int PER = WIDE_N / NT;
#pragma unroll
  for (int i = 0; i < PER; ++i) t[i] = 0.f;
#pragma unroll 1
  for (int64_t cc = s.c_first; cc <= s.c_last; ++cc) {
    if (cc == static_cast<int64_t>(blockIdx.x)) continue;
    float q[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int c = tid + i * NT;
      q[i] = c < s.wt ? __ldcg(partial_at(p, cc, s.c_first, MT, mm, c)) : 0.f;
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) t[i] += q[i];
  }
}

// Owner, ahead of time (epilogue warp): wait, gather every row into S
// ([MT][512] in shared memory), reset the counter.
template <int MT, int NT, class Sync, class Bcast>
__device__ __noinline__ bool owner_prefetch(const SegInfo& s, int tid, const GemvParams& p, float* S,
                                            volatile int* abort, Sync sync, Bcast bcast) {
  if (!owner_wait<NT>(s, tid, p, abort, sync, bcast)) return false;
#pragma unroll 1
  for (int mm = 0; mm < MT; ++mm) {
    float t[WIDE_N / NT];
    gather_row<MT, NT>(s, tid, p, mm, t);
#pragma unroll
    for (int i = 0; i < WIDE_N / NT; ++i) S[mm * WIDE_N + tid + i * NT] = t[i];
  }
  sync();
  if (tid == 0) *(p.ws_counters + s.c_first) = 0;  // all have counted: nobody else touches it in this launch
  return true;
}

// Finish one segment with NT threads: sum the consumer warps' column sums in
// `red` ([NCW][MT][256]), then write y (whole tile), publish a partial
// (split, not owner) or add the others' partials and write y (owner: from S
// in shared memory when the epilogue warp gathered them ahead, else loaded
// here after owner_wait). release() is called once `red` has been read.
// Memory writes are skipped when ok is false; the barriers are not.
template <int MT, int NCW, int NT, class Sync, class Release>
__device__ __forceinline__ void finish_segment(const float* red, const SegInfo& s, int tid, bool ok,
                                               const GemvParams& p, const float* S, Sync sync, Release release) {
  constexpr int PER = WIDE_N / NT;
  const MatScalars& m = *s.m;
  const bool publish = s.split && !s.owner;
  const int nrows = min(MT, m.M - s.mc * MT);
#pragma unroll 1
  for (int mm = 0; mm < MT; ++mm) {
    float v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int c = tid + i * NT;
      const int cg = s.wide ? (c >> 8) : -1;  // column half that owns column c (wide tiles)
      float t = 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w)
        if (cg < 0 || (w & 1) == cg) t += red[(w * MT + mm) * 256 + (c & 255)];
      v[i] = t;
    }
    if (!ok || mm >= nrows) continue;
    if (publish) {
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int c = tid + i * NT;
        if (c < s.wt) *partial_at(p, blockIdx.x, s.c_first, MT, mm, c) = v[i];
      }
    } else {
      if (s.owner) {
        if (S != nullptr) {
#pragma unroll
          for (int i = 0; i < PER; ++i) v[i] += S[mm * WIDE_N + tid + i * NT];
        } else {
          float t[PER];
          gather_row<MT, NT>(s, tid, p, mm, t);
#pragma unroll
          for (int i = 0; i < PER; ++i) v[i] += t[i];
        }
      }
      const int64_t row = static_cast<int64_t>(s.mc * MT + mm);
      float* yrow = m.y + row * m.ldy + s.col0;
      const int ncol = min(s.wt, m.N - s.col0);
      if (epi_active(m.epi)) {
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int c = tid + i * NT;
          if (c < ncol) yrow[c] = epi_apply(v[i], m.epi, row, s.col0 + c);
        }
      } else {
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int c = tid + i * NT;
          if (c < ncol) yrow[c] = v[i];
        }
      }
    }
  }
  release();
  if (publish) {
    __threadfence();
    sync();
    if (tid == 0 && ok) atomicAdd(p.ws_counters + s.c_first, 1);
  } else if (s.owner && S == nullptr) {
    sync();
    if (tid == 0) *(p.ws_counters + s.c_first) = 0;
  }
}

template <int MT>
__global__ void __launch_bounds__(Cfg<MT>::NTHREADS, 1) w4_gemv_kernel(const __grid_constant__ GemvParams p) {
  using C = Cfg<MT>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + C::NSTAGES;
  uint64_t* red_full = empty + C::NSTAGES;
  uint64_t* red_empty = red_full + 2;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(red_empty + 2);
  int* bcast_slot = reinterpret_cast<int*>(red_empty + 2) + 4;
  float* red = reinterpret_cast<float*>(smem + C::RED_OFF);
  float* own = reinterpret_cast<float*>(smem + C::OWN_OFF);
  MatScalars* ms = reinterpret_cast<MatScalars*>(smem + C::SCAL_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t lo = range_lo(blockIdx.x, p.W, G);
  const int64_t hi = range_lo(blockIdx.x + 1, p.W, G);
  const int g0 = p.cta_g[blockIdx.x][0];
  const int g1 = p.cta_g[blockIdx.x][1];

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::NCW);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&red_full[b], C::NCW);
      mbar_init(&red_empty[b], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // scalars of the matrices this range touches: a warp per matrix, a lane per word
  for (int g = g0 + warp; g <= g1; g += C::NTHREADS / 32)
    if (lane < MS_WORDS)
      reinterpret_cast<uint64_t*>(ms + g)[lane] = reinterpret_cast<const uint64_t*>(&p.mat[g].s)[lane];
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int it = 0;
    bool ok = true;
    SegIter si;
    seg_init(si, ms, g0, g1, lo, hi, p.cta_fin[blockIdx.x]);
    int64_t sa, sb;
    while (ok && seg_next(si, ms, sa, sb)) {
      const Pos ps = locate(ms, g1, sa, g0);
      const MatScalars& m = ms[ps.g];
      const MatParams& mp = p.mat[ps.g];
      const int32_t col0 = ps.col0;
      const int32_t ncols = min(ps.wide ? WIDE_N : NARROW_N, m.N - col0);
      const int32_t mrows = min(MT, m.M - ps.mc * MT);
      const float* xrow0 = m.x + static_cast<int64_t>(ps.mc) * MT * m.ldx;
      int32_t u = ps.unit;
      const int32_t u_end = u + static_cast<int32_t>(sb - sa);
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

  if (warp > C::NCW) {
    // ------------------------------------------------------- epilogue warps
    if constexpr (C::ASYNC) {
      const int e = warp - 1 - C::NCW;  // takes segments k with k % 2 == e, in buffer e
      const float* rb = red + e * C::RED_FLOATS;
      SegIter si;
      seg_init(si, ms, g0, g1, lo, hi, p.cta_fin[blockIdx.x]);
      int64_t sa, sb;
      int k = 0;
      while (seg_next(si, ms, sa, sb)) {
        if ((k & 1) == e) {
          const uint32_t use = static_cast<uint32_t>(k >> 1);
          const Pos ps = locate(ms, g1, sa, g0);
          const SegInfo info = seg_info(ms, ps, sa, lo, p.cta_fin[blockIdx.x], p.W, G);
          const auto wsync = [] { __syncwarp(); };
          const auto wbcast = [](int v) { return __shfl_sync(0xffffffffu, v, 0); };
          float* S = own + e * MT * WIDE_N;
          bool ok = true;
          if (info.owner) ok = owner_prefetch<MT, 32>(info, lane, p, S, abort_flag, wsync, wbcast);
          bool okw = true;
          if (lane == 0)
            okw = mbar_wait_bounded(&red_full[e], use & 1, p.timeout_ns, abort_flag, p.err, K_GEMV, 4);
          ok = ok && __shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0 && !*abort_flag;
          finish_segment<MT, C::NCW, 32>(rb, info, lane, ok, p, S, wsync, [&] {
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_empty[e]);
          });
        }
        ++k;
      }
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
  SegIter si;
  seg_init(si, ms, g0, g1, lo, hi, p.cta_fin[blockIdx.x]);
  int64_t sa, sb;
  int k = 0;
  while (seg_next(si, ms, sa, sb)) {
    const Pos ps = locate(ms, g1, sa, g0);

    // accumulators: MT <= 2 -> acc[mm*4 + pp] = columns {2pp, 2pp+1} of row mm
    //               MT >= 4 -> this warp's slice red[cw][mm][256] in shared memory
    constexpr int NACC = C::ASYNC ? MT * 4 : 1;
    float2 acc[NACC];
#pragma unroll
    for (int i = 0; i < NACC; ++i) acc[i] = make_float2(0.f, 0.f);
    float* wacc = red + cw * MT * 256 + lane * 8;
    if constexpr (!C::ASYNC) {
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) {
        reinterpret_cast<float4*>(wacc + mm * 256)[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4*>(wacc + mm * 256)[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }

    int32_t u = ps.unit;
    const int32_t u_end = u + static_cast<int32_t>(sb - sa);
    while (u < u_end) {
      const int32_t n = min(SU - (u % SU), u_end - u);  // same grid as the producer
      const int s = it % C::NSTAGES;
      const uint32_t round = it / C::NSTAGES;
      if (ok) ok = mbar_wait_bounded(&full[s], round & 1, p.timeout_ns, abort_flag, p.err, K_GEMV, 3);
      if (ok) {
        const uint8_t* st = smem + s * C::STAGE_BYTES;
        if (ps.wide)
          stage_items<MT, true, C::NCW, C::IPW>(st, u, n, cw, sub, lane, kMagic, acc, wacc);
        else
          stage_items<MT, false, C::NCW, C::IPW>(st, u, n, cw, sub, lane, kMagic, acc, wacc);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      ++it;
      u += n;
    }

    // ---- segment done
    if constexpr (C::ASYNC) {
      // hand this warp's sums to epilogue warp k % 2 through buffer k % 2
      const int rbi = k & 1;
      const uint32_t use = static_cast<uint32_t>(k >> 1);
      if (use > 0) {
        bool okw = true;
        if (lane == 0)
          okw = mbar_wait_bounded(&red_empty[rbi], (use - 1) & 1, p.timeout_ns, abort_flag, p.err, K_GEMV, 5);
        okw = __shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0;
        ok = ok && okw;
      }
      float* dst = red + rbi * C::RED_FLOATS + cw * MT * 256 + lane * 8;
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) {
        reinterpret_cast<float4*>(dst + mm * 256)[0] =
            make_float4(acc[mm * 4 + 0].x, acc[mm * 4 + 0].y, acc[mm * 4 + 1].x, acc[mm * 4 + 1].y);
        reinterpret_cast<float4*>(dst + mm * 256)[1] =
            make_float4(acc[mm * 4 + 2].x, acc[mm * 4 + 2].y, acc[mm * 4 + 3].x, acc[mm * 4 + 3].y);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_full[rbi]);
    } else {
      named_bar_sync(1, C::NCW * 32);
      const SegInfo info = seg_info(ms, ps, sa, lo, p.cta_fin[blockIdx.x], p.W, G);
      const auto bsync = [] { named_bar_sync(1, C::NCW * 32); };
      const auto bbcast = [bcast_slot, ctid](int v) {
        if (ctid == 0) *bcast_slot = v;
        named_bar_sync(1, C::NCW * 32);
        const int r = *bcast_slot;
        named_bar_sync(1, C::NCW * 32);
        return r;
      };
      bool okg = true;
      if (info.owner) okg = owner_wait<C::NCW * 32>(info, ctid, p, abort_flag, bsync, bbcast);
      finish_segment<MT, C::NCW, C::NCW * 32>(red, info, ctid, ok && okg, p, nullptr, bsync, bsync);
    }
    ++k;
  }
}

// Cooperative launch: all CTAs are resident at once (or the launch fails), so
// an owner's bounded wait for the other contributors of a split tile ends.
template <int MT>
w4_status launch_mt(const GemvParams& prm, int grid, cudaStream_t st, const w4host::DeviceInfo& di) {
  using C = Cfg<MT>;
  static int configured_dev[64] = {};
  if (di.dev < 64 && !configured_dev[di.dev]) {
    cudaError_t e = cudaFuncSetAttribute(w4_gemv_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return w4host::cuda_fail(e, "cudaFuncSetAttribute(w4_gemv)");
    configured_dev[di.dev] = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(C::NTHREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, w4_gemv_kernel<MT>, prm);
  if (e != cudaSuccess) return w4host::cuda_fail(e, "launch w4_gemv");
  return W4_OK;
}

int pick_mt(const w4_desc* d, int count) {
  int64_t mx = 0;
  for (int i = 0; i < count; ++i) mx = std::max(mx, d[i].M);
  return mx <= 1 ? 1 : mx <= 2 ? 2 : mx <= 4 ? 4 : 8;
}

// Column tiling of one weight: ntw wide tiles (the last possibly partial) and
// an optional narrow tile for a remainder of at most 256 columns; or, when a
// wide tile (2*nb units) would be taller than 2*rmin + 1 units (rmin = the
// smallest CTA share), narrow tiles only, so that no tile spans more than one
// CTA's whole range. Either way the weight has nb * ceil(N / 256) units.
void tiling(int64_t N, int64_t nb, int64_t rmin, int32_t* ntw, int32_t* nnar) {
  if (2 * nb > 2 * rmin + 1) {
    *ntw = 0;
    *nnar = static_cast<int32_t>((N + NARROW_N - 1) / NARROW_N);
    return;
  }
  int64_t w = N / WIDE_N;
  const int64_t rem = N - w * WIDE_N;
  int32_t nar = 0;
  if (rem > NARROW_N) ++w;
  else if (rem > 0) nar = 1;
  *ntw = static_cast<int32_t>(w);
  *nnar = nar;
}

// Split-tile roles of CTAs whose ranges are [c*W/G, (c+1)*W/G): bit 0 of
// fin[c] set when c finishes the tile holding its first unit (also the one
// bit read when its whole range lies in one tile), bit 1 when it finishes the
// tile holding its last unit. Each tile that straddles CTAs gets exactly one
// finisher; the other contributors publish their pieces, which they process
// first (the piece at the start of the range, then the one at its end), so a
// published piece is done after the units its CTA publishes up to and
// including it. The finisher processes its piece last, so a publish done
// late in its CTA's range can make the finisher wait; the assignment
// minimises the sum over published pieces of late(f) = max(0, f - 1/2)^2, f
// the completion as a fraction of the CTA's range (dynamic programming over
// the CTAs, the state being whether a CTA publishes the piece at its start). A tile that holds
// some CTA's whole range is finished by the last such CTA: a range inside one
// tile cannot be published early.
// tile_of(f, &start, &units) gives the tile holding flat unit f.
template <class TileOf>
void cta_roles(int64_t W, int G, TileOf tile_of, uint8_t* fin) {
  auto rlo = [&](int64_t c) { return c * W / G; };
  auto cta = [&](int64_t f) { return ((f + 1) * G + W - 1) / W - 1; };
  constexpr double kInf = 1e30;
  auto late = [](double f) { return f > 0.5 ? (f - 0.5) * (f - 0.5) : 0.0; };
  for (int c = 0; c < G; ++c) fin[c] = 0;
  // dp[c][s]: least cost of the decisions left of CTA c, with s = 1
  // when c publishes the piece at the start of its range (of size head[c])
  std::vector<double> dp0(G + 1, kInf), dp1(G + 1, kInf);
  std::vector<int64_t> head(G + 1, 0);
  // how each CTA's state was reached: kind 0 none, 1 forced span from `from`,
  // 2 c-1 published (A), 3 c published its start (B); prev = state of c-1 / from
  std::vector<int> kind0(G + 1, 0), kind1(G + 1, 0), prev0(G + 1, 0), prev1(G + 1, 0), from0(G + 1, 0),
      from1(G + 1, 0);
  dp0[0] = 0.0;
  int c = 0;
  while (c + 1 < G) {
    const int64_t lo = rlo(c), hi = rlo(c + 1);
    int64_t ts, tu;
    tile_of(hi - 1, &ts, &tu);
    const int64_t te = ts + tu;
    const double best_any = std::min(dp0[c], dp1[c]);
    const int arg_any = dp1[c] < dp0[c] ? 1 : 0;
    if (te <= hi) {  // the range ends at a tile end
      if (best_any < dp0[c + 1]) {
        dp0[c + 1] = best_any;
        kind0[c + 1] = 0;
        prev0[c + 1] = arg_any;
      }
      ++c;
      continue;
    }
    const int cl = static_cast<int>(cta(te - 1));
    const double R = static_cast<double>(hi - lo);
    const int64_t a = hi - ts;  // c's piece (the end of its range)
    if (cl - c >= 2) {
      // forced: c and cl publish, the last CTA inside finishes, any other CTA
      // inside publishes its whole range
      const int64_t b = te - rlo(cl);
      double span = late(static_cast<double>(b) / static_cast<double>(rlo(cl + 1) - rlo(cl)));
      if (cl - c >= 3) span += late(1.0) * (cl - c - 2);
      for (int st = 0; st < 2; ++st) {
        const double base = st ? dp1[c] : dp0[c];
        if (base >= kInf) continue;
        const double v = base + late(static_cast<double>((st ? head[c] : 0) + a) / R) + span;
        if (v < dp1[cl]) {
          dp1[cl] = v;
          kind1[cl] = 1;
          prev1[cl] = st;
          from1[cl] = c;
        }
      }
      head[cl] = b;
      c = cl;
      continue;
    }
    const int64_t b = te - hi;  // c+1's piece (the start of its range)
    const double R1 = static_cast<double>(rlo(c + 2) - hi);
    head[c + 1] = b;
    for (int st = 0; st < 2; ++st) {
      const double base = st ? dp1[c] : dp0[c];
      if (base >= kInf) continue;
      // A: c publishes its piece, c+1 finishes
      const double va = base + late(static_cast<double>((st ? head[c] : 0) + a) / R);
      if (va < dp0[c + 1]) {
        dp0[c + 1] = va;
        kind0[c + 1] = 2;
        prev0[c + 1] = st;
      }
    }
    // B: c finishes, c+1 publishes its first piece
    const double vb = best_any + late(static_cast<double>(b) / R1);
    if (vb < dp1[c + 1]) {
      dp1[c + 1] = vb;
      kind1[c + 1] = 3;
      prev1[c + 1] = arg_any;
    }
    ++c;
  }
  // walk back from the better final state, setting the finishers
  int st = dp1[G - 1] < dp0[G - 1] ? 1 : 0;
  c = G - 1;
  while (c > 0) {
    const int kind = st ? kind1[c] : kind0[c];
    const int pv = st ? prev1[c] : prev0[c];
    if (kind == 1) {  // forced span from `from` to c
      const int f = st ? from1[c] : from0[c];
      fin[c - 1] |= 3;
      c = f;
      st = pv;
      continue;
    }
    const int64_t hi = rlo(c);  // boundary between c-1 and c
    int64_t ts, tu;
    tile_of(hi - 1, &ts, &tu);
    const int64_t te = ts + tu;
    if (kind == 2) fin[c] |= (rlo(c + 1) <= te) ? 3 : 1;   // c finishes its first piece (or whole range)
    if (kind == 3) fin[c - 1] |= (ts == rlo(c - 1)) ? 3 : 2;  // c-1 finishes its last piece (or whole range)
    c -= 1;
    st = pv;
  }
}

struct Plan {
  int mt = 1;
  int64_t W = 0;
  int grid = 0;
  int64_t rmin = 0;  // smallest CTA share, W / grid
};

// Workspace: [COUNTER_SLOTS int32 counters][grid][2][MT][WIDE_N] fp32 partials (a CTA
// publishes at most two partials: the pieces at the start and at the end of its range).
constexpr int COUNTER_SLOTS = 1024;  // >= GRID_MAX (one per CTA)
constexpr size_t COUNTER_BYTES = COUNTER_SLOTS * sizeof(int32_t);

Plan make_plan(const w4_desc* d, int count, int sms) {
  Plan pl;
  pl.mt = pick_mt(d, count);
  for (int i = 0; i < count; ++i) {
    if (d[i].M == 0 || d[i].N == 0 || d[i].K == 0) continue;
    const int64_t nmc = (d[i].M + pl.mt - 1) / pl.mt;
    const int64_t nb = d[i].K / 32;
    pl.W += nmc * nb * ((d[i].N + NARROW_N - 1) / NARROW_N);
  }
  pl.grid = static_cast<int>(std::min<int64_t>(std::min(sms, GRID_MAX), pl.W));
  pl.rmin = pl.grid > 0 ? pl.W / pl.grid : 0;
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

// Launch parameters of recent calls, per host thread. A decode loop calls with
// the same descriptors (weights, inputs and outputs at the same addresses)
// every step; the parameters are a function of the descriptor fields, the
// workspace address and the device alone, so an exact match reuses them and
// skips the tiling, the tensor-map lookups and the role assignment.
struct PlanEntry {
  int dev = -1;
  int count = 0;
  const void* ws = nullptr;
  size_t need = 0;
  int grid = 0;
  int mt = 0;
  uint64_t used = 0;
  w4_desc descs[W4_GROUP_MAX];
  GemvParams prm;
};
constexpr int kPlanEntries = 4;

// Field-by-field equality of two descriptor arrays: padding bytes a caller
// left uninitialised play no part.
bool same_descs(const w4_desc* a, const w4_desc* b, int count) {
  for (int i = 0; i < count; ++i) {
    const w4_desc& p = a[i];
    const w4_desc& q = b[i];
    if (p.x != q.x || p.ldx != q.ldx || p.qw != q.qw || p.scales != q.scales || p.zp != q.zp || p.y != q.y ||
        p.ldy != q.ldy || p.M != q.M || p.K != q.K || p.N != q.N || p.bias != q.bias || p.residual != q.residual ||
        p.ldr != q.ldr || p.act != q.act || p.reserved != q.reserved)
      return false;
  }
  return true;
}

w4_status launch_planned(const PlanEntry& e, cudaStream_t st, const DeviceInfo& di) {
  switch (e.mt) {
    case 1: return launch_mt<1>(e.prm, e.grid, st, di);
    case 2: return launch_mt<2>(e.prm, e.grid, st, di);
    case 4: return launch_mt<4>(e.prm, e.grid, st, di);
    default: return launch_mt<8>(e.prm, e.grid, st, di);
  }
}

w4_status launch_gemv(const w4_desc* d, int count, void* ws, size_t ws_size, cudaStream_t st, const DeviceInfo& di) {
  if (count > W4_GROUP_MAX) return fail(W4_ERR_SHAPE, "at most %d matrices per GEMV launch", W4_GROUP_MAX);
  static thread_local std::unique_ptr<PlanEntry[]> owned;  // kPlanEntries entries of ~37 KB, host memory
  static thread_local uint64_t clock = 0;
  if (!owned) owned.reset(new PlanEntry[kPlanEntries]);
  PlanEntry* cache = owned.get();
  ++clock;
  for (int i = 0; i < kPlanEntries; ++i) {
    PlanEntry& e = cache[i];
    if (e.dev == di.dev && e.count == count && e.ws == ws && same_descs(e.descs, d, count)) {
      if (ws_size < e.need) return fail(W4_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", e.need, ws_size);
      e.used = clock;
      e.prm.timeout_ns = wait_timeout_ns();
      return launch_planned(e, st, di);
    }
  }
  const Plan pl = make_plan(d, count, di.sms);
  if (pl.W == 0) return W4_OK;
  // the kernel's flat-index arithmetic is 32-bit: W * grid must stay below 2^32
  if (pl.W * pl.grid >= (int64_t(1) << 32))
    return fail(W4_ERR_SHAPE, "%lld units over %d CTAs is beyond one GEMV launch; split the group",
                static_cast<long long>(pl.W), pl.grid);
  const size_t need = ws_bytes(pl);
  if (ws == nullptr || ws_size < need)
    return fail(W4_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws == nullptr ? size_t(0) : ws_size);
  if ((reinterpret_cast<uintptr_t>(ws) & 15) != 0) return fail(W4_ERR_WORKSPACE, "workspace must be 16-byte aligned");

  static_assert(sizeof(GemvParams) <= 32000, "kernel parameters must fit the 32 KB limit");
  int victim = 0;  // least recently used entry
  for (int i = 1; i < kPlanEntries; ++i)
    if (cache[i].used < cache[victim].used) victim = i;
  PlanEntry& ent = cache[victim];
  ent.dev = -1;  // invalid until the parameters are complete
  GemvParams& prm = ent.prm;
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
    m.epi = Epi{s.bias, s.residual, s.ldr, s.act, 0};
    m.M = static_cast<int32_t>(s.M);
    m.K = static_cast<int32_t>(s.K);
    m.N = static_cast<int32_t>(s.N);
    m.nb = static_cast<int32_t>(s.K / 32);
    tiling(s.N, s.K / 32, pl.rmin, &m.ntw, &m.nnar);
    m.nmc = static_cast<int32_t>((s.M + pl.mt - 1) / pl.mt);
    m.u_off = uoff;
    m.u_wide = static_cast<int64_t>(m.ntw) * m.nmc * 2 * m.nb;
    uoff += m.u_wide + static_cast<int64_t>(m.nnar) * m.nmc * m.nb;
    ++g;
  }
  if (uoff != pl.W) return fail(W4_ERR_SHAPE, "internal: tiling covers %lld units, plan %lld", static_cast<long long>(uoff),
                                static_cast<long long>(pl.W));
  {
    const int ng = g;
    auto tile_of = [&](int64_t f, int64_t* start, int64_t* units) {
      int gi = 0;
      while (gi + 1 < ng && prm.mat[gi + 1].s.u_off <= f) ++gi;
      const MatScalars& m = prm.mat[gi].s;
      const int64_t local = f - m.u_off;
      if (local < m.u_wide) {
        *units = 2 * m.nb;
        *start = f - local % *units;
      } else {
        *units = m.nb;
        *start = f - (local - m.u_wide) % *units;
      }
    };
    cta_roles(uoff, pl.grid, tile_of, prm.cta_fin);
  }
  prm.count = g;
  prm.W = uoff;
  // first and last matrix of each CTA's range [c*W/G, (c+1)*W/G)
  {
    int gm = 0;
    for (int c = 0; c < pl.grid; ++c) {
      const int64_t lo = static_cast<int64_t>(c) * uoff / pl.grid;
      const int64_t hi = static_cast<int64_t>(c + 1) * uoff / pl.grid;
      while (gm + 1 < g && prm.mat[gm + 1].s.u_off <= lo) ++gm;
      int gl = gm;
      while (gl + 1 < g && prm.mat[gl + 1].s.u_off <= hi - 1) ++gl;
      prm.cta_g[c][0] = static_cast<uint8_t>(gm);
      prm.cta_g[c][1] = static_cast<uint8_t>(gl);
    }
  }
  prm.ws_counters = static_cast<int32_t*>(ws);
  prm.ws_partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + COUNTER_BYTES);
  prm.err = di.err;
  prm.timeout_ns = wait_timeout_ns();
  ent.count = count;
  ent.ws = ws;
  ent.need = need;
  ent.grid = pl.grid;
  ent.mt = pl.mt;
  ent.used = clock;
  std::memcpy(ent.descs, d, sizeof(w4_desc) * count);
  ent.dev = di.dev;
  return launch_planned(ent, st, di);
}

}  // namespace w4host
