// i8_head: logits[m, v] = s_v * sum_k h[m, k] * T[k, v] for the int8 tied
// LM head of "ONNX export, quantization and the browser runtime", section
// "Quantization (train/quantize.py)", steps 3 (embedding_int8: int8, one
// scale per token, [768, V] layout) and 4 (last_token_logits: only the last
// position's rows h are multiplied).
//
// Two kernels share the exact int8 -> fp32 decode: the byte, biased by 0x80,
// is placed in the mantissa of 2^23 (0x4B0000uu) by one PRMT, then one
// subtraction removes 2^23 + 128. The per-token scale is applied once per
// column after the sum.
//
// Row k of T starts at byte k*ldt, which is not aligned when ldt is odd
// (V = 50257). With T 16-byte aligned, (k*ldt) mod 16 depends only on
// k mod 16, so the rows k = 16 g + j (one residue j) share ONE misalignment:
// a thread that reads aligned 16-byte chunks of only those rows sees every
// column at the same place in its chunk, and the reduction across residues
// undoes the per-residue shift.
//
// i8_rows_kernel (M <= 2): one column slice of at most 368 columns per CTA
// and all K rows of it, so no CTA shares a tile with another. Thread
// (chunk c of 24, residue j of 16) copies, with 16-byte asynchronous copies,
// chunk c of the 16-byte-aligned window around the slice of each of its rows
// (k = j mod 16) into its own shared-memory slot, six stages of four rows
// ahead of the ones it converts (the copy holding the table's last byte reads
// only up to it and zero-fills the rest). It converts rows k and k + 16
// together, so the subtraction and the FMA are packed f32x2 instructions with
// h[k], h[k+16] as one operand. At the end the 16 residues' column sums are
// added with their shifts undone. No thread waits on another except at that
// final reduction.
//
// i8_head_kernel (M >= 3): persistent stream-K over 16-row groups of narrow
// column tiles. A warp takes one row of every 16-row group (one residue);
// each lane loads aligned chunks of it, keeping the loads of the next D rows
// in flight while it converts and accumulates the current D. A tile whose
// rows straddle CTAs is finished by the last CTA to arrive, which adds the
// partials in CTA order (deterministic) through the caller's workspace and
// resets the counter to zero.
#include <cuda_runtime.h>

#include <algorithm>

#include "w4_device.cuh"
#include "w4_internal.h"

namespace {

using namespace w4dev;

constexpr int NW = 16;  // warps per CTA = rows per group (the alignment period)
constexpr int COUNTER_SLOTS = 1024;
constexpr size_t COUNTER_BYTES = COUNTER_SLOTS * sizeof(int32_t);

template <int MT>
struct HCfg {
  static constexpr int CB = MT <= 2 ? 16 : (MT == 4 ? 8 : 4);  // bytes per lane chunk
  static constexpr int WIN = 32 * CB;                          // window columns per warp
  static constexpr int TV = 31 * CB;                           // tile columns
  static constexpr int D = MT == 1 ? 8 : (MT == 8 ? 2 : 4);   // rows per batch (two batches in flight)
  static constexpr int MINB = 1;                               // CTAs per SM
  static constexpr int RED_FLOATS = NW * MT * WIN;
  static constexpr int SMEM = RED_FLOATS * 4 + NW * 4 + 16;
};

// One PRMT: bytes of the result are [biased byte j, 0x00, 0x00, 0x4B]; the
// 0x4B000000 word is passed in a register so the selector is the only
// immediate.
__device__ __forceinline__ float byte_magic(uint32_t biased_word, uint32_t magic, int j /*compile time*/) {
  uint32_t r;
  switch (j) {
    case 0: asm("prmt.b32 %0, %1, %2, 0x7540;" : "=r"(r) : "r"(biased_word), "r"(magic)); break;
    case 1: asm("prmt.b32 %0, %1, %2, 0x7541;" : "=r"(r) : "r"(biased_word), "r"(magic)); break;
    case 2: asm("prmt.b32 %0, %1, %2, 0x7542;" : "=r"(r) : "r"(biased_word), "r"(magic)); break;
    default: asm("prmt.b32 %0, %1, %2, 0x7543;" : "=r"(r) : "r"(biased_word), "r"(magic)); break;
  }
  return __uint_as_float(r);
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
__device__ __noinline__ Chunk<CB> load_chunk_clipped(const int8_t* p, const int8_t* end) {
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

struct HeadParams {
  const float* h;
  int64_t ldh;
  const int8_t* table;
  int64_t ldt;
  const float* scales;
  float* logits;
  int64_t ldl;
  int32_t M, K, V;
  int32_t ntiles, NG, nmc;
  int64_t U;  // total units
  int32_t* ws_counters;
  float* ws_partials;  // [grid][2][MT][TV]
};

__device__ __forceinline__ int64_t cta_of(int64_t f, int64_t W, int64_t G) { return ((f + 1) * G + W - 1) / W - 1; }
__device__ __forceinline__ int64_t range_lo(int64_t i, int64_t W, int64_t G) { return (i * W) / G; }

template <int MT>
__global__ void __launch_bounds__(NW * 32, HCfg<MT>::MINB) i8_head_kernel(const __grid_constant__ HeadParams p) {
  using C = HCfg<MT>;
  constexpr int CB = C::CB;
  extern __shared__ __align__(16) float hsm[];
  float* red = hsm;                                          // [NW][MT][WIN]
  int* shift = reinterpret_cast<int*>(hsm + C::RED_FLOATS);  // [NW]
  int* bcast = shift + NW;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t lo = range_lo(blockIdx.x, p.U, G);
  const int64_t hi = range_lo(blockIdx.x + 1, p.U, G);
  const int8_t* table_end = p.table + (static_cast<int64_t>(p.K) - 1) * p.ldt + p.V;
  uint32_t kMagic;  // 0x4B000000 (the bits of 2^23) held in a register
  asm("mov.b32 %0, 0x4B000000;" : "=r"(kMagic));

  int64_t f = lo;
  while (f < hi) {
    const int64_t tile_l = f / p.NG;  // = mc * ntiles + tile
    const int32_t g0 = static_cast<int32_t>(f - tile_l * p.NG);
    const int64_t seg_end = min(hi, (tile_l + 1) * p.NG);
    const int32_t g1 = static_cast<int32_t>(seg_end - tile_l * p.NG);
    const int32_t mc = static_cast<int32_t>(tile_l / p.ntiles);
    const int32_t tile = static_cast<int32_t>(tile_l - static_cast<int64_t>(mc) * p.ntiles);
    const int64_t v0 = static_cast<int64_t>(tile) * C::TV;
    const int32_t m0 = mc * MT;
    const int mrows = min(MT, p.M - m0);

    // this warp's rows: k = 16 g + warp, g in [g0, g1), k < K; one window shift
    const int r = static_cast<int>(
        reinterpret_cast<uintptr_t>(p.table + (static_cast<int64_t>(g0) * NW + warp) * p.ldt + v0) & (CB - 1));
    const int8_t* wbase = p.table + v0 - r + lane * CB;

    float2 acc[MT * CB / 2];
#pragma unroll
    for (int i = 0; i < MT * CB / 2; ++i) acc[i] = make_float2(0.f, 0.f);

    // Software pipeline: the loads of the next D rows are in flight while the
    // current D rows are converted and accumulated.
    // Whether a batch's windows can reach past the end of the table is decided
    // once per batch for the whole warp (the window of row k ends at
    // win_end0 + k * ldt), so the usual path carries no per-row bounds logic.
    const int8_t* win_end0 = p.table + v0 - r + 32 * CB;
    auto load_batch = [&](int32_t gb, Chunk<CB> (&ch)[C::D], float (&hv)[C::D][MT]) {
      const int64_t k_hi = min(static_cast<int64_t>(gb + C::D) * NW - 1, static_cast<int64_t>(p.K) - 1);
      const bool careful = win_end0 + k_hi * p.ldt > table_end;
      if (!careful) {
        const bool full = (gb + C::D <= g1) && ((gb + C::D) * NW <= p.K);
        if (full) {
#pragma unroll
          for (int j = 0; j < C::D; ++j) {
            const int32_t k = (gb + j) * NW + warp;
            ch[j] = load_chunk<CB>(wbase + static_cast<int64_t>(k) * p.ldt);
#pragma unroll
            for (int mm = 0; mm < MT; ++mm)
              hv[j][mm] = (mm < mrows) ? __ldg(p.h + static_cast<int64_t>(m0 + mm) * p.ldh + k) : 0.f;
          }
          return;
        }
      }
#pragma unroll
      for (int j = 0; j < C::D; ++j) {
        const int32_t k = (gb + j) * NW + warp;
        if (gb + j < g1 && k < p.K) {
          const int8_t* q = wbase + static_cast<int64_t>(k) * p.ldt;
          ch[j] = (!careful || q + CB <= table_end) ? load_chunk<CB>(q) : load_chunk_clipped<CB>(q, table_end);
#pragma unroll
          for (int mm = 0; mm < MT; ++mm)
            hv[j][mm] = (mm < mrows) ? __ldg(p.h + static_cast<int64_t>(m0 + mm) * p.ldh + k) : 0.f;
        } else {
#pragma unroll
          for (int i = 0; i < CB / 4; ++i) ch[j].w[i] = 0u;  // q = 0
#pragma unroll
          for (int mm = 0; mm < MT; ++mm) hv[j][mm] = 0.f;
        }
      }
    };
    Chunk<CB> cur[C::D];
    float hcur[C::D][MT];
    load_batch(g0, cur, hcur);
    for (int32_t gb = g0; gb < g1; gb += C::D) {
      Chunk<CB> nxt[C::D];
      float hnxt[C::D][MT];
      if (gb + C::D < g1) load_batch(gb + C::D, nxt, hnxt);
#pragma unroll
      for (int j = 0; j < C::D; ++j) {
#pragma unroll
        for (int i = 0; i < CB / 4; ++i) {
          const uint32_t bw = cur[j].w[i] ^ 0x80808080u;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float qv = byte_magic(bw, kMagic, e) - 8388736.0f;  // exact int8 value
#pragma unroll
            for (int mm = 0; mm < MT; ++mm) {
              float2& a2 = acc[mm * (CB / 2) + i * 2 + (e >> 1)];
              if (e & 1) a2.y = fmaf(hcur[j][mm], qv, a2.y);
              else a2.x = fmaf(hcur[j][mm], qv, a2.x);
            }
          }
        }
      }
      if (gb + C::D < g1) {
#pragma unroll
        for (int j = 0; j < C::D; ++j) {
          cur[j] = nxt[j];
#pragma unroll
          for (int mm = 0; mm < MT; ++mm) hcur[j][mm] = hnxt[j][mm];
        }
      }
    }

    // ---- reduce the warps (undoing each warp's window shift)
#pragma unroll
    for (int mm = 0; mm < MT; ++mm) {
      float* dst = red + (warp * MT + mm) * C::WIN + lane * CB;
#pragma unroll
      for (int pp = 0; pp < CB / 2; ++pp) {
        dst[2 * pp] = acc[mm * (CB / 2) + pp].x;
        dst[2 * pp + 1] = acc[mm * (CB / 2) + pp].y;
      }
    }
    if (lane == 0) shift[warp] = r;
    __syncthreads();

    const int64_t t_start = tile_l * p.NG;
    const int64_t c_first = cta_of(t_start, p.U, G);
    const int64_t c_last = cta_of(t_start + p.NG - 1, p.U, G);
    const bool split = c_first != c_last;
    const int slot = (split && static_cast<int64_t>(blockIdx.x) == c_first && lo < t_start) ? 1 : 0;
    for (int idx = threadIdx.x; idx < MT * C::TV; idx += NW * 32) {
      const int mm = idx / C::TV;
      const int c = idx - mm * C::TV;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) v += red[(w * MT + mm) * C::WIN + c + shift[w]];
      const int64_t col = v0 + c;
      if (!split) {
        if (mm < mrows && col < p.V) p.logits[static_cast<int64_t>(m0 + mm) * p.ldl + col] = v * __ldg(p.scales + col);
      } else {
        p.ws_partials[((static_cast<int64_t>(blockIdx.x) * 2 + slot) * MT + mm) * C::TV + c] = v;
      }
    }
    if (split) {
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) bcast[0] = atomicAdd(&p.ws_counters[c_first], 1);
      __syncthreads();
      if (bcast[0] == static_cast<int>(c_last - c_first)) {
        __threadfence();
        for (int idx = threadIdx.x; idx < MT * C::TV; idx += NW * 32) {
          const int mm = idx / C::TV;
          const int c = idx - mm * C::TV;
          float v = 0.f;
          for (int64_t cc = c_first; cc <= c_last; ++cc) {
            const int sl = (cc == c_first && range_lo(cc, p.U, G) < t_start) ? 1 : 0;
            v += __ldcg(&p.ws_partials[((cc * 2 + sl) * MT + mm) * C::TV + c]);
          }
          const int64_t col = v0 + c;
          if (mm < mrows && col < p.V)
            p.logits[static_cast<int64_t>(m0 + mm) * p.ldl + col] = v * __ldg(p.scales + col);
        }
        if (threadIdx.x == 0) p.ws_counters[c_first] = 0;
      }
    }
    __syncthreads();  // red / shift are reused by the next segment
    f = seg_end;
  }
}

// ---------------------------------------------------------------- greedy decoding

// A 64-bit key whose unsigned order is the order of (logit, -token): the
// logit's bits made monotonic (non-negative: sign bit set; negative: all bits
// flipped; -0 taken as +0) above the complement of the token id, so the
// maximum key is the largest logit and, among equal logits, the lowest token
// id. 0 is below every key of a number.
__device__ __forceinline__ unsigned long long argmax_key(float logit, uint32_t token) {
  uint32_t b = __float_as_uint(logit);
  if (b == 0x80000000u) b = 0u;  // -0 and +0 are the same logit: the lower id must win the tie
  const uint32_t o = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return (static_cast<unsigned long long>(o) << 32) | static_cast<unsigned long long>(0xFFFFFFFFu - token);
}

__device__ __forceinline__ unsigned long long warp_max_key(unsigned long long k) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) k = max(k, __shfl_xor_sync(0xffffffffu, k, o));
  return k;
}

// keys[m] <- max over the logits of row m (for heads whose logits were
// written to a buffer first).
__global__ void __launch_bounds__(256) argmax_rows_kernel(const float* __restrict__ logits, int64_t ldl, int32_t V,
                                                          unsigned long long* keys) {
  const int m = blockIdx.y;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * 2048;
  unsigned long long best = 0ull;
  for (int64_t c = c0 + threadIdx.x; c < min(c0 + 2048, static_cast<int64_t>(V)); c += 256)
    best = max(best, argmax_key(__ldg(logits + m * ldl + c), static_cast<uint32_t>(c)));
  best = warp_max_key(best);
  if ((threadIdx.x & 31) == 0 && best != 0ull) atomicMax(keys + m, best);
}

// tokens[m] (and best[m], when given) from keys[m].
__global__ void argmax_finish_kernel(const unsigned long long* keys, int32_t M, int32_t* tokens, float* best) {
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  if (m >= M) return;
  const unsigned long long k = keys[m];
  tokens[m] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(k & 0xFFFFFFFFull));
  if (best != nullptr) {
    const uint32_t o = static_cast<uint32_t>(k >> 32);
    best[m] = __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
  }
}

// ---------------------------------------------------------------- i8_rows_kernel

constexpr int RROWS = 64;             // rows per stage
constexpr int RWIN = 384;             // window bytes per row (24 chunks of 16 B)
constexpr int RTV = RWIN - 16;        // columns a slice may hold (any shift fits)
constexpr int RST = 6;                // stages in flight per thread
constexpr int RTHREADS = 384;         // 24 chunks x 16 residues
constexpr int RSTAGE = RROWS * RWIN;  // 24 KB
constexpr int RH_MAX_BYTES = 32768;   // h rows kept in shared memory

struct RowsParams {
  const float* h;
  int64_t ldh;
  const int8_t* table;
  int64_t ldt;
  const float* scales;
  float* logits;
  int64_t ldl;
  int32_t M, K, V;
  int32_t ntiles;  // column slices, [t*V/ntiles, (t+1)*V/ntiles)
  int32_t kpad;    // K rounded up to whole stages
  int32_t pad;
  // greedy decoding: when set, logits are not written; each CTA folds the
  // best (logit, token) of its slice into keys[m] (see argmax_key)
  unsigned long long* keys;
};

template <int MT>
size_t rows_smem_bytes(int kpad) {
  return static_cast<size_t>(RST) * RSTAGE + static_cast<size_t>(MT) * 16 * RWIN * 4 +
         static_cast<size_t>(MT) * kpad * 4 + 64;
}

template <int MT>
__global__ void __launch_bounds__(RTHREADS, 1) i8_rows_kernel(const __grid_constant__ RowsParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  float* red = reinterpret_cast<float*>(smem + RST * RSTAGE);  // [MT][16 residues][RWIN]
  float* hs = red + MT * 16 * RWIN;                            // [MT][kpad], zero past K
  int* shifts = reinterpret_cast<int*>(hs + MT * p.kpad);      // [16]

  const int t = threadIdx.x;
  const int ch = t % 24;   // 16-byte chunk of the row window
  const int res = t / 24;  // residue of this thread's rows mod 16
  const int nst = p.kpad / RROWS;
  const uintptr_t tend = reinterpret_cast<uintptr_t>(p.table + static_cast<int64_t>(p.K - 1) * p.ldt + p.V);
  const int64_t step16 = 16 * p.ldt;  // from row k to row k + 16
  uint32_t kMagic;                    // 0x4B000000 (the bits of 2^23) held in a register
  asm("mov.b32 %0, 0x4B000000;" : "=r"(kMagic));
  const float2 kOff = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)

  for (int i = t; i < MT * p.kpad; i += RTHREADS) {
    const int mm = i / p.kpad, k = i - mm * p.kpad;
    hs[i] = (mm < p.M && k < p.K) ? p.h[static_cast<int64_t>(mm) * p.ldh + k] : 0.f;
  }
  __syncthreads();

  for (int tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x) {
    const int64_t v0 = static_cast<int64_t>(tile) * p.V / p.ntiles;
    const int64_t v1 = static_cast<int64_t>(tile + 1) * p.V / p.ntiles;
    const int ncols = static_cast<int>(v1 - v0);
    // This thread's chunk of row k = res + 16 j is at a0 + j * step16; it is
    // part of the row's window iff 16 ch < (window end - window start), the
    // same for every row of the residue.
    const uintptr_t x0 = reinterpret_cast<uintptr_t>(p.table + static_cast<int64_t>(res) * p.ldt + v0);
    const uintptr_t a0 = (x0 & ~static_cast<uintptr_t>(15)) + 16 * ch;
    const bool active = a0 < x0 + static_cast<uintptr_t>(ncols);
    uint8_t* mine = smem + t * 16;  // this thread's slot: [stage][row q][thread] of 16 B

    // stage sg holds this thread's rows k = 64 sg + res + 16 q, q = 0..3
    auto issue = [&](int sg) {
      if (sg < nst && active) {
        uint8_t* dst = mine + (sg % RST) * RSTAGE;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int k = sg * RROWS + res + 16 * q;
          if (k < p.K) {
            const uintptr_t src = a0 + static_cast<uintptr_t>(4 * sg + q) * static_cast<uintptr_t>(step16);
            const uint32_t n = tend - src >= 16 ? 16u : static_cast<uint32_t>(tend - src);  // rest zero-filled
            cp_async_16(dst + q * RTHREADS * 16, reinterpret_cast<const void*>(src), n);
          }
        }
      }
      cp_async_commit();
    };

    float2 acc[MT][16];
#pragma unroll
    for (int mm = 0; mm < MT; ++mm)
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[mm][c] = make_float2(0.f, 0.f);
#pragma unroll 1
    for (int sg = 0; sg < RST - 1; ++sg) issue(sg);
#pragma unroll 1
    for (int sg = 0; sg < nst; ++sg) {
      issue(sg + RST - 1);
      cp_async_wait_group<RST - 1>();  // this thread's copies of stage sg have landed
      const uint8_t* src = mine + (sg % RST) * RSTAGE;
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        // rows k and k + 16 (q = 2 pr and 2 pr + 1), both residue res
        const uint4 A = *reinterpret_cast<const uint4*>(src + (2 * pr) * RTHREADS * 16);
        const uint4 B = *reinterpret_cast<const uint4*>(src + (2 * pr + 1) * RTHREADS * 16);
        const int k0 = sg * RROWS + res + 32 * pr;
        float2 hp[MT];
#pragma unroll
        for (int mm = 0; mm < MT; ++mm) hp[mm] = make_float2(hs[mm * p.kpad + k0], hs[mm * p.kpad + k0 + 16]);
        const uint32_t wa[4] = {A.x, A.y, A.z, A.w};
        const uint32_t wb[4] = {B.x, B.y, B.z, B.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t a = wa[i] ^ 0x80808080u;
          const uint32_t b = wb[i] ^ 0x80808080u;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 d = __fadd2_rn(make_float2(byte_magic(a, kMagic, e), byte_magic(b, kMagic, e)), kOff);
#pragma unroll
            for (int mm = 0; mm < MT; ++mm) acc[mm][i * 4 + e] = __ffma2_rn(hp[mm], d, acc[mm][i * 4 + e]);
          }
        }
      }
    }
    cp_async_wait_group<0>();
    // ---- reduce the residues: column c of the slice sits at byte c + shift[j]
    // of residue j's window
#pragma unroll
    for (int mm = 0; mm < MT; ++mm) {
      float* dst = red + (mm * 16 + res) * RWIN + ch * 16;
#pragma unroll
      for (int c = 0; c < 16; c += 4)
        *reinterpret_cast<float4*>(dst + c) =
            make_float4(acc[mm][c].x + acc[mm][c].y, acc[mm][c + 1].x + acc[mm][c + 1].y,
                        acc[mm][c + 2].x + acc[mm][c + 2].y, acc[mm][c + 3].x + acc[mm][c + 3].y);
    }
    if (t < 16)
      shifts[t] = static_cast<int>(reinterpret_cast<uintptr_t>(p.table + static_cast<int64_t>(t) * p.ldt + v0) & 15);
    __syncthreads();
    unsigned long long best[MT];
#pragma unroll
    for (int mm = 0; mm < MT; ++mm) best[mm] = 0ull;
    for (int c = t; c < ncols; c += RTHREADS) {
      const float sc = __ldg(p.scales + v0 + c);
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) {
        if (mm >= p.M) break;
        float v = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) v += red[(mm * 16 + j) * RWIN + c + shifts[j]];
        const float logit = v * sc;
        if (p.keys == nullptr) p.logits[static_cast<int64_t>(mm) * p.ldl + v0 + c] = logit;
        else best[mm] = max(best[mm], argmax_key(logit, static_cast<uint32_t>(v0 + c)));
      }
    }
    if (p.keys != nullptr) {
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) {
        if (mm >= p.M) break;
        const unsigned long long b = warp_max_key(best[mm]);
        if ((t & 31) == 0 && b != 0ull) atomicMax(p.keys + mm, b);
      }
    }
    __syncthreads();  // red and shifts are reused by the next slice
  }
}

template <int MT>
w4_status launch_rows_mt(const RowsParams& prm, int grid, cudaStream_t st, const w4host::DeviceInfo& di) {
  const size_t smem = rows_smem_bytes<MT>(prm.kpad);
  static size_t configured[64] = {};
  if (di.dev < 64 && configured[di.dev] < smem) {
    cudaError_t e = cudaFuncSetAttribute(i8_rows_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return w4host::cuda_fail(e, "cudaFuncSetAttribute(i8_rows)");
    configured[di.dev] = smem;
  }
  i8_rows_kernel<MT><<<grid, RTHREADS, smem, st>>>(prm);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : w4host::cuda_fail(e, "launch i8_rows");
}

// The rows kernel takes M <= 2 while h fits its shared-memory copy.
bool rows_eligible(int64_t M, int64_t K) {
  const int64_t kpad = (K + RROWS - 1) / RROWS * RROWS;
  return M <= 2 && M * kpad * 4 <= RH_MAX_BYTES;
}

w4_status launch_rows(const w4host::HeadArgs& a, cudaStream_t st, const w4host::DeviceInfo& di,
                      unsigned long long* keys = nullptr) {
  RowsParams prm;
  prm.keys = keys;
  prm.h = a.h;
  prm.ldh = a.ldh;
  prm.table = a.table;
  prm.ldt = a.ldt;
  prm.scales = a.scales;
  prm.logits = a.logits;
  prm.ldl = a.ldl;
  prm.M = static_cast<int32_t>(a.M);
  prm.K = static_cast<int32_t>(a.K);
  prm.V = static_cast<int32_t>(a.V);
  prm.kpad = static_cast<int32_t>((a.K + RROWS - 1) / RROWS * RROWS);
  prm.pad = 0;
  // slices of at most RTV columns, at least one per SM when V allows 32-column
  // slices, and a whole number of rounds over the SMs
  int64_t nt = (a.V + RTV - 1) / RTV;
  nt = std::max<int64_t>(nt, std::min<int64_t>(di.sms, (a.V + 31) / 32));
  if (nt > di.sms) nt = (nt + di.sms - 1) / di.sms * di.sms;
  prm.ntiles = static_cast<int32_t>(nt);
  const int grid = static_cast<int>(std::min<int64_t>(nt, di.sms));
  return a.M <= 1 ? launch_rows_mt<1>(prm, grid, st, di) : launch_rows_mt<2>(prm, grid, st, di);
}

struct HPlan {
  int mt;
  int tv;
  int64_t ntiles, NG, nmc, U;
  int grid;
};

HPlan head_plan(int64_t M, int64_t K, int64_t V, int sms) {
  HPlan pl;
  pl.mt = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;
  const int cb = pl.mt <= 2 ? 16 : (pl.mt == 4 ? 8 : 4);
  pl.tv = 31 * cb;
  pl.ntiles = (V + pl.tv - 1) / pl.tv;
  pl.NG = (K + NW - 1) / NW;
  pl.nmc = (M + pl.mt - 1) / pl.mt;
  pl.U = pl.ntiles * pl.NG * pl.nmc;
  const int per_sm = 1;
  pl.grid = static_cast<int>(std::min<int64_t>(std::min(per_sm * sms, COUNTER_SLOTS), pl.U));
  return pl;
}

template <int MT>
w4_status launch_head_mt(const HeadParams& prm, int grid, cudaStream_t st, const w4host::DeviceInfo& di) {
  using C = HCfg<MT>;
  static int configured[64] = {};
  if (di.dev < 64 && !configured[di.dev]) {
    cudaError_t e = cudaFuncSetAttribute(i8_head_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return w4host::cuda_fail(e, "cudaFuncSetAttribute(i8_head)");
    configured[di.dev] = 1;
  }
  i8_head_kernel<MT><<<grid, NW * 32, C::SMEM, st>>>(prm);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : w4host::cuda_fail(e, "launch i8_head");
}

}  // namespace

namespace w4host {

size_t head_workspace_bytes(int64_t M, int64_t K, int64_t V, int sms) {
  if (M <= 0 || K <= 0 || V <= 0) return 0;
  if (rows_eligible(M, K)) return 0;
  const HPlan pl = head_plan(M, K, V, sms);
  return COUNTER_BYTES + static_cast<size_t>(pl.grid) * 2 * pl.mt * pl.tv * sizeof(float);
}

w4_status launch_head(const HeadArgs& a, void* ws, size_t ws_size, cudaStream_t st, const DeviceInfo& di) {
  if (a.K > 0x7fffffff || a.V > 0x7fffffff || a.M > 0x7fffffff)
    return fail(W4_ERR_SHAPE, "head sizes must be below 2^31 on the fast path");
  if (rows_eligible(a.M, a.K)) return launch_rows(a, st, di);
  const HPlan pl = head_plan(a.M, a.K, a.V, di.sms);
  const size_t need = head_workspace_bytes(a.M, a.K, a.V, di.sms);
  if (ws == nullptr || ws_size < need)
    return fail(W4_ERR_WORKSPACE, "head workspace of %zu bytes needed, %zu given", need,
                ws == nullptr ? size_t(0) : ws_size);
  if ((reinterpret_cast<uintptr_t>(ws) & 15) != 0) return fail(W4_ERR_WORKSPACE, "workspace must be 16-byte aligned");
  HeadParams prm;
  prm.h = a.h;
  prm.ldh = a.ldh;
  prm.table = a.table;
  prm.ldt = a.ldt;
  prm.scales = a.scales;
  prm.logits = a.logits;
  prm.ldl = a.ldl;
  prm.M = static_cast<int32_t>(a.M);
  prm.K = static_cast<int32_t>(a.K);
  prm.V = static_cast<int32_t>(a.V);
  prm.ntiles = static_cast<int32_t>(pl.ntiles);
  prm.NG = static_cast<int32_t>(pl.NG);
  prm.nmc = static_cast<int32_t>(pl.nmc);
  prm.U = pl.U;
  prm.ws_counters = static_cast<int32_t*>(ws);
  prm.ws_partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + COUNTER_BYTES);
  switch (pl.mt) {
    case 1: return launch_head_mt<1>(prm, pl.grid, st, di);
    case 2: return launch_head_mt<2>(prm, pl.grid, st, di);
    case 4: return launch_head_mt<4>(prm, pl.grid, st, di);
    default: return launch_head_mt<8>(prm, pl.grid, st, di);
  }
}

bool head_rows_path(int64_t M, int64_t K) { return K > 0 && rows_eligible(M, K); }

w4_status launch_head_keys(const HeadArgs& a, unsigned long long* keys, cudaStream_t st, const DeviceInfo& di) {
  return launch_rows(a, st, di, keys);
}

w4_status launch_argmax_rows(const float* logits, int64_t ldl, int64_t M, int64_t V, unsigned long long* keys,
                             cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>((V + 2047) / 2048), static_cast<unsigned>(M));
  argmax_rows_kernel<<<grid, 256, 0, st>>>(logits, ldl, static_cast<int32_t>(V), keys);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch argmax_rows");
}

w4_status launch_argmax_finish(const unsigned long long* keys, int64_t M, int32_t* tokens, float* best,
                               cudaStream_t st) {
  argmax_finish_kernel<<<static_cast<unsigned>((M + 127) / 128), 128, 0, st>>>(keys, static_cast<int32_t>(M), tokens,
                                                                              best);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch argmax_finish");
}

}  // namespace w4host
