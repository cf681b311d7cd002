// i8t: the int8 tied LM head on the 5th-generation tensor cores, for up to 8
// rows at a time (the last positions of up to 8 sequences), with the table in
// its tile layout.
//
// The head is the one of "ONNX export, quantization and the browser runtime",
// section "Quantization (train/quantize.py)", steps 3 (embedding_int8: one
// int8 code per (row, token) and one fp32 scale per token, layout [K, V]) and
// 4 (the last position only): logits[m, v] = s_v * sum_k h[m, k] T[k, v].
//
// Arithmetic: integer MMAs (kind::i8) on the codes as they are stored. Each
// row m of h is written in fixed point against its own largest magnitude:
// with |h[m, k]| < 2^E for every k, h[m, k] = 2^(E - 6) sum_p d_p 2^(-7 p)
// + r, p = 0..7, each digit d_p an integer in [-64, 64] (rounded to nearest
// one at a time, so the remainder after each digit is exact in fp32) and
// |r| <= 2^(E - 56). Every element within 2^31 of the row's largest is
// therefore represented exactly, and the rest to 2^-55 of that largest. The
// tensor core forms D_p[v] = sum_k T[k, v] d_p[k] exactly in int32 (|D_p| <=
// 64 * 128 * 1024 = 2^23), and the read-back adds the eight D_p with their
// weights in fp64 and multiplies by the scale: the logit is the exact dot
// product of the codes with h (up to r) rounded once or twice, well inside
// the fp32 summation error of a plain evaluation. The result does not depend
// on the order of anything (integer sums), so it is deterministic.
//
// Tile layout (K % 32 == 0, 32 <= K <= 1024): tiles of 128 tokens in token
// order (the last one padded with code 0 and scale 0); a tile is K / 32 units
// of 4096 bytes followed by 512 bytes of scales:
//   unit u: the code of row 32 u + 16 h + i (h in 0..1, i in 0..15) and token
//           128 t + c at (c / 8) * 256 + h * 128 + (c % 8) * 16 + i: the
//           K-major, unswizzled operand layout of the tensor core (8 x 16-byte
//           core matrices; 128 bytes between the two K halves, 256 between
//           groups of 8 tokens);
//   scales: token 128 t + c at K * 128 + 4 c.
// Restoring gives the page's table and scales back bit for bit.
//
// Design (sm_100a), one persistent CTA per SM over a contiguous run of tiles:
//  * the CTA writes its rows of h as digits into the B operand once (row
//    8 m + p holds digit p of row m; K-major, unswizzled), all of K resident
//    in shared memory;
//  * warp 2 streams the tiles in stages of up to 128 rows of K (16 KB, one
//    bulk copy, no multicast) through a ring of 10 to 13 stages; the codes do
//    not depend on the previous launch, so the first stages are requested
//    before it has finished;
//  * warps 0 and 1 each issue the MMAs of every other stage (four MMAs of
//    M 128, N 8 M rounded up to 16, K 32) into accumulators of their own in
//    tensor memory, one per tile, so that the wait of one issuing thread (an
//    mbarrier wait right after MMAs costs it a few hundred clocks) overlaps
//    the other's MMAs. The MMA's commit frees the stage for the next copy;
//  * warps 4-7 (one per quarter of tensor-memory lanes, a lane per token)
//    read a tile's two accumulators (two tiles in flight), add them, weigh
//    the digits, scale, and store the logits, or fold them into 64-bit keys
//    for the greedy token.
// Every wait is bounded; on timeout the CTA records the error, stops issuing,
// lets its copies and MMAs in flight finish, and returns.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>

#include "w4_device.cuh"
#include "w4_internal.h"

namespace {

using namespace w4dev;

constexpr int TT = 128;                    // tokens per tile (MMA M)
constexpr int UK = 32;                     // rows of K per unit (one MMA)
constexpr int UB = TT * UK;                // 4096 code bytes per unit
constexpr int SU = 4;                      // units per stage
constexpr int SB = SU * UB;                // 16 KB per stage
constexpr int NMAX = 8;                    // rows of h per call
constexpr int ND = 8;                      // digits per row of h
constexpr int KMAX = 1024;
constexpr int MAXNS = 13;                  // stages at most
constexpr int NWARP = 8;
constexpr int NT = NWARP * 32;
constexpr int GI = KMAX / 4 / 32;          // groups of 4 elements of a row of h per lane at most
constexpr uint32_t TCOLS = 256;            // tensor memory: 2 issuers x 2 tiles x NB <= 64 columns
constexpr int SMEM_MAX = 227 * 1024;
constexpr int BAR_BYTES = 512;             // barriers, tensor-memory slot, abort flag, row exponents

__host__ __device__ constexpr int nb_for(int M) { return M <= 2 ? 16 : (M <= 4 ? 32 : (M <= 6 ? 48 : 64)); }
// even: the two issuers take the stages of one parity each
__host__ __device__ constexpr int stages_for(int NB, int K) {
  return ((SMEM_MAX - NB * K - BAR_BYTES) / SB < MAXNS ? (SMEM_MAX - NB * K - BAR_BYTES) / SB : MAXNS) & ~1;
}
__host__ __device__ constexpr int smem_for(int NB, int K) { return stages_for(NB, K) * SB + NB * K + BAR_BYTES; }
static_assert(stages_for(64, KMAX) >= 8, "stage ring of the widest case");
static_assert(smem_for(64, KMAX) <= SMEM_MAX, "shared memory of one CTA");

struct HParamsT {
  const float* h;
  int64_t ldh;
  const uint8_t* tiles;
  float* logits;                // NULL when keys are made
  int64_t ldl;
  unsigned long long* keys;     // [M] argmax keys, or NULL
  int32_t K, V, M, ntiles;
  int64_t tile_bytes;
  ErrorWord* err;
  uint64_t timeout_ns;
};

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Bounded wait that ignores the abort flag: lets copies and MMAs in flight land.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return;
  const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
  while (!mbar_try_wait_sleep(a, parity, 100000u))
    if (globaltimer_ns() - t0 > timeout_ns) return;
}

// Wait of a thread that issues MMAs: plain try_wait in a loop, so that it
// resumes as soon as the phase completes (a suspended thread wakes late, and
// the tensor core has no other feed). Bounded by `budget` clocks and the
// CTA's abort flag; records the error on timeout.
__device__ __forceinline__ bool spin_wait(uint64_t* bar, uint32_t parity, long long budget, volatile int* abort_flag,
                                          ErrorWord* err, int32_t detail) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const long long t0 = clock64();
#pragma unroll 1
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(a, parity)) return true;
    if ((it & 63u) == 0 && (*abort_flag || clock64() - t0 > budget)) break;
  }
  if (!*abort_flag) {
    *abort_flag = 1;
    record_error(err, W4_ERR_TIMEOUT, K_HEADT, detail);
  }
  return false;
}

// K-major, no swizzle, LBO 128 bytes (the two 16-byte K halves of a 32-byte
// row), SBO 256 bytes (groups of 8 rows), descriptor version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((128u >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((256u >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// D (s32, tensor memory) (+)= A (s8, shared) . B (s8, shared)^T, K 32.
__device__ __forceinline__ void mma_i8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, bool acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc ? 1u : 0u)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ unsigned long long head_key_t(float logit, uint32_t token) {
  uint32_t b = __float_as_uint(logit);
  if (b == 0x80000000u) b = 0u;  // -0 ranks as +0
  const uint32_t o = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return (static_cast<unsigned long long>(o) << 32) | static_cast<unsigned long long>(0xFFFFFFFFu - token);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Biased exponent field of |x| (0 for zero and subnormals, 255 for Inf/NaN).
__device__ __forceinline__ int exp_field(float x) { return static_cast<int>((__float_as_uint(x) >> 23) & 0xFFu); }

// Stages of a CTA: stage g is stage j = g % nst of its tile t0 + g / nst, the
// units 4 j .. min(4 j + 4, upt) - 1 of that tile; issuer j % 2 takes it.
template <int NB>
__global__ void __launch_bounds__(NT, 1) i8t_head_kernel(const __grid_constant__ HParamsT p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int t0 = static_cast<int>((static_cast<int64_t>(blockIdx.x) * p.ntiles) / G);
  const int t1 = static_cast<int>((static_cast<int64_t>(blockIdx.x + 1) * p.ntiles) / G);
  const int upt = p.K / UK;              // units per tile
  const int nst = (upt + SU - 1) / SU;   // stages per tile
  const int NS = stages_for(NB, p.K);    // ring stages
  const int GS = (t1 - t0) * nst;        // stages of this CTA
  const bool two = nst >= 2;             // does issuer 1 take part

  uint8_t* stages = smem;
  uint8_t* bs = smem + NS * SB;
  uint64_t* full = reinterpret_cast<uint64_t*>(bs + NB * p.K);
  uint64_t* empty = full + MAXNS;
  uint64_t* dready = empty + MAXNS;  // [issuer][tile parity]
  uint64_t* dfree = dready + 4;      // [issuer][tile parity]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(dfree + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  int* emax = reinterpret_cast<int*>(tslot + 2);  // [NMAX] largest exponent field of each row

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(TCOLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&dready[i], 1);
      mbar_init(&dfree[i], 4);
    }
    *abort_flag = 0;
    for (int m = 0; m < NMAX; ++m) emax[m] = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  // ---- the first stages before the wait: the table is a constant
  int issued = 0;
  if (warp == 2 && lane == 0) {
    for (; issued < NS && issued < GS; ++issued) {
      const int t = t0 + issued / nst, j = issued - (issued / nst) * nst;
      const int nu = min(SU, upt - SU * j);
      mbar_arrive_expect_tx(&full[issued], nu * UB);
      bulk_g2s(stages + issued * SB, p.tiles + t * p.tile_bytes + static_cast<int64_t>(j) * SB, nu * UB,
               &full[issued]);
    }
  }
  // B starts as zeros (digit rows of absent rows of h, and the padding to NB)
  for (int i = threadIdx.x; i < NB * p.K / 16; i += NT) reinterpret_cast<uint4*>(bs)[i] = make_uint4(0u, 0u, 0u, 0u);
  pdl_launch_dependents();
  pdl_wait();  // h, the logits and the keys follow the previous launch
  __syncthreads();  // the zeros land before any digit

  // ---- B: row 8 m + p holds digit p of row m, all of K. Warp w takes row
  // m = w / wpr (wpr = 8 / M warps per row, at least 1) and the w % wpr-th
  // contiguous share of its groups of 4 consecutive k (lane l: groups
  // gs0 + l + 32 i), loaded with 16-byte loads where h allows. The row's
  // largest exponent field F comes from one shared atomic per warp and one
  // CTA barrier. With |h| < 2^(F - 126), x = h * 2^(132 - F) lies in
  // (-64, 64): digit 0 is x rounded to nearest, and each next digit is 128
  // times the (exact) remainder, rounded; adding 1.5 * 2^23 rounds to an
  // integer and leaves it in the low mantissa bits.
  const int wpr = p.M >= NWARP ? 1 : NWARP / p.M;
  const int bm = warp / wpr, share = warp - bm * wpr;
  const int G4 = p.K >> 2;  // groups of 4 k in a row
  const int gs0 = (share * G4) / wpr, gs1 = ((share + 1) * G4) / wpr;
  float hx[GI][4];
  if (bm < p.M) {
    const float* row = p.h + static_cast<int64_t>(bm) * p.ldh;
    const bool vec = ((reinterpret_cast<uintptr_t>(row) & 15u) == 0);
#pragma unroll
    for (int i = 0; i < GI; ++i) {
      const int g = gs0 + lane + 32 * i;
      if (g < gs1) {
        if (vec) {
          const float4 v4 = *reinterpret_cast<const float4*>(row + 4 * g);
          hx[i][0] = v4.x;
          hx[i][1] = v4.y;
          hx[i][2] = v4.z;
          hx[i][3] = v4.w;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) hx[i][e] = row[4 * g + e];
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) hx[i][e] = 0.f;
      }
    }
    int F = 0;
#pragma unroll
    for (int i = 0; i < GI; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) F = max(F, exp_field(hx[i][e]));
    F = __reduce_max_sync(0xffffffffu, F);
    if (lane == 0 && F > 0) atomicMax(&emax[bm], F);
  }
  __syncthreads();
  if (bm < p.M) {
    const int F = emax[bm];
    if (F != 0 && F != 255) {  // zero (or subnormal) row: digits 0; non-finite: see read-back
      const int n = 132 - F;   // -122 .. 131: two factors of 2^-61 .. 2^66
      const float f1 = __int_as_float((127 + (n >> 1)) << 23);
      const float f2 = __int_as_float((127 + n - (n >> 1)) << 23);
      constexpr float kRound = 12582912.f;  // 1.5 * 2^23
#pragma unroll
      for (int i = 0; i < GI; ++i) {
        const int g = gs0 + lane + 32 * i;
        if (g >= gs1) break;
        uint32_t tb[ND][4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float x = (hx[i][e] * f1) * f2;  // exact for every element that has a nonzero digit
#pragma unroll
          for (int d = 0; d < ND; ++d) {
            const float t = x + kRound;                                // 1.5 * 2^23 + rint(x)
            tb[d][e] = __float_as_uint(t);                             // low byte: rint(x)
            const float r128 = __fmaf_rn(t, 128.f, -kRound * 128.f);  // 128 rint(x), exact
            x = __fmaf_rn(x, 128.f, -r128);                            // 128 (x - rint(x)), exact
          }
        }
        const int k = 4 * g;
        const uint32_t off =
            static_cast<uint32_t>((k >> 5) * (NB * 32) + bm * 256 + ((k >> 4) & 1) * 128 + (k & 15));
#pragma unroll
        for (int d = 0; d < ND; ++d) {
          const uint32_t lo = __byte_perm(tb[d][0], tb[d][1], 0x0040u);
          const uint32_t hi = __byte_perm(tb[d][2], tb[d][3], 0x0040u);
          *reinterpret_cast<uint32_t*>(bs + off + d * 16) = __byte_perm(lo, hi, 0x5410u);
        }
      }
    }
  }
  fence_async_smem();  // B is read by the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 2) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && issued < GS) {
      int s = issued % NS, t = t0 + issued / nst, j = issued - (issued / nst) * nst;
      uint32_t ph = static_cast<uint32_t>(issued / NS) & 1u;
#pragma unroll 1
      for (; issued < GS; ++issued) {
        if (!mbar_wait_bounded(&empty[s], ph ^ 1u, p.timeout_ns, abort_flag, p.err, K_HEADT, 1)) break;
        const int nu = min(SU, upt - SU * j);
        mbar_arrive_expect_tx(&full[s], nu * UB);
        bulk_g2s(stages + s * SB, p.tiles + t * p.tile_bytes + static_cast<int64_t>(j) * SB, nu * UB, &full[s]);
        if (++s == NS) {
          s = 0;
          ph ^= 1u;
        }
        if (++j == nst) {
          j = 0;
          ++t;
        }
      }
    }
    if (lane == 0)
      for (int i = issued > NS ? issued - NS : 0; i < issued; ++i)
        mbar_wait_drain(&full[i % NS], static_cast<uint32_t>(i / NS) & 1u, p.timeout_ns);
  } else if (warp < 2) {
    // ------------------------------------------------------------ MMA issuers
    // Nothing but waits, descriptor adds and MMAs in the loop: scalar work of
    // the issuing thread delays its next MMA.
    const int X = warp;
    if (lane == 0 && (X == 0 || two)) {
      constexpr uint32_t IDESC = (2u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(NB) >> 3) << 17) |
                                 ((static_cast<uint32_t>(TT) >> 4) << 24);
      constexpr uint64_t ASTEP = UB >> 4, BSTEP = (NB * 32) >> 4;  // one K32 step, in 16-byte units
      const long long budget = static_cast<long long>(p.timeout_ns) * 2;  // clocks, at most 2 per ns
      const uint64_t adesc0 = sdesc(smem_u32(stages));
      const uint64_t bdesc0 = sdesc(smem_u32(bs));
      const int tail = upt - SU * (nst - 1);  // units of the last stage of a tile
      // The CTA's stages g = X, X + 2, ... (every stage when issuer 1 is idle);
      // stage g is stage j = g % nst of tile g / nst. With the ring's even size
      // a ring slot always serves the same issuer, which so sees every phase
      // of its barrier in order.
      const int step = two ? 2 : 1;
      int g = two ? X : 0, ti = 0, j = g;  // j < nst: issuer 1 runs only when nst >= 2
      int s = g;                           // ring slot of stage g (g < NS)
      uint32_t ph = 0;
      int cur = -1;                        // the tile whose accumulator takes this issuer's MMAs
      int s_last = -1;                     // ring slot and phase parity of the last commit to empty
      uint32_t ph_last = 0;
      bool first = true;
      uint32_t dt = 0;
#pragma unroll 1
      while (g < GS) {
        if (ti != cur) {
          if (cur >= 0) mma_commit(&dready[2 * X + (cur & 1)]);
          cur = ti;
          const int d = ti & 1;
          if (ti >= 2 && !spin_wait(&dfree[2 * X + d], static_cast<uint32_t>((ti >> 1) - 1) & 1u, budget, abort_flag,
                                    p.err, 2))
            break;
          dt = tmem + static_cast<uint32_t>((2 * X + d) * NB);
          first = true;
        }
        if (!spin_wait(&full[s], ph, budget, abort_flag, p.err, 3)) break;
        tc_fence_after();
        const uint64_t ad = adesc0 + static_cast<uint64_t>(s) * (SB >> 4);
        const uint64_t bd = bdesc0 + static_cast<uint64_t>(j) * (SU * BSTEP);
        if (j < nst - 1 || tail == SU) {
          mma_i8(dt, ad, bd, IDESC, !first);
          mma_i8(dt, ad + ASTEP, bd + BSTEP, IDESC, true);
          mma_i8(dt, ad + 2 * ASTEP, bd + 2 * BSTEP, IDESC, true);
          mma_i8(dt, ad + 3 * ASTEP, bd + 3 * BSTEP, IDESC, true);
        } else {
          for (int q = 0; q < tail; ++q) mma_i8(dt, ad + q * ASTEP, bd + q * BSTEP, IDESC, !first || q != 0);
        }
        first = false;
        mma_commit(&empty[s]);
        s_last = s;
        ph_last = ph;
        g += step;
        j += step;
        while (j >= nst) {
          j -= nst;
          ++ti;
        }
        s += step;
        if (s >= NS) {
          s -= NS;
          ph ^= 1u;
        }
      }
      if (g >= GS && cur >= 0) mma_commit(&dready[2 * X + (cur & 1)]);
      // the last commit to empty covers every MMA of this thread
      if (s_last >= 0) mbar_wait_drain(&empty[s_last], ph_last, p.timeout_ns);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ read back (warps 4-7)
    const int q = warp & 3;
    const int c = 32 * q + lane;
    const uint32_t lanes = static_cast<uint32_t>(32 * q) << 16;
    // weight of digit 0 of row m: 2^(F - 132); NaN for a row with Inf or NaN
    double w0[NMAX];
#pragma unroll
    for (int m = 0; m < NMAX; ++m) {
      const int F = emax[m];
      // (2^-7 for the pairing of the digits below)
      w0[m] = F == 255 ? __longlong_as_double(0x7FF8000000000000ll) : (F == 0 ? 0.0 : ldexp(1.0, F - 139));
    }
    unsigned long long best[NMAX];
#pragma unroll
    for (int m = 0; m < NMAX; ++m) best[m] = 0ull;
#pragma unroll 1
    for (int t = t0; t < t1; ++t) {
      const int ti = t - t0, d = ti & 1;
      const int v = t * TT + c;
      const float sc = *reinterpret_cast<const float*>(p.tiles + t * p.tile_bytes + static_cast<int64_t>(p.K) * TT + 4 * c);
      // suspended waits: a spinning warp here would take issue slots from the
      // issuers, and the accumulators are double-buffered
      bool okw = mbar_wait_bounded(&dready[d], static_cast<uint32_t>(ti >> 1) & 1u, p.timeout_ns, abort_flag, p.err,
                                   K_HEADT, 6);
      if (okw && two)
        okw = mbar_wait_bounded(&dready[2 + d], static_cast<uint32_t>(ti >> 1) & 1u, p.timeout_ns, abort_flag, p.err,
                                K_HEADT, 7);
      if (!__all_sync(0xffffffffu, okw)) break;
      tc_fence_after();
      int acc[NB];
#pragma unroll
      for (int cc = 0; cc < NB; cc += 16) {
        uint32_t a0[16], a1[16];
        tmem_ld16(tmem + lanes + static_cast<uint32_t>(d * NB + cc), a0);
        if (two) tmem_ld16(tmem + lanes + static_cast<uint32_t>((2 + d) * NB + cc), a1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[cc + i] = static_cast<int>(a0[i]) + (two ? static_cast<int>(a1[i]) : 0);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&dfree[d]);
        if (two) mbar_arrive(&dfree[2 + d]);
      }
      if (v < p.V) {
#pragma unroll
        for (int m = 0; m < NMAX; ++m) {
          if (8 * m < NB && m < p.M) {
            // digits in pairs, exact in int32 (|D| <= 2^23): P_i = 128 D_2i + D_2i+1
            const int* D = acc + 8 * m;
            const double pa = static_cast<double>(D[0] * 128 + D[1]);
            const double pb = static_cast<double>(D[2] * 128 + D[3]);
            const double pc = static_cast<double>(D[4] * 128 + D[5]);
            const double pd = static_cast<double>(D[6] * 128 + D[7]);
            // sum_p D_p 2^(-7 p) = 2^-7 (P_a + 2^-14 (P_b + 2^-14 (P_c + 2^-14 P_d)))
            const double sum = fma(fma(fma(pd, 0x1p-14, pc), 0x1p-14, pb), 0x1p-14, pa);
            const float y = static_cast<float>(static_cast<double>(sc) * (sum * w0[m]));
            if (p.keys == nullptr) p.logits[static_cast<int64_t>(m) * p.ldl + v] = y;
            else best[m] = max(best[m], head_key_t(y, static_cast<uint32_t>(v)));
          }
        }
      }
    }
    if (p.keys != nullptr) {
#pragma unroll
      for (int m = 0; m < NMAX; ++m) {
        unsigned long long b = best[m];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) b = max(b, __shfl_xor_sync(0xffffffffu, b, off));
        if (lane == 0 && m < p.M && b != 0ull) atomicMax(p.keys + m, b);
      }
    }
  }

  // ---- teardown: copies landed, MMAs done, tensor-memory reads complete
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  __syncwarp();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TCOLS) : "memory");
}

// ---------------------------------------------------------------- tile layout

struct HeadTileGeom {
  int32_t ntiles;
  int64_t tile_bytes, bytes;
};

bool head_tile_geom(int64_t K, int64_t V, HeadTileGeom* g) {
  if (K < UK || K % UK != 0 || K > KMAX || V <= 0 || V > (int64_t(1) << 30)) return false;
  g->ntiles = static_cast<int32_t>((V + TT - 1) / TT);
  g->tile_bytes = K * TT + TT * 4;
  g->bytes = g->tile_bytes * g->ntiles;
  return true;
}

// One output word (4 codes, or a scale) of the tile layout per thread.
__global__ void i8t_repack_kernel(const int8_t* __restrict__ table, int64_t ldt, const float* __restrict__ scales,
                                  int64_t K, int64_t V, HeadTileGeom g, uint32_t* __restrict__ out) {
  const int64_t words = g.bytes / 4;
  for (int64_t o = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; o < words;
       o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = (o * 4) / g.tile_bytes;
    const int64_t in = o * 4 - t * g.tile_bytes;  // byte in the tile
    uint32_t v = 0;
    if (in < K * TT) {
      const int64_t u = in / UB;
      const int rem = static_cast<int>(in - u * UB);
      const int c = (rem >> 8) * 8 + ((rem >> 4) & 7);  // token in the tile
      const int64_t k0 = u * UK + ((rem >> 7) & 1) * 16 + (rem & 15);
      const int64_t tok = t * TT + c;
      if (tok < V) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          v |= static_cast<uint32_t>(static_cast<uint8_t>(table[(k0 + e) * ldt + tok])) << (8 * e);
      }
    } else {
      const int64_t tok = t * TT + (in - K * TT) / 4;
      v = tok < V ? __float_as_uint(scales[tok]) : 0u;
    }
    out[o] = v;
  }
}

// One table byte or one scale per thread.
__global__ void i8t_restore_kernel(const uint8_t* __restrict__ in, int64_t K, int64_t V, HeadTileGeom g,
                                   int8_t* __restrict__ table, int64_t ldt, float* __restrict__ scales) {
  const int64_t n = K * V + V;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (e < K * V) {
      const int64_t k = e / V, tok = e - k * V;
      const int64_t t = tok / TT, c = tok - t * TT, u = k / UK, kk = k - u * UK;
      table[k * ldt + tok] =
          static_cast<int8_t>(in[t * g.tile_bytes + u * UB + (c >> 3) * 256 + (kk >> 4) * 128 + (c & 7) * 16 + (kk & 15)]);
    } else {
      const int64_t tok = e - K * V, t = tok / TT, c = tok - t * TT;
      scales[tok] = *reinterpret_cast<const float*>(in + t * g.tile_bytes + K * TT + 4 * c);
    }
  }
}

bool aligned_to(const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) == 0; }

template <int NB>
w4_status launch_nb(const HParamsT& p, int grid, cudaStream_t st, const w4host::DeviceInfo& di) {
  using namespace w4host;
  static int configured[64] = {};
  if (di.dev < 64 && !configured[di.dev]) {
    const cudaError_t e =
        cudaFuncSetAttribute(i8t_head_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_MAX);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(i8t_head)");
    configured[di.dev] = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem_for(NB, p.K));
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, i8t_head_kernel<NB>, p);
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch i8t_head");
}

w4_status launch_i8t(const HParamsT& base, const HeadTileGeom& g, cudaStream_t st, const w4host::DeviceInfo& di) {
  HParamsT p = base;
  p.ntiles = g.ntiles;
  p.tile_bytes = g.tile_bytes;
  p.err = di.err;
  p.timeout_ns = w4host::wait_timeout_ns();
  const int grid = static_cast<int>(std::min<int64_t>(di.sms, g.ntiles));
  switch (nb_for(p.M)) {
    case 16: return launch_nb<16>(p, grid, st, di);
    case 32: return launch_nb<32>(p, grid, st, di);
    case 48: return launch_nb<48>(p, grid, st, di);
    default: return launch_nb<64>(p, grid, st, di);
  }
}

w4_status check_i8t(const float* h, int64_t ldh, const void* tiles, int64_t K, int64_t V, int64_t M,
                    HeadTileGeom* g) {
  using namespace w4host;
  if (K < 0 || V < 0 || M < 0) return fail(W4_ERR_SHAPE, "negative size");
  if (M > NMAX) return fail(W4_ERR_SHAPE, "the tensor-core head takes at most %d rows (M=%lld)", NMAX, (long long)M);
  if (M == 0 || V == 0) return W4_OK;
  if (!head_tile_geom(K, V, g))
    return fail(W4_ERR_SHAPE, "the head tile layout takes K %% 32 == 0, 32 <= K <= %d, 0 < V <= 2^30 (K=%lld)", KMAX,
                (long long)K);
  if (h == nullptr || tiles == nullptr) return fail(W4_ERR_NULL, "h and the tiles must not be NULL");
  if (M > 1 && ldh < K) return fail(W4_ERR_SHAPE, "ldh < K");
  if (!aligned_to(h, 4)) return fail(W4_ERR_ALIGN, "h must be 4-byte aligned");
  if (!aligned_to(tiles, 16)) return fail(W4_ERR_ALIGN, "the tiles must be 16-byte aligned");
  return W4_OK;
}

}  // namespace

extern "C" {

size_t i8t_head_repacked_bytes(int64_t K, int64_t V) {
  HeadTileGeom g;
  return head_tile_geom(K, V, &g) ? static_cast<size_t>(g.bytes) : 0;
}

w4_status i8t_head_repack(const int8_t* table, int64_t ldt, const float* scales, int64_t K, int64_t V, void* tiles,
                          void* stream) {
  using namespace w4host;
  HeadTileGeom g;
  if (!head_tile_geom(K, V, &g))
    return fail(W4_ERR_SHAPE, "the head tile layout takes K %% 32 == 0, 32 <= K <= %d, 0 < V <= 2^30", KMAX);
  if (ldt < V) return fail(W4_ERR_SHAPE, "ldt < V");
  if (table == nullptr || scales == nullptr || tiles == nullptr) return fail(W4_ERR_NULL, "NULL buffer");
  if (!aligned_to(scales, 4) || !aligned_to(tiles, 16)) return fail(W4_ERR_ALIGN, "scales 4-byte, tiles 16-byte aligned");
  const DeviceInfo* di = nullptr;
  w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  const int64_t blocks = std::min<int64_t>((g.bytes / 4 + 255) / 256, static_cast<int64_t>(di->sms) * 32);
  i8t_repack_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      table, ldt, scales, K, V, g, static_cast<uint32_t*>(tiles));
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch i8t_repack");
}

w4_status i8t_head_repack_restore(const void* tiles, int64_t K, int64_t V, int8_t* table, int64_t ldt, float* scales,
                                  void* stream) {
  using namespace w4host;
  HeadTileGeom g;
  if (!head_tile_geom(K, V, &g))
    return fail(W4_ERR_SHAPE, "the head tile layout takes K %% 32 == 0, 32 <= K <= %d, 0 < V <= 2^30", KMAX);
  if (ldt < V) return fail(W4_ERR_SHAPE, "ldt < V");
  if (table == nullptr || scales == nullptr || tiles == nullptr) return fail(W4_ERR_NULL, "NULL buffer");
  if (!aligned_to(scales, 4) || !aligned_to(tiles, 16)) return fail(W4_ERR_ALIGN, "scales 4-byte, tiles 16-byte aligned");
  const DeviceInfo* di = nullptr;
  w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  const int64_t blocks = std::min<int64_t>((K * V + V + 255) / 256, static_cast<int64_t>(di->sms) * 32);
  i8t_restore_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(tiles), K, V, g, table, ldt, scales);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch i8t_restore");
}

w4_status i8t_head_logits(const float* h, int64_t ldh, const void* tiles, int64_t K, int64_t V, int64_t M,
                          float* logits, int64_t ldl, void* stream) {
  using namespace w4host;
  HeadTileGeom g;
  w4_status rc = check_i8t(h, ldh, tiles, K, V, M, &g);
  if (rc != W4_OK) return rc;
  if (M == 0 || V == 0) return W4_OK;
  if (logits == nullptr) return fail(W4_ERR_NULL, "logits is NULL");
  if (M > 1 && ldl < V) return fail(W4_ERR_SHAPE, "ldl < V");
  if (!aligned_to(logits, 4)) return fail(W4_ERR_ALIGN, "logits must be 4-byte aligned");
  const DeviceInfo* di = nullptr;
  rc = current_device(&di);
  if (rc != W4_OK) return rc;
  HParamsT p{};
  p.h = h;
  p.ldh = M > 1 ? ldh : K;
  p.tiles = static_cast<const uint8_t*>(tiles);
  p.logits = logits;
  p.ldl = M > 1 ? ldl : V;
  p.keys = nullptr;
  p.K = static_cast<int32_t>(K);
  p.V = static_cast<int32_t>(V);
  p.M = static_cast<int32_t>(M);
  return launch_i8t(p, g, static_cast<cudaStream_t>(stream), *di);
}

w4_status i8t_head_argmax(const float* h, int64_t ldh, const void* tiles, int64_t K, int64_t V, int64_t M,
                          int32_t* tokens, float* best_logits, void* keys, void* stream) {
  using namespace w4host;
  HeadTileGeom g;
  w4_status rc = check_i8t(h, ldh, tiles, K, V, M, &g);
  if (rc != W4_OK) return rc;
  if (M == 0 || V == 0) return W4_OK;
  if (tokens == nullptr || keys == nullptr) return fail(W4_ERR_NULL, "tokens and keys must not be NULL");
  if (!aligned_to(tokens, 4) || !aligned_to(best_logits, 4) || !aligned_to(keys, 8))
    return fail(W4_ERR_ALIGN, "tokens / best 4-byte, keys 8-byte aligned");
  const DeviceInfo* di = nullptr;
  rc = current_device(&di);
  if (rc != W4_OK) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto* k = static_cast<unsigned long long*>(keys);
  cudaError_t e = cudaMemsetAsync(k, 0, static_cast<size_t>(M) * 8, st);
  if (e != cudaSuccess) return cuda_fail(e, "clear argmax keys");
  HParamsT p{};
  p.h = h;
  p.ldh = M > 1 ? ldh : K;
  p.tiles = static_cast<const uint8_t*>(tiles);
  p.logits = nullptr;
  p.ldl = 0;
  p.keys = k;
  p.K = static_cast<int32_t>(K);
  p.V = static_cast<int32_t>(V);
  p.M = static_cast<int32_t>(M);
  rc = launch_i8t(p, g, st, *di);
  if (rc != W4_OK) return rc;
  return launch_argmax_finish(k, M, tokens, best_logits, st);
}

}  // extern "C"
