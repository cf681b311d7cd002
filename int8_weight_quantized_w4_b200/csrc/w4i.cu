// w4i: the decode matmuls (one row of x) on the 5th-generation tensor cores
// with integer MMAs, on W4 weights in their tile layout (w4t_repack).
//
// The weight format is the one of "ONNX export, quantization and the browser
// runtime", section "Quantization (train/quantize.py)", step 2 (dq4): blocks
// of 32 along K, one fp32 scale and one uint4 zero point per (block,
// column), w = (q - zp) * scale; y = x . W with fp32 compute.
//
// Arithmetic. x is written in fixed point against its largest magnitude:
// with |x_k| < 2^E for every k, x_k = 2^(E - 6) sum_p d_pk 2^(-7 p) + r_k,
// p = 0..7, each digit d_pk an integer in [-64, 64] (rounded to nearest one
// at a time, so the remainder after each digit is exact in fp32) and
// |r_k| <= 2^(E - 56): every element within 2^31 of the largest is exact.
// Per block b and column n,
//   sum_{k in b} x_k w_kn = s_bn 2^(E - 6) sum_p 2^(-7 p) E_pbn,
//   E_pbn = sum_{k in b} d_pk (q_kn - zp_bn) = D_pbn - zp_bn Z_pb,
// with D_pbn = sum_k d_pk q_kn formed exactly by an integer MMA (the codes q
// as they are stored, 0..15) and Z_pb = sum_{k in b} d_pk per block, both
// exact in int32; E is exact too. The eight E_p are paired exactly in int32
// (128 E_0 + E_1, ...), weighed in fp32 (one rounding of a value of at most
// about 2^22), scaled by s in fp32 and summed over the blocks in fp32, as a
// plain fp32 evaluation would; the result is multiplied by 2^(E - 13) once.
//
// Design (sm_100a):
//  * w4i_digits_kernel writes, once per call and distinct x, the digits of x
//    in the MMA's B-operand layout (K-major, unswizzled, 8 digit rows; the K
//    order within each 8 rows permuted as the decode below leaves the codes),
//    the block sums Z_pb and 2^(E - 13) into the caller's workspace.
//  * w4i_gemv_kernel: one persistent CTA per SM over a list of 128-column
//    tiles the host deals out largest first. The MMA's M = 128 are the
//    tile's columns (operand A: the codes as bytes, tensor memory), N = 16
//    its digit rows (operand B: the 8 digit rows of x and 8 rows of zeros,
//    shared memory); each block (K = 32) has an accumulator of its own in
//    tensor memory. With A out of shared memory, the weight ring takes
//    almost all of it (14 stages, 147 KB in flight per SM).
//    - warp 2 streams each tile's digits (one bulk copy, from L2) into one of
//      two B slots, and the tile's blocks in groups of four (one bulk copy of
//      up to 10496 bytes, no multicast) through a ring of stages;
//    - warps 4-7 and 12-15, two teams of four, take the groups of one parity
//      each (a warp one quarter of the tile's columns, the tensor-memory
//      lanes it may write): two logic operations per word of 8 nibbles give
//      the codes as bytes in a fixed permutation of K, stored into tensor
//      memory as the A operand, and the group's scales and zero points go to
//      a slot of their own (warp j those of block j); then the stage goes
//      back to the producer;
//    - warps 0 and 1 take the groups of one parity each and issue their MMAs
//      (kind::i8, M 128, N 16, K 32; one per block); one commit frees the A
//      operand, one hands the accumulators to the read-back;
//    - warps 8-11 and 16-19, two sets of one warp per quarter of
//      tensor-memory lanes (a thread per column), read back the blocks of
//      the groups of one parity each, form E_p, weigh and scale it into a
//      running sum; at a tile's end the two sums meet in shared memory and
//      the set that comes second adds them (set 0's first) and applies the
//      fused epilogue.
//  * Every wait is bounded; on timeout the CTA records the error, stops
//    issuing work, lets its copies and MMAs in flight finish, and returns.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <memory>
#include <queue>
#include <vector>

#include "w4_device.cuh"
#include "w4_internal.h"

namespace {

using namespace w4dev;

constexpr int TN = 128;                    // columns of a tile = MMA M
constexpr int BLK = 2624;                  // bytes of one block of a tile (tile layout)
constexpr int GB = 4;                      // blocks per group
constexpr int GBYTES = GB * BLK;           // 10496 bytes per weight stage
constexpr int SZ = 576;                    // scales and zero points of one block
constexpr int SSLOT = GB * SZ;             // 2304 bytes: those of one group
constexpr int KMAX = 3072;                 // rows of K this path takes
constexpr int ND = 8;                      // digits per element of x
constexpr int ICAP = 64;                   // matrices per launch
constexpr int LCAP = 4096;                 // tiles per launch
// Every ring below has an even number of slots and every role pairs with
// the groups of one parity (decode team t, issuer t and read-back set t take
// the groups G with G % 2 == t), so each barrier's phases are all observed,
// in order, by the same waiters: a parity wait is never a phase ahead of a
// phase its waiter has not seen complete (which would pass spuriously).
constexpr int NWS = 14;                    // weight stages
constexpr int NA = 4;                      // A slots: free again once the group's MMAs complete
constexpr int NS = 6;                      // scale slots and accumulator groups: free after the read-back
constexpr int NWARP = 20;
constexpr int NT = NWARP * 32;
// tensor memory: NS groups x 4 blocks x 16 accumulator columns, then NA
// groups x 4 blocks x 8 columns of A (32 code bytes per lane = column)
constexpr uint32_t TCOLS = 512;
constexpr uint32_t TA0 = NS * GB * 16;
static_assert(TA0 + NA * GB * 8 <= TCOLS, "tensor memory of one CTA");
// digits buffer of one x (workspace and B slots): [K/32 x 256 digit bytes]
// [K/32 x 4 int32: the block sums of the digits in pairs, 128 Z_2i + Z_2i+1]
// [double 2^(E - 13)][8 bytes pad]
__host__ __device__ constexpr int dig_bytes(int K) { return K * 8 + K / 2 + 16; }
constexpr int BSLOT = (dig_bytes(KMAX) + 127) / 128 * 128;  // 26240
constexpr int OFF_W = 0;
constexpr int OFF_S = OFF_W + NWS * GBYTES;                 // 146944
constexpr int OFF_B = OFF_S + NS * SSLOT;                   // + 13824
constexpr int OFF_Z = OFF_B + 2 * BSLOT;                    // + 52480: 256 zero bytes, the B rows past the digits
constexpr int OFF_C = OFF_Z + 256;                          // the two read-back sets' partial sums of a tile:
constexpr int CBYTES = 2 * 2 * TN * 4 + 2 * 4 * 4 * 2;      // [tile parity][set][column] + counts + sequence
constexpr int OFF_BAR = OFF_C + CBYTES;
constexpr int NBAR = 2 * NWS + 2 * NA + 3 * NS + 4;
constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory of one CTA");
static_assert(OFF_S % 128 == 0 && OFF_B % 128 == 0 && OFF_Z % 128 == 0 && OFF_BAR % 8 == 0,
              "alignment");
static_assert(NWS % 2 == 0 && NA % 2 == 0 && NS % 2 == 0, "rings pair with group parity");

struct IMat {
  const uint8_t* wt;   // tile layout
  const uint8_t* dig;  // digits of x (workspace)
  float* y;
  const float* bias;
  const float* res;
  int32_t N, nb, act, pad;
};

struct IParams {
  IMat m[ICAP];
  uint32_t first[257];  // CTA c takes list[first[c] .. first[c + 1])
  uint32_t list[LCAP];  // (matrix << 16) | column tile
  ErrorWord* err;
  uint64_t timeout_ns;
};

struct DigSrc {
  const float* x;
  uint8_t* dst;
  int32_t K, pad;
};

struct DigParams {
  DigSrc s[ICAP];
  int32_t count;
};

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// The decode below leaves the codes of a word (rows 8 j + r, r = 0..7, of a
// block) as bytes in the order of rows 0, 4, 1, 5 (w & 0x0F0F0F0F) and 2, 6,
// 3, 7 ((w >> 4) & 0x0F0F0F0F): the tile layout's nibble order. Byte e of
// half hw (0 or 1) holds row (e / 2) + 2 hw + 4 (e % 2); the digits of x take
// the same order, so every product pairs the right x with the right code.

// ---------------------------------------------------------------- digits of x

// One CTA per distinct x. Elements in groups of 4 that share one 32-bit word
// of every digit row: group t is block b = t / 8, word j = (t / 2) % 4, half
// hw = t % 2 (rows {0, 4, 1, 5} or {2, 6, 3, 7} of the 8 at 32 b + 8 j).
__global__ void __launch_bounds__(256) w4i_digits_kernel(const __grid_constant__ DigParams p) {
  __shared__ float xs[KMAX];
  __shared__ int fmax_s;
  pdl_launch_dependents();
  pdl_wait();  // x may be the previous launch's output
  const DigSrc& S = p.s[blockIdx.x];
  const int K = S.K;
  if (threadIdx.x == 0) fmax_s = 0;
  __syncthreads();
  int F = 0;
  for (int k = threadIdx.x; k < K; k += 256) {
    const float v = S.x[k];
    xs[k] = v;
    F = max(F, static_cast<int>((__float_as_uint(v) >> 23) & 0xFFu));
  }
  F = __reduce_max_sync(0xffffffffu, F);
  if ((threadIdx.x & 31) == 0) atomicMax(&fmax_s, F);
  __syncthreads();
  F = fmax_s;
  const int nb = K / 32;
  uint8_t* dig = S.dst;
  int* zs = reinterpret_cast<int*>(dig + nb * 256);
  if (threadIdx.x == 0) {
    // 2^(E - 13) with E = F - 126 (|x| < 2^E): digit 0 weighs 2^(E - 6), and
    // the read-back pairs digits as 128 E_0 + E_1 (a further 2^-7)
    *reinterpret_cast<double*>(dig + nb * 256 + nb * 16) =
        F == 255 ? __longlong_as_double(0x7FF8000000000000ll) : (F == 0 ? 0.0 : ldexp(1.0, F - 139));
  }
  const bool finite = F != 0 && F != 255;
  const int n = 132 - F;  // x * 2^n lies in (-64, 64); two factors of 2^-61 .. 2^66
  const float f1 = __int_as_float((127 + (n >> 1)) << 23);
  const float f2 = __int_as_float((127 + n - (n >> 1)) << 23);
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23: adding it rounds to an integer in the low bits
  const int groups = K / 4;              // a multiple of 8
  for (int t0 = 0; t0 < groups; t0 += 256) {  // uniform trip count: the shuffles below
    const int t = t0 + threadIdx.x;
    const bool act = t < groups;
    const int b = t >> 3, j = (t >> 1) & 3, hw = t & 1;
    uint32_t w[ND];
    int zsum[ND];
#pragma unroll
    for (int d = 0; d < ND; ++d) {
      w[d] = 0u;
      zsum[d] = 0;
    }
    if (act && finite) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        // byte e of the word: row perm^-1(4 hw + e) of the 8
        const int r = (e >> 1) + 2 * hw + 4 * (e & 1);
        float x = (xs[32 * b + 8 * j + r] * f1) * f2;  // exact for every element with a nonzero digit
#pragma unroll
        for (int d = 0; d < ND; ++d) {
          const float tt = x + kRound;
          const int di = __float_as_int(tt) - 0x4B400000;  // rint(x), in [-64, 64]
          w[d] |= (static_cast<uint32_t>(di) & 0xFFu) << (8 * e);
          zsum[d] += di;
          const float r128 = __fmaf_rn(tt, 128.f, -kRound * 128.f);  // 128 rint(x), exact
          x = __fmaf_rn(x, 128.f, -r128);                            // 128 (x - rint(x)), exact
        }
      }
    }
    if (act) {
      const int off = b * 256 + (j >> 1) * 128 + (j & 1) * 8 + hw * 4;
#pragma unroll
      for (int d = 0; d < ND; ++d) *reinterpret_cast<uint32_t*>(dig + off + d * 16) = w[d];
    }
    // block sums: the 8 groups of a block are 8 consecutive lanes
#pragma unroll
    for (int d = 0; d < ND; ++d) {
      int v = zsum[d];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      zsum[d] = v;
    }
    if (act && (t & 7) == 0) {
#pragma unroll
      for (int i = 0; i < ND / 2; ++i) zs[b * 4 + i] = zsum[2 * i] * 128 + zsum[2 * i + 1];
    }
  }
}

// ---------------------------------------------------------------- the GEMV

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
    record_error(err, W4_ERR_TIMEOUT, K_GEMVI, detail);
  }
  return false;
}

// Wait of a warp on the decode -> MMA -> read-back loop: try_wait, then
// short sleeps between tries (a thread suspended with a long time hint wakes
// several hundred clocks after the phase completes, while a tight spin takes
// issue slots from the warps that share its scheduler). Bounded by `budget`
// clocks and the CTA's abort flag; records the error on timeout.
__device__ __forceinline__ bool poll_wait(uint64_t* bar, uint32_t parity, long long budget, volatile int* abort_flag,
                                          ErrorWord* err, int32_t detail) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const long long t0 = clock64();
#pragma unroll 1
  for (uint32_t it = 1;; ++it) {
    __nanosleep(64);
    if (mbar_try_wait(a, parity)) return true;
    if ((it & 15u) == 0 && (*abort_flag || clock64() - t0 > budget)) break;
  }
  if (!*abort_flag) {
    *abort_flag = 1;
    record_error(err, W4_ERR_TIMEOUT, K_GEMVI, detail);
  }
  return false;
}

__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return;
  const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
  while (!mbar_try_wait_sleep(a, parity, 100000u))
    if (globaltimer_ns() - t0 > timeout_ns) return;
}

// K-major, no swizzle, LBO 128 bytes (the two 16-byte K halves), SBO bytes
// between groups of 8 rows, descriptor version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((128u >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// D (s32, tensor memory) = A (s8, tensor memory) . B (s8, shared)^T, K 32.
__device__ __forceinline__ void mma_i8(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, 0, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc)
      : "memory");
}

// Eight 32-bit columns of this warp's 32 tensor-memory lanes.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t* v) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr));
}

// Iterates a CTA's tiles and their groups in order.
struct GroupWalk {
  int i, i1;     // tile index in the list, end
  int mat, ct;   // matrix and column tile of tile i
  int nb, ng;    // blocks and groups of tile i
  int g;         // group within the tile
  int G;         // group index within the CTA
  __device__ void load(const IParams& p) {
    const uint32_t e = p.list[i];
    mat = static_cast<int>(e >> 16);
    ct = static_cast<int>(e & 0xFFFFu);
    nb = p.m[mat].nb;
    ng = (nb + GB - 1) / GB;
  }
  __device__ bool next_group(const IParams& p) {  // false at the end of the CTA's work
    ++G;
    if (++g < ng) return true;
    g = 0;
    if (++i >= i1) return false;
    load(p);
    return true;
  }
};

__global__ void __launch_bounds__(NT, 1) w4i_gemv_kernel(const __grid_constant__ IParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c0 = static_cast<int>(p.first[blockIdx.x]);
  const int c1 = static_cast<int>(p.first[blockIdx.x + 1]);

  uint8_t* wst = smem + OFF_W;
  uint8_t* ssl = smem + OFF_S;
  uint8_t* bsl = smem + OFF_B;
  uint8_t* zrow = smem + OFF_Z;
  uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* wempty = wfull + NWS;
  uint64_t* aready = wempty + NWS;  // [NA] A of the group decoded (both warps of its team)
  uint64_t* afree = aready + NA;    // [NA] the group's MMAs complete (commit)
  uint64_t* sready = afree + NA;    // [NS] scales and zero points of the group copied
  uint64_t* dready = sready + NS;   // [NS] the group's accumulators complete (commit)
  uint64_t* sfree = dready + NS;    // [NS] the group read back
  uint64_t* bfull = sfree + NS;     // [2]
  uint64_t* bempty = bfull + 2;     // [2]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(TCOLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < NWS; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 4);  // the four warps of the team
    }
    for (int a = 0; a < NA; ++a) {
      mbar_init(&aready[a], 4);
      mbar_init(&afree[a], 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sready[s], 4);
      mbar_init(&dready[s], 1);
      mbar_init(&sfree[s], 4);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bfull[s], 1);
      mbar_init(&bempty[s], 10);  // both issuers' commits and the eight read-back warps
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 16) reinterpret_cast<uint4*>(zrow)[threadIdx.x] = make_uint4(0u, 0u, 0u, 0u);
  float* part = reinterpret_cast<float*>(smem + OFF_C);              // [2][2][TN]
  int* ccount = reinterpret_cast<int*>(smem + OFF_C + 2 * 2 * TN * 4);  // [2][4]
  int* cseq = ccount + 8;                                              // [2][4]
  if (threadIdx.x < 16) ccount[threadIdx.x] = 0;
  fence_async_smem();  // the zero rows are read by the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const bool any = c1 > c0;

  // ---- the first weight stages before the wait: the weights are constants
  int issuedG = 0;
  if (warp == 2 && lane == 0 && any) {
    GroupWalk w{c0, c1, 0, 0, 0, 0, 0, 0};
    w.load(p);
    do {
      const IMat& m = p.m[w.mat];
      const int nbg = min(GB, w.nb - GB * w.g);
      const uint8_t* src = m.wt + (static_cast<int64_t>(w.ct) * m.nb + GB * w.g) * BLK;
      mbar_arrive_expect_tx(&wfull[issuedG], nbg * BLK);
      bulk_g2s(wst + issuedG * GBYTES, src, nbg * BLK, &wfull[issuedG]);
      ++issuedG;
    } while (issuedG < NWS && w.next_group(p));
  }
  pdl_launch_dependents();
  pdl_wait();  // the digits, y, bias and the residual follow the previous launch

  if (warp == 2) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && any) {
      GroupWalk w{c0, c1, 0, 0, 0, 0, 0, 0};
      w.load(p);
      int tile = 0;
      do {
        const IMat& m = p.m[w.mat];
        if (w.g == 0) {  // the tile's digits into B slot tile % 2
          const int bs = tile & 1;
          if (tile >= 2 && !mbar_wait_bounded(&bempty[bs], static_cast<uint32_t>((tile >> 1) - 1) & 1u, p.timeout_ns,
                                              abort_flag, p.err, K_GEMVI, 1))
            break;
          const int nbytes = dig_bytes(32 * m.nb);
          mbar_arrive_expect_tx(&bfull[bs], nbytes);
          bulk_g2s(bsl + bs * BSLOT, m.dig, nbytes, &bfull[bs]);
          ++tile;
        }
        if (w.G >= issuedG) {
          const int s = w.G % NWS;
          // polled: a suspended producer wakes late and every stage waits on it
          if (!poll_wait(&wempty[s], static_cast<uint32_t>(w.G / NWS - 1) & 1u,
                         static_cast<long long>(p.timeout_ns) * 2, abort_flag, p.err, 2))
            break;
          const int nbg = min(GB, w.nb - GB * w.g);
          const uint8_t* src = m.wt + (static_cast<int64_t>(w.ct) * m.nb + GB * w.g) * BLK;
          mbar_arrive_expect_tx(&wfull[s], nbg * BLK);
          bulk_g2s(wst + s * GBYTES, src, nbg * BLK, &wfull[s]);
          issuedG = w.G + 1;
        }
      } while (w.next_group(p));
      // let every copy in flight land before the CTA ends
      for (int G = issuedG > NWS ? issuedG - NWS : 0; G < issuedG; ++G)
        mbar_wait_drain(&wfull[G % NWS], static_cast<uint32_t>(G / NWS) & 1u, p.timeout_ns);
      for (int t = tile > 2 ? tile - 2 : 0; t < tile; ++t)
        mbar_wait_drain(&bfull[t & 1], static_cast<uint32_t>(t >> 1) & 1u, p.timeout_ns);
    }
  } else if (warp < 2) {
    // ------------------------------------------------------------ MMA issuers (groups X, X + 2, ...)
    const int X = warp;
    if (lane == 0 && any) {
      constexpr uint32_t IDESC = (2u << 4) | (1u << 7) | (1u << 10) | ((16u >> 3) << 17) | ((128u >> 4) << 24);
      const long long budget = static_cast<long long>(p.timeout_ns) * 2;  // clocks, at most 2 per ns
      GroupWalk w{c0, c1, 0, 0, 0, 0, 0, 0};
      w.load(p);
      int tile = 0, lastG = -1;
      do {
        const int bs = tile & 1;
        if (w.g == 0) {
          if (tile > 0) mma_commit(&bempty[(tile - 1) & 1]);  // this issuer's MMAs of the previous tile
          ++tile;
          if (!spin_wait(&bfull[bs], static_cast<uint32_t>(((tile - 1) >> 1)) & 1u, budget, abort_flag, p.err, 3))
            break;
        }
        if ((w.G & 1) != X) continue;
        const int a = w.G % NA, sl = w.G % NS;
        if (!spin_wait(&aready[a], static_cast<uint32_t>(w.G / NA) & 1u, budget, abort_flag, p.err, 4)) break;
        tc_fence_after();
        const int nbg = min(GB, w.nb - GB * w.g);
        // B rows 0-7: the digits of this K-step; rows 8-15: the zero block
        // (SBO = the distance from the digits to it, so it shrinks by 256
        // bytes with each K-step while the start grows by 256)
        const uint32_t bstart = smem_u32(bsl + ((tile - 1) & 1) * BSLOT) + static_cast<uint32_t>(GB * w.g * 256);
        const uint32_t at = tmem + TA0 + static_cast<uint32_t>(a * GB * 8);
        const uint64_t bd = sdesc(bstart, smem_u32(zrow) - bstart);
        constexpr uint64_t BSTEP = static_cast<uint64_t>(256u >> 4) - (static_cast<uint64_t>(256u >> 4) << 32);
        const uint32_t dt = tmem + static_cast<uint32_t>(sl * GB * 16);
        for (int q = 0; q < nbg; ++q)
          mma_i8(dt + 16 * q, at + 8 * q, bd + static_cast<uint64_t>(q) * BSTEP, IDESC);
        mma_commit(&afree[a]);
        mma_commit(&dready[sl]);
        lastG = w.G;
      } while (w.next_group(p));
      if (tile > 0) mma_commit(&bempty[(tile - 1) & 1]);
      // the last group's commit arrives when every MMA of this thread is done
      if (lastG >= 0) mbar_wait_drain(&dready[lastG % NS], static_cast<uint32_t>(lastG / NS) & 1u, p.timeout_ns);
    }
  } else if ((warp >= 8 && warp < 12) || warp >= 16) {
    // ------------------------------------------------------------ read back (warps 8-11 and 16-19)
    const int q = warp & 3;
    const int c = 32 * q + lane;  // column of the tile
    const uint32_t lanes = static_cast<uint32_t>(32 * q) << 16;
    const long long budget = static_cast<long long>(p.timeout_ns) * 2;  // clocks, at most 2 per ns
    const int set = warp >= 16 ? 1 : 0;  // the groups G with G % 2 == set
    if (any) {
      GroupWalk w{c0, c1, 0, 0, 0, 0, 0, 0};
      w.load(p);
      int tile = -1;
      float acc = 0.f;
      double w0 = 0.0;
      const int4* pz = nullptr;
      do {
        const IMat& m = p.m[w.mat];
        if (w.g == 0) {
          ++tile;
          const bool okb = mbar_wait_bounded(&bfull[tile & 1], static_cast<uint32_t>(tile >> 1) & 1u, p.timeout_ns,
                                             abort_flag, p.err, K_GEMVI, 5);
          if (!__all_sync(0xffffffffu, okb)) break;
          const uint8_t* bsp = bsl + (tile & 1) * BSLOT;
          pz = reinterpret_cast<const int4*>(bsp + m.nb * 256);
          w0 = *reinterpret_cast<const double*>(bsp + m.nb * 256 + m.nb * 16);
          acc = 0.f;
        }
        if ((w.G & 1) == set) {
          const int sl = w.G % NS;
          const uint32_t par = static_cast<uint32_t>(w.G / NS) & 1u;
          const int nbg = min(GB, w.nb - GB * w.g);
          bool okw = poll_wait(&sready[sl], par, budget, abort_flag, p.err, 6);
          if (!__all_sync(0xffffffffu, okw)) break;
          // scales, zero points and block sums while the MMAs finish
          const uint8_t* sz = ssl + sl * SSLOT;
          float sc[GB];
          int zp[GB];
          int4 z[GB];
#pragma unroll
          for (int b = 0; b < GB; ++b) {
            if (b < nbg) {
              sc[b] = *reinterpret_cast<const float*>(sz + b * SZ + 4 * c);
              const uint32_t zw = *reinterpret_cast<const uint32_t*>(sz + b * SZ + 512 + 4 * (c >> 3));
              zp[b] = static_cast<int>((zw >> (4 * (c & 7))) & 0xFu);
              z[b] = pz[GB * w.g + b];  // 128 Z_0 + Z_1, 128 Z_2 + Z_3, ...
            }
          }
          okw = poll_wait(&dready[sl], par, budget, abort_flag, p.err, 7);
          if (!__all_sync(0xffffffffu, okw)) break;
          tc_fence_after();
          uint32_t dv[GB][8];
#pragma unroll
          for (int b = 0; b < GB; ++b)
            if (b < nbg) tmem_ld8(tmem + lanes + static_cast<uint32_t>((sl * GB + b) * 16), dv[b]);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sfree[sl]);
#pragma unroll
          for (int b = 0; b < GB; ++b) {
            if (b < nbg) {
              const int* D = reinterpret_cast<const int*>(dv[b]);
              // P_i = 128 E_2i + E_2i+1 = (128 D_2i + D_2i+1) - zp (128 Z_2i + Z_2i+1), exact in int32
              // and in fp32 (|P| < 2^23: |D| <= 32 * 15 * 64, |Z| <= 32 * 64)
              const float pa = static_cast<float>(D[0] * 128 + D[1] - zp[b] * z[b].x);
              const float pb = static_cast<float>(D[2] * 128 + D[3] - zp[b] * z[b].y);
              const float pc = static_cast<float>(D[4] * 128 + D[5] - zp[b] * z[b].z);
              const float pd = static_cast<float>(D[6] * 128 + D[7] - zp[b] * z[b].w);
              const float v = __fmaf_rn(__fmaf_rn(__fmaf_rn(pd, 0x1p-14f, pc), 0x1p-14f, pb), 0x1p-14f, pa);
              acc = __fmaf_rn(sc[b], v, acc);
            }
          }
        }
        if (w.g == w.ng - 1) {
          // the tile's last group: the two sets' sums meet in shared memory;
          // whichever set comes second writes y = sum(set 0) + sum(set 1)
          const int pb = tile & 1;
          volatile int* seqp = cseq + pb * 4 + q;
          // buffer pb is free once the combine of tile - 2 has finished
          bool okc = true;
          if (lane == 0) {
            const long long tw = clock64();
            while (*seqp != (tile >> 1)) {
              __nanosleep(64);
              if (*abort_flag || clock64() - tw > budget) {
                okc = false;
                break;
              }
            }
          }
          okc = __shfl_sync(0xffffffffu, okc, 0);
          if (!okc) break;
          part[(pb * 2 + set) * TN + c] = acc;
          __threadfence_block();
          __syncwarp();
          int old = 0;
          if (lane == 0) old = atomicAdd(&ccount[pb * 4 + q], 1);
          old = __shfl_sync(0xffffffffu, old, 0);
          if (old == 1) {
            __threadfence_block();
            const float y0 = *reinterpret_cast<volatile float*>(&part[(pb * 2 + 0) * TN + c]);
            const float y1 = *reinterpret_cast<volatile float*>(&part[(pb * 2 + 1) * TN + c]);
            const int64_t n = static_cast<int64_t>(w.ct) * TN + c;
            if (n < m.N) {
              const float v = static_cast<float>(static_cast<double>(y0 + y1) * w0);
              const Epi e{m.bias, m.res, 0, m.act, 0};
              m.y[n] = epi_active(e) ? epi_apply(v, e, 0, n) : v;
            }
            __syncwarp();
            if (lane == 0) {
              ccount[pb * 4 + q] = 0;
              __threadfence_block();
              *seqp = (tile >> 1) + 1;
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bempty[pb]);
        }
      } while (w.next_group(p));
    }
  } else if (warp >= 4 && warp != 8 && warp != 9 && warp != 10 && warp != 11) {
    // ------------------------------------------------------------ decode (warps 4-7 and 12-15)
    // two teams of four; team t takes the groups G with G % 2 == t; warp j
    // of the team decodes columns 32 j .. 32 j + 31 (its tensor-memory lanes)
    // of every block of the group and copies block j's scales
    const int team = warp >= 12 ? 1 : 0, j = warp & 3;
    const uint32_t lanes = static_cast<uint32_t>(32 * j) << 16;
    const long long budget = static_cast<long long>(p.timeout_ns) * 2;  // clocks, at most 2 per ns
    if (any) {
      GroupWalk w{c0, c1, 0, 0, 0, 0, 0, 0};
      w.load(p);
      do {
        if ((w.G & 1) != team) continue;
        const int s = w.G % NWS, a = w.G % NA, sl = w.G % NS;
        bool okw = poll_wait(&wfull[s], static_cast<uint32_t>(w.G / NWS) & 1u, budget, abort_flag, p.err, 8);
        if (okw && w.G >= NA)
          okw = poll_wait(&afree[a], static_cast<uint32_t>(w.G / NA - 1) & 1u, budget, abort_flag, p.err, 9);
        if (okw && w.G >= NS)
          okw = poll_wait(&sfree[sl], static_cast<uint32_t>(w.G / NS - 1) & 1u, budget, abort_flag, p.err, 10);
        if (!__all_sync(0xffffffffu, okw)) break;
        const int nbg = min(GB, w.nb - GB * w.g);
        const uint8_t* stg = wst + s * GBYTES;
        const int c = 32 * j + lane;  // column of the tile = tensor-memory lane
        // A column 8 b + i of lane c: code bytes 4 i .. 4 i + 3 of block b
        const uint32_t at = tmem + lanes + TA0 + static_cast<uint32_t>(a * GB * 8);
#pragma unroll
        for (int b = 0; b < GB; ++b) {
          if (b < nbg) {
            const uint4 nib = *reinterpret_cast<const uint4*>(stg + b * BLK + c * 16);
            uint32_t v[8];
            v[0] = nib.x & 0x0F0F0F0Fu;
            v[1] = (nib.x >> 4) & 0x0F0F0F0Fu;
            v[2] = nib.y & 0x0F0F0F0Fu;
            v[3] = (nib.y >> 4) & 0x0F0F0F0Fu;
            v[4] = nib.z & 0x0F0F0F0Fu;
            v[5] = (nib.z >> 4) & 0x0F0F0F0Fu;
            v[6] = nib.w & 0x0F0F0F0Fu;
            v[7] = (nib.w >> 4) & 0x0F0F0F0Fu;
            tmem_st8(at + 8 * b, v);
          }
        }
        if (j < nbg) {
          // block j's scales (512 bytes) and zero points (64 bytes)
          const uint8_t* src = stg + j * BLK;
          uint8_t* sdst = ssl + sl * SSLOT + j * SZ;
          *reinterpret_cast<uint4*>(sdst + 16 * lane) = *reinterpret_cast<const uint4*>(src + 2048 + 16 * lane);
          if (lane < 4)
            *reinterpret_cast<uint4*>(sdst + 512 + 16 * lane) = *reinterpret_cast<const uint4*>(src + 2560 + 16 * lane);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();  // A is read by the tensor core
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&aready[a]);
          mbar_arrive(&sready[sl]);
          mbar_arrive(&wempty[s]);
        }
      } while (w.next_group(p));
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

// ---------------------------------------------------------------- host plan

bool aligned_to(const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) == 0; }
int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }
bool active(const w4r_desc& d) { return d.M > 0 && d.N > 0 && d.K > 0; }
bool same_x(const w4r_desc& a, const w4r_desc& b) { return a.x == b.x && a.K == b.K; }

// Workspace offset of each descriptor's digits (-1: none), one per distinct
// (x, K). Returns the bytes needed.
int64_t assign_digits(const w4r_desc* d, int count, std::vector<int64_t>* off) {
  off->assign(count, -1);
  int64_t total = 0;
  for (int i = 0; i < count; ++i) {
    if (!active(d[i])) continue;
    for (int k = 0; k < i; ++k)
      if ((*off)[k] >= 0 && same_x(d[k], d[i])) {
        (*off)[i] = (*off)[k];
        break;
      }
    if ((*off)[i] >= 0) continue;
    (*off)[i] = total;
    total += round_up(dig_bytes(static_cast<int>(d[i].K)), 256);
  }
  return total;
}

void plan_tiles(const std::vector<uint32_t>& tiles, const std::vector<int>& cost, int G, IParams* prm) {
  const int T = static_cast<int>(tiles.size());
  std::vector<int> order(T);
  for (int t = 0; t < T; ++t) order[t] = t;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  using Slot = std::pair<int64_t, int>;
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
  for (int c = 0; c < G; ++c) heap.push({0, c});
  std::vector<std::vector<int>> per(G);
  for (int t : order) {
    Slot sl = heap.top();
    heap.pop();
    per[sl.second].push_back(t);
    sl.first += cost[t];
    heap.push(sl);
  }
  uint32_t pos = 0;
  for (int c = 0; c < G; ++c) {
    std::sort(per[c].begin(), per[c].end());
    prm->first[c] = pos;
    for (int t : per[c]) prm->list[pos++] = tiles[t];
  }
  prm->first[G] = pos;
}

struct ILaunch {
  int grid = 0;
  DigParams dig;
  int ndig = 0;
  IParams prm;
};

struct ICallPlan {
  int dev = -1;
  uint64_t used = 0;
  std::vector<w4r_desc> descs;
  const void* ws = nullptr;
  std::vector<std::unique_ptr<ILaunch>> launches;
};

bool same_descs(const std::vector<w4r_desc>& a, const w4r_desc* b, int count) {
  if (static_cast<int>(a.size()) != count) return false;
  for (int i = 0; i < count; ++i) {
    const w4r_desc& p = a[i];
    const w4r_desc& q = b[i];
    if (p.x != q.x || p.wr != q.wr || p.y != q.y || p.M != q.M || p.K != q.K || p.N != q.N || p.bias != q.bias ||
        p.residual != q.residual || p.act != q.act)
      return false;
  }
  return true;
}

// One launch pair (digits, GEMV) per run of at most ICAP matrices and LCAP
// tiles; the digits of an x shared with an earlier launch of the call are
// written again by this launch's digit kernel (same bytes, same place).
void build_plan(const w4r_desc* d, int count, void* ws, int sms, w4dev::ErrorWord* err, ICallPlan* cp) {
  cp->launches.clear();
  std::vector<int64_t> off;
  assign_digits(d, count, &off);
  uint8_t* base = static_cast<uint8_t*>(ws);
  std::unique_ptr<ILaunch> L;
  std::vector<uint32_t> tiles;
  std::vector<int> cost;
  std::vector<int64_t> dig_done;
  int nm = 0;
  auto flush = [&]() {
    if (L && !tiles.empty()) {
      L->grid = std::min(std::min(sms, 256), static_cast<int>(tiles.size()));
      plan_tiles(tiles, cost, L->grid, &L->prm);
      L->prm.err = err;
      cp->launches.push_back(std::move(L));
    }
    L.reset(new ILaunch);
    std::memset(&L->prm, 0, sizeof(L->prm));
    std::memset(&L->dig, 0, sizeof(L->dig));
    tiles.clear();
    cost.clear();
    dig_done.clear();
    nm = 0;
  };
  flush();
  for (int i = 0; i < count; ++i) {
    if (!active(d[i])) continue;
    const int nb = static_cast<int>(d[i].K / 32);
    const int ntiles = static_cast<int>((d[i].N + TN - 1) / TN);
    if (nm == ICAP || static_cast<int>(tiles.size()) + ntiles > LCAP) flush();
    if (std::find(dig_done.begin(), dig_done.end(), off[i]) == dig_done.end()) {
      DigSrc& s = L->dig.s[L->dig.count++];
      s.x = d[i].x;
      s.dst = base + off[i];
      s.K = static_cast<int32_t>(d[i].K);
      dig_done.push_back(off[i]);
    }
    IMat& m = L->prm.m[nm];
    m.wt = static_cast<const uint8_t*>(d[i].wr);
    m.dig = base + off[i];
    m.y = d[i].y;
    m.bias = d[i].bias;
    m.res = d[i].residual;
    m.N = static_cast<int32_t>(d[i].N);
    m.nb = nb;
    m.act = d[i].act;
    for (int ct = 0; ct < ntiles; ++ct) {
      tiles.push_back((static_cast<uint32_t>(nm) << 16) | static_cast<uint32_t>(ct));
      cost.push_back(nb);
    }
    ++nm;
  }
  flush();
}

w4_status launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t st, void** args,
                     const char* what) {
  using namespace w4host;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
  return e == cudaSuccess ? W4_OK : cuda_fail(e, what);
}

w4_status check_idesc(const w4r_desc& d) {
  using namespace w4host;
  if (d.M < 0 || d.K < 0 || d.N < 0) return fail(W4_ERR_SHAPE, "negative size");
  if (d.act < W4_ACT_NONE || d.act > W4_ACT_GELU_ERF) return fail(W4_ERR_VALUE, "unknown activation %d", int(d.act));
  if (d.reserved != 0) return fail(W4_ERR_VALUE, "reserved field must be 0");
  if (d.M == 0 || d.N == 0) return W4_OK;
  if (d.M != 1) return fail(W4_ERR_SHAPE, "the integer tensor-core GEMV takes one row of x (M=%lld)", (long long)d.M);
  if (d.K % 32 != 0 || d.K > KMAX) return fail(W4_ERR_SHAPE, "K must be a multiple of 32 up to %d (K=%lld)", KMAX,
                                             (long long)d.K);
  if (d.N % 8 != 0 || d.N > (int64_t(1) << 23)) return fail(W4_ERR_SHAPE, "N must be a multiple of 8 (N=%lld)",
                                                            (long long)d.N);
  if (d.K == 0) return W4_OK;
  if (d.x == nullptr || d.wr == nullptr || d.y == nullptr) return fail(W4_ERR_NULL, "x, wr and y must not be NULL");
  if (!aligned_to(d.x, 4) || !aligned_to(d.y, 4)) return fail(W4_ERR_ALIGN, "x and y must be 4-byte aligned");
  if (!aligned_to(d.wr, 16)) return fail(W4_ERR_ALIGN, "wr must be 16-byte aligned");
  if ((d.bias != nullptr && !aligned_to(d.bias, 4)) || (d.residual != nullptr && !aligned_to(d.residual, 4)))
    return fail(W4_ERR_ALIGN, "bias and residual must be 4-byte aligned");
  if ((d.N + TN - 1) / TN > 0xFFFF) return fail(W4_ERR_SHAPE, "N too large");
  return W4_OK;
}

}  // namespace

extern "C" {

size_t w4i_workspace_size(const w4t_desc* descs, int32_t count) {
  if (descs == nullptr || count <= 0) return 0;
  std::vector<int64_t> off;
  return static_cast<size_t>(assign_digits(descs, count, &off));
}

w4_status w4i_matmul_grouped(const w4t_desc* descs, int32_t count, void* workspace, size_t workspace_bytes,
                             void* stream) {
  using namespace w4host;
  if (count < 0) return fail(W4_ERR_SHAPE, "negative count");
  if (count == 0) return W4_OK;
  if (descs == nullptr) return fail(W4_ERR_NULL, "descs is NULL");
  int work = 0;
  for (int32_t i = 0; i < count; ++i) {
    const w4_status rc = check_idesc(descs[i]);
    if (rc != W4_OK) {
      char why[256];
      snprintf(why, sizeof(why), "%s", w4_last_error());
      return fail(rc, "descriptor %d: %s", i, why);
    }
    if (active(descs[i])) ++work;
  }
  const DeviceInfo* di = nullptr;
  w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int32_t i = 0; i < count; ++i) {
    const w4r_desc& d = descs[i];
    if (d.M > 0 && d.N > 0 && d.K == 0) {
      w4_desc z{};
      z.y = d.y;
      z.ldy = d.N;
      z.M = d.M;
      z.N = d.N;
      z.bias = d.bias;
      z.residual = d.residual;
      z.ldr = d.N;
      z.act = d.act;
      rc = launch_zero_fill(d.y, d.N, d.M, d.N, st, &z);
      if (rc != W4_OK) return rc;
    }
  }
  if (work == 0) return W4_OK;
  std::vector<int64_t> off;
  const int64_t need = assign_digits(descs, count, &off);
  if (workspace == nullptr) return fail(W4_ERR_WORKSPACE, "workspace is NULL, %lld bytes needed", (long long)need);
  if (!aligned_to(workspace, 16)) return fail(W4_ERR_WORKSPACE, "workspace must be 16-byte aligned");
  if (static_cast<int64_t>(workspace_bytes) < need)
    return fail(W4_ERR_WORKSPACE, "workspace of %zu bytes, %lld needed", workspace_bytes, (long long)need);

  static thread_local std::unique_ptr<ICallPlan[]> cache;
  static thread_local uint64_t clock = 0;
  constexpr int kEntries = 4;
  if (!cache) cache.reset(new ICallPlan[kEntries]);
  ++clock;
  ICallPlan* hit = nullptr;
  for (int e = 0; e < kEntries && hit == nullptr; ++e)
    if (cache[e].dev == di->dev && cache[e].ws == workspace && same_descs(cache[e].descs, descs, count)) hit = &cache[e];
  if (hit == nullptr) {
    int victim = 0;
    for (int e = 1; e < kEntries; ++e)
      if (cache[e].used < cache[victim].used) victim = e;
    ICallPlan& cp = cache[victim];
    cp.dev = -1;
    build_plan(descs, count, workspace, di->sms, di->err, &cp);
    cp.descs.assign(descs, descs + count);
    cp.ws = workspace;
    cp.dev = di->dev;
    hit = &cp;
  }
  hit->used = clock;
  static int configured[64] = {};
  if (di->dev < 64 && !configured[di->dev]) {
    const cudaError_t e = cudaFuncSetAttribute(w4i_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(w4i_gemv)");
    configured[di->dev] = 1;
  }
  const uint64_t tmo = wait_timeout_ns();
  for (auto& L : hit->launches) {
    void* dargs[] = {&L->dig};
    rc = launch_pdl(reinterpret_cast<const void*>(w4i_digits_kernel), dim3(L->dig.count), dim3(256), 0, st, dargs,
                    "launch w4i_digits");
    if (rc != W4_OK) return rc;
    L->prm.timeout_ns = tmo;
    void* gargs[] = {&L->prm};
    rc = launch_pdl(reinterpret_cast<const void*>(w4i_gemv_kernel), dim3(L->grid), dim3(NT), SMEM_BYTES, st, gargs,
                    "launch w4i_gemv");
    if (rc != W4_OK) return rc;
  }
  return W4_OK;
}

w4_status w4i_matmul(const w4t_desc* d, void* workspace, size_t workspace_bytes, void* stream) {
  return w4i_matmul_grouped(d, 1, workspace, workspace_bytes, stream);
}

}  // extern "C"
