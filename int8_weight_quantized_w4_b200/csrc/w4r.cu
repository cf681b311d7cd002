// w4r: the streaming layout of a W4 weight, and the decode GEMV (M = 1) that
// reads it.
//
// The weight format is the one of "ONNX export, quantization and the browser
// runtime", section "Quantization (train/quantize.py)", step 2 (dq4): blocks
// of 32 along K, one fp32 scale and one uint4 zero point per (block,
// column), w = (q - zp) * scale. The streaming layout holds exactly the same
// 32-bit words as the three page-format buffers (nibble words of 8
// consecutive columns of one row, fp32 scales, zero-point words of 8
// columns), only in another order: the order in which one warp of the GEMV
// consumes them. Repacking is a permutation of words, done once when the
// weights are loaded; the GEMV then streams each warp's share of the weight as
// one contiguous run of bytes, so every copy is a plain bulk copy with no
// tensor map, no split along K and no scratch memory.
//
// Layout (K % 32 == 0, N % 8 == 0; nb = K / 32):
//   gs = 32 / gcd(nb, 32) strips of 8 columns form a group (8 * gs columns,
//   all K rows); A = gs * nb / 32 rounds make a group; a round is 5248 bytes,
//   one 164-byte "atom" (8 columns x 32 rows, one block) for each of 32 lanes:
//     lane l: strip s = l % gs, phase p = l / gs, block b = p + r * (32 / gs)
//     [0, 4096)     nibble words: word j of 16-byte chunk c of lane l at
//                   c * 512 + l * 16 + j * 4 is row 32 b + 4 c + j, columns
//                   8 (G gs + s) .. +7 of the [K, N] nibble tensor (the
//                   page's aligned 4-byte word: nibble i = column +i)
//     [4096, 5120)  scales: float i of lane l at 4096 + (i / 4) * 512 + l * 16
//                   + (i % 4) * 4 is scale[b][8 (G gs + s) + i]
//     [5120, 5248)  zero-point words: lane l at 5120 + l * 4 (nibble i = the
//                   zero point of column +i in block b)
//   Groups follow each other in column order; strips past N (when N is not a
//   multiple of 8 gs) are zero in the repacked buffer and never written.
//
// GEMV design (sm_100a, M = 1):
//  * One persistent CTA per SM takes a contiguous share of the launch's groups
//    (all matrices' groups in one flat list), cut by the host so that every
//    CTA streams about the same number of rounds (a group is nb gs / 32
//    rounds: 3 for K = 3072, 8 for K = 8192).
//    Each of its 16 warps is an independent stream: warp w owns the groups
//    lo + w, lo + w + 16, ... of that share, so every output column is summed
//    inside one warp, with no partial sums in memory and no workspace. For
//    the GPT-2 shapes a group is 96 atoms (15.7 KB) and a CTA about 24 groups.
//  * A warp streams its rounds, group after group, through a ring of 2
//    stages; its lane 0 issues one bulk copy per round (no multicast) as soon
//    as the stage it refills has been read, so the SM keeps up to 32 rounds
//    (168 KB) of its stream in flight. Four warps per scheduler (measured
//    against 3 warps x 3 stages and 2 x 4: 15.7 vs 16.2 and 18.8 us for the
//    GPT-2 body) hide more of the decode's dependency stalls.
//  * The CTA stages the x of every matrix its share touches in shared memory
//    as [row quad c][block b][4 floats], so lanes reading different blocks hit
//    different banks (the host splits a launch whose shares would need more
//    than 14336 floats).
//  * The launch lets the next launch in the stream start early (programmatic
//    dependent launch): a CTA requests its first rounds before it waits for
//    the previous launch to finish, and reads x / writes y only after that
//    wait. The weights are constants of the model; x and y may belong to the
//    previous launch.
//  * Dequantisation: one LOP3 per weight builds the float 2^23 + q*16^j
//    exactly (nibble j of a half-word); rows k and k+1 are taken together, so
//    one FADD2 subtracts the zero point's float from both (exact) and one
//    FFMA2 accumulates with (x_k, x_k+1). The scale (times 16^-j) is applied
//    once per block and column: y += s * sum_k x_k (q_k - zp).
//  * The 32 / gs lanes of a strip are added by a butterfly of shuffles; the
//    lane with phase 0 writes 8 columns through the fused epilogue.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "w4_device.cuh"
#include "w4_internal.h"

namespace {

using namespace w4dev;

constexpr int ROUND_BYTES = 5248;
constexpr int NIB_BYTES = 4096;
constexpr int SC_BYTES = 1024;
constexpr int ROUND_WORDS = ROUND_BYTES / 4;  // 1312
constexpr int PW = 16;                        // warps per CTA, each its own stream
constexpr int PST = 2;                        // stages per warp
constexpr int RCAP = 128;                     // matrices per launch
// floats of x a CTA can hold: 14336 takes any three consecutive matrices of
// a stack with K up to 3072, 3072 and 8192 (the range of a CTA over a
// 128-matrix launch touches at most three), so such a stack is one launch
constexpr int XCAP = 14336;
constexpr int XCAP_STEP = 12288;              // the same in the fused step, whose CTA also holds h
constexpr int STAGE_SMEM = PW * PST * ROUND_BYTES;
constexpr int SMEM_BYTES = STAGE_SMEM + XCAP * 4 + PW * PST * 8 + PW * 4;
// the fused decode step: the head's rounds share the stages, its h follows
constexpr int HROUND = w4host::kStreamHeadRound;  // table bytes of a head round
constexpr int HKS = 2048;                         // rows of the head's h a CTA of the step holds
constexpr int SMEM_STEP = STAGE_SMEM + XCAP_STEP * 4 + PW * PST * 8 + PW * 4 + HKS * 4;
static_assert(HROUND + 32 * 32 <= ROUND_BYTES, "a head round and its scales fit a stage");
static_assert(SMEM_BYTES <= 227 * 1024 && SMEM_STEP <= 227 * 1024, "shared memory of one CTA");
static_assert((STAGE_SMEM + XCAP_STEP * 4 + PW * PST * 8 + PW * 4) % 16 == 0, "h 16-byte aligned");

struct RMat {
  const uint8_t* wr;
  const float* x;
  float* y;
  const float* bias;
  const float* res;
  int64_t ldr;
  int32_t K;
  int32_t N;
  int32_t g0;       // first group of this matrix in the launch's flat list
  int32_t ngroups;  // groups of 8 gs columns
  int32_t act;
  int32_t gsl;      // log2(gs)
};

// The int8 head in its streaming layout, streamed by the same launch (the
// fused decode step): groups of 8 * 2^gsl token columns, A rounds of table
// bytes each, the group's scales after its last round.
struct RHead {
  const uint8_t* tr;
  const float* h;
  float* logits;              // or nullptr: greedy decoding into keys
  unsigned long long* keys;   // the 64-bit (logit, token) key of the maximum
  int64_t group_bytes;
  int32_t K, V, gsl, A;
};

constexpr int GMAX = 256;  // CTAs of a launch at most

struct RParams {
  RMat m[RCAP];
  int32_t count;
  int32_t T;   // body groups of the launch
  int32_t TH;  // head groups (the fused step; 0 otherwise)
  RHead hd;
  // body groups of CTA c: [cfirst[c], cfirst[c + 1]), cut so that every CTA
  // streams about the same number of rounds (groups of a large K have more)
  int32_t cfirst[GMAX + 1];
  ErrorWord* err;
  uint64_t timeout_ns;
};

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Range of groups [lo, hi) of CTA c out of G (T * G < 2^31 by the host).
__device__ __forceinline__ int range_lo(int c, int T, int G) { return (c * T) / G; }

// Matrix holding flat group gg: the last one whose first group is <= gg.
__device__ __forceinline__ int mat_of(const RParams& p, int gg) {
  int lo = 0, hi = p.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.m[mid].g0 <= gg) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// One atom: 8 columns x 32 rows for this lane, accumulated into acc[0..7].
// st: the stage; xb: x of the atom's block in the [c][b][4] layout, c-th
// quad at xb + c * xq floats.
__device__ __forceinline__ void atom_m1(const uint8_t* st, int lane, const float* xb, int xq, uint32_t kMagic,
                                        float (&acc)[8]) {
  const uint32_t zw = *reinterpret_cast<const uint32_t*>(st + NIB_BYTES + SC_BYTES + lane * 4);
  float2 nz[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    // -(2^23 + zp 16^j): the nibble in the mantissa of -2^23
    const float z = __uint_as_float(0xCB000000u | ((i < 4 ? zw : (zw >> 16)) & (0xFu << (4 * (i & 3)))));
    nz[i] = make_float2(z, z);
  }
  float2 P[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) P[i] = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 wv = *reinterpret_cast<const uint4*>(st + c * 512 + lane * 16);
    const float4 x4 = *reinterpret_cast<const float4*>(xb + c * xq);
    const float2 xa = make_float2(x4.x, x4.y);
    const float2 xb2 = make_float2(x4.z, x4.w);
    const uint32_t wl[4] = {wv.x, wv.y, wv.z, wv.w};
    uint32_t wh[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) wh[t] = __umulhi(wl[t], 65536u);  // wl >> 16 on the FMA pipe
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int sl = i & 3;
      const float2 m01 = make_float2(magic_nib_r(i < 4 ? wl[0] : wh[0], kMagic, sl),
                                     magic_nib_r(i < 4 ? wl[1] : wh[1], kMagic, sl));
      const float2 m23 = make_float2(magic_nib_r(i < 4 ? wl[2] : wh[2], kMagic, sl),
                                     magic_nib_r(i < 4 ? wl[3] : wh[3], kMagic, sl));
      P[i] = __ffma2_rn(xa, __fadd2_rn(m01, nz[i]), P[i]);
      P[i] = __ffma2_rn(xb2, __fadd2_rn(m23, nz[i]), P[i]);
    }
  }
  const float4 s0 = *reinterpret_cast<const float4*>(st + NIB_BYTES + lane * 16);
  const float4 s1 = *reinterpret_cast<const float4*>(st + NIB_BYTES + 512 + lane * 16);
  const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = fmaf(P[i].x + P[i].y, sv[i] * inv_slot_scale(i & 3), acc[i]);
}

// The rounds one warp streams, in order: units u = warp + PW t of its CTA,
// each a group of A rounds; in the fused step the CTA's nhc head groups come
// first (unit u < nhc is head group hlo + u), then its body groups (unit u is
// body group lo + u - nhc). Producer (lane 0) and consumers walk the same
// sequence.
struct RoundWalk {
  int t, r, ngw;  // unit ordinal of this warp, round in it, units of this warp
  int g, A;       // matrix of the current body group, rounds of the current unit
  const uint8_t* base;
  int rb, last;   // bytes between rounds; bytes of the unit's last round
};

template <bool HEAD>
__device__ __forceinline__ void walk_group(RoundWalk& w, const RParams& p, int lo, int nhc, int hlo, int warp) {
  const int u = warp + PW * w.t;
  if (HEAD && u < nhc) {
    w.A = p.hd.A;
    w.base = p.hd.tr + static_cast<int64_t>(hlo + u) * p.hd.group_bytes;
    w.rb = HROUND;
    w.last = HROUND + (32 << p.hd.gsl);  // the group's scales ride on its last round
    return;
  }
  const int gg = lo + u - nhc;
  while (w.g + 1 < p.count && p.m[w.g + 1].g0 <= gg) ++w.g;
  const RMat& m = p.m[w.g];
  w.A = ((m.K >> 5) << m.gsl) >> 5;
  w.base = m.wr + static_cast<int64_t>(gg - m.g0) * w.A * ROUND_BYTES;
  w.rb = ROUND_BYTES;
  w.last = ROUND_BYTES;
}

template <bool HEAD>
__global__ void __launch_bounds__(PW * 32, 1) w4r_gemv_m1_kernel(const __grid_constant__ RParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int lo = p.cfirst[blockIdx.x];
  const int hi = p.cfirst[blockIdx.x + 1];
  const int nbc = hi - lo;  // body groups of this CTA
  const int hlo = HEAD ? range_lo(blockIdx.x, p.TH, G) : 0;
  const int nhc = HEAD ? range_lo(blockIdx.x + 1, p.TH, G) - hlo : 0;  // head groups of this CTA
  const int units = nbc + nhc;
  const int ngw = units > warp ? (units - warp + PW - 1) / PW : 0;  // units of this warp

  constexpr int XC = HEAD ? XCAP_STEP : XCAP;
  uint8_t* stg = smem + warp * (PST * ROUND_BYTES);
  float* xs = reinterpret_cast<float*>(smem + STAGE_SMEM);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + STAGE_SMEM + XC * 4) + warp * PST;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + STAGE_SMEM + XC * 4 + PW * PST * 8) + warp;
  // the head's h (fused step only)
  float* hs = reinterpret_cast<float*>(smem + STAGE_SMEM + XC * 4 + PW * PST * 8 + PW * 4);

  // ---- x into L2 now: a cache hint only (the values are read after the
  // wait), so that the staging below does not queue behind weight bytes
  if (threadIdx.x == 0) {
    if (nbc > 0) {
      const int g1 = mat_of(p, hi - 1);
      for (int g = mat_of(p, lo); g <= g1; ++g)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.m[g].x), "r"(p.m[g].K * 4) : "memory");
    }
    if (HEAD && nhc > 0)
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.hd.h), "r"(p.hd.K * 4) : "memory");
  }
  // ---- the first round of every warp before the wait: the weights do not
  // depend on the previous launch, so they stream while it finishes
  const int gfirst = nbc > 0 ? mat_of(p, lo) : 0;
  RoundWalk iw{0, 0, ngw, gfirst, 0, nullptr, 0, 0};  // issue cursor, kept in step by every lane
  int issued = 0;
  // one bulk copy of the round under the cursor into stage `stage`; the
  // cursor moves on (warp-uniform)
  auto issue = [&](int stage) {
    if (lane == 0) {
      const uint32_t bytes = static_cast<uint32_t>(iw.r == iw.A - 1 ? iw.last : iw.rb);
      mbar_arrive_expect_tx(&bar[stage], bytes);
      bulk_g2s(stg + stage * ROUND_BYTES, iw.base + static_cast<int64_t>(iw.r) * iw.rb, bytes, &bar[stage]);
    }
    ++issued;
    if (++iw.r == iw.A) {
      iw.r = 0;
      if (++iw.t < ngw) walk_group<HEAD>(iw, p, lo, nhc, hlo, warp);
    }
  };
  if (ngw > 0) {
    walk_group<HEAD>(iw, p, lo, nhc, hlo, warp);
    if (lane == 0) {
      for (int s = 0; s < PST; ++s) mbar_init(&bar[s], 1);
      *abort_flag = 0;
      fence_mbar_init();
    }
    issue(0);
  }
  __syncwarp();
  pdl_launch_dependents();
  pdl_wait();  // x, h and the outputs may be the previous launch's

  // ---- x of every matrix this CTA's range touches, [quad c][block b][4]
  // each: requested before the rest of the weights, which would otherwise
  // queue ahead of it
  const int glast = nbc > 0 ? mat_of(p, hi - 1) : gfirst;
  if (nbc > 0) {
    int xo = 0;
    for (int g = gfirst; g <= glast; ++g) {
      const int K = p.m[g].K;
      const int nb = K >> 5;
      const float* xg = p.m[g].x;
      for (int i = threadIdx.x; i < (K >> 2); i += PW * 32) {
        const int b = i >> 3, c = i & 7;
        cp_async_16(xs + xo + (c * nb + b) * 4, xg + 4 * i, 16);
      }
      xo += K;
    }
  }
  cp_async_commit();
  // ---- the head's h, [row pair c][16-row block b][2]
  if (HEAD && nhc > 0) {
    const int nbh = p.hd.K >> 4;
    for (int i = threadIdx.x; i < (p.hd.K >> 2); i += PW * 32) {
      const int b = i >> 2, q = i & 3;  // floats 16 b + 4 q .. +3: row pairs 2q, 2q+1
      const float4 v = __ldg(reinterpret_cast<const float4*>(p.hd.h) + i);
      *reinterpret_cast<float2*>(hs + ((2 * q) * nbh + b) * 2) = make_float2(v.x, v.y);
      *reinterpret_cast<float2*>(hs + ((2 * q + 1) * nbh + b) * 2) = make_float2(v.z, v.w);
    }
  }
  cp_async_wait_group<0>();
  __syncthreads();
  // ---- the warp's other stages, once x is in: the first round is already
  // here or in flight, so the stream does not stall meanwhile
  for (int s = 1; s < PST && iw.t < ngw; ++s) issue(s);
  if (ngw == 0) return;

  uint32_t kMagic;  // 0x4B000000 (the bits of 2^23) held in a register
  asm("mov.b32 %0, 0x4B000000;" : "=r"(kMagic));

  bool ok = true;
  int s = 0;
  uint32_t par = 0;
  int g = gfirst;
  int xo = 0;  // x offset of matrix g in shared memory
#pragma unroll 1
  for (int t = 0; t < ngw && ok; ++t) {
    const int u = warp + PW * t;
    if (HEAD && u < nhc) {
      // ---------------------------------------------------- a head group
      const int hg = hlo + u;
      const int gsl = p.hd.gsl;
      const int gs = 1 << gsl;
      const int A = p.hd.A;
      const int phase = lane >> gsl;
      const int pstride = 32 >> gsl;
      const float* hw = hs + phase * 2;
      const int hq = (p.hd.K >> 4) * 2;
      const float2 nbias = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
      float2 P[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) P[i] = make_float2(0.f, 0.f);
      float sv[8];
#pragma unroll 1
      for (int r = 0; r < A; ++r) {
        ok = mbar_wait_bounded(&bar[s], par, p.timeout_ns, abort_flag, p.err, K_GEMVR, 3);
        if (__any_sync(0xffffffffu, !ok)) {
          ok = false;
          break;
        }
        const uint8_t* st = stg + s * ROUND_BYTES;
        atom_i8(st, lane, hw + r * pstride * 2, hq, kMagic, nbias, P);
        if (r == A - 1) {
          const float4* sp = reinterpret_cast<const float4*>(st + HROUND + (lane & (gs - 1)) * 32);
          const float4 s0 = sp[0], s1 = sp[1];
          sv[0] = s0.x; sv[1] = s0.y; sv[2] = s0.z; sv[3] = s0.w;
          sv[4] = s1.x; sv[5] = s1.y; sv[6] = s1.z; sv[7] = s1.w;
        }
        __syncwarp();
        if (iw.t < ngw) {  // refill this stage with the round PST ahead
          if (lane == 0) fence_proxy_async_smem();
          issue(s);
        }
        if (++s == PST) {
          s = 0;
          par ^= 1u;
        }
      }
      if (!ok) break;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = P[i].x + P[i].y;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1)
        if (off >= gs) {
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
        }
      const int col = ((hg << gsl) + (lane & (gs - 1))) * 8;
      if (p.hd.keys != nullptr) {
        unsigned long long best = 0ull;
        if (phase == 0) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (col + i < p.hd.V) best = max(best, head_key(acc[i] * sv[i], static_cast<uint32_t>(col + i)));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
        if (lane == 0 && best != 0ull) atomicMax(p.hd.keys, best);
      } else if (phase == 0) {
        float* lp = p.hd.logits + col;
        if (col + 8 <= p.hd.V) {
#pragma unroll
          for (int i = 0; i < 8; ++i) lp[i] = acc[i] * sv[i];
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (col + i < p.hd.V) lp[i] = acc[i] * sv[i];
        }
      }
      continue;
    }
    // ------------------------------------------------------ a body group
    const int gg = lo + u - nhc;
    while (g < glast && p.m[g + 1].g0 <= gg) {
      xo += p.m[g].K;
      ++g;
    }
    const RMat& m = p.m[g];
    const int nb = m.K >> 5;
    const int gsl = m.gsl;
    const int A = (nb << gsl) >> 5;
    const int gs = 1 << gsl;
    const int phase = lane >> gsl;
    const int pstride = 32 >> gsl;
    const float* xw = xs + xo + phase * 4;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll 1
    for (int r = 0; r < A; ++r) {
      ok = mbar_wait_bounded(&bar[s], par, p.timeout_ns, abort_flag, p.err, K_GEMVR, 1);
      if (__any_sync(0xffffffffu, !ok)) {
        ok = false;
        break;
      }
      atom_m1(stg + s * ROUND_BYTES, lane, xw + r * pstride * 4, nb * 4, kMagic, acc);
      __syncwarp();
      if (iw.t < ngw) {  // refill this stage with the round PST ahead (the walk is warp-uniform)
        if (lane == 0) fence_proxy_async_smem();
        issue(s);
      }
      if (++s == PST) {
        s = 0;
        par ^= 1u;
      }
    }
    if (!ok) break;

    // ---- the lanes of a strip: butterfly over the phase bits
#pragma unroll
    for (int off = 1; off < 32; off <<= 1)
      if (off >= gs) {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
      }
    const int col = (((gg - m.g0) << gsl) + (lane & (gs - 1))) * 8;
    if (phase == 0 && col < m.N) {
      float* yp = m.y + col;
      const Epi epi{m.bias, m.res, m.ldr, m.act, 0};
      float v[8];
      if (epi_active(epi)) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = epi_apply(acc[i], epi, 0, col + i);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = acc[i];
      }
      if ((reinterpret_cast<uintptr_t>(yp) & 15) == 0) {
        reinterpret_cast<float4*>(yp)[0] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4*>(yp)[1] = make_float4(v[4], v[5], v[6], v[7]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) yp[i] = v[i];
      }
    }
  }

  if (!ok && lane == 0) {
    // copies still in flight must land before the CTA exits: wait (bounded)
    // for the last fill of every stage
    for (int st = 0; st < PST; ++st) {
      const int fills = issued > st ? (issued - st + PST - 1) / PST : 0;
      if (fills > 0) mbar_wait_bounded(&bar[st], (fills - 1) & 1, p.timeout_ns, nullptr, p.err, K_GEMVR, 2);
    }
  }
}

// ---------------------------------------------------------------- repacking

struct RepackGeom {
  int32_t nb, gsl, A, ngroups;
  int64_t words;  // 32-bit words of the repacked buffer
};

// Where word o of the repacked buffer comes from: kind 0 nibble word, 1
// scale, 2 zero-point word; src = its index in that page-format array as
// 32-bit words; false for a padding word (a strip past N).
__device__ __forceinline__ bool repack_source(int64_t o, const RepackGeom& g, int64_t N, int* kind, int64_t* src) {
  const int64_t round_id = o / ROUND_WORDS;
  const int w = static_cast<int>(o - round_id * ROUND_WORDS);
  const int64_t group = round_id / g.A;
  const int r = static_cast<int>(round_id - group * g.A);
  int lane, row = 0, i = 0;
  if (w < 1024) {
    const int c = w >> 7;
    lane = (w >> 2) & 31;
    row = 4 * c + (w & 3);
    *kind = 0;
  } else if (w < 1280) {
    const int v = w - 1024;
    lane = (v >> 2) & 31;
    i = (v >> 7) * 4 + (v & 3);
    *kind = 1;
  } else {
    lane = w - 1280;
    *kind = 2;
  }
  const int gs = 1 << g.gsl;
  const int strip = lane & (gs - 1);
  const int phase = lane >> g.gsl;
  const int64_t b = phase + static_cast<int64_t>(r) * (32 >> g.gsl);
  const int64_t col = (group * gs + strip) * 8;
  if (col >= N) return false;
  if (*kind == 0) *src = ((b * 32 + row) * N + col) >> 3;
  else if (*kind == 1) *src = b * N + col + i;
  else *src = (b * N + col) >> 3;
  return true;
}

__global__ void w4r_repack_kernel(const uint32_t* __restrict__ qw, const uint32_t* __restrict__ sc,
                                  const uint32_t* __restrict__ zp, int64_t N, RepackGeom g, uint32_t* __restrict__ out) {
  for (int64_t o = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; o < g.words;
       o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int kind;
    int64_t s;
    uint32_t v = 0;
    if (repack_source(o, g, N, &kind, &s)) v = kind == 0 ? qw[s] : (kind == 1 ? sc[s] : zp[s]);
    out[o] = v;
  }
}

__global__ void w4r_restore_kernel(const uint32_t* __restrict__ in, int64_t N, RepackGeom g, uint32_t* __restrict__ qw,
                                   uint32_t* __restrict__ sc, uint32_t* __restrict__ zp) {
  for (int64_t o = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; o < g.words;
       o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int kind;
    int64_t s;
    if (repack_source(o, g, N, &kind, &s)) {
      if (kind == 0) qw[s] = in[o];
      else if (kind == 1) sc[s] = in[o];
      else zp[s] = in[o];
    }
  }
}

int gcd32(int a) {
  int b = 32;
  while (b != 0) {
    const int t = a % b;
    a = b;
    b = t;
  }
  return a;
}

bool geom_of(int64_t K, int64_t N, RepackGeom* g) {
  if (K <= 0 || N <= 0 || K % 32 != 0 || N % 8 != 0 || K > (int64_t(1) << 30) || N > (int64_t(1) << 30)) return false;
  g->nb = static_cast<int32_t>(K / 32);
  const int gs = 32 / gcd32(g->nb);
  g->gsl = __builtin_ctz(gs);
  g->A = g->nb / gcd32(g->nb);
  g->ngroups = static_cast<int32_t>((N + 8 * gs - 1) / (8 * gs));
  g->words = static_cast<int64_t>(g->ngroups) * g->A * ROUND_WORDS;
  return true;
}

bool aligned_to(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool overlaps(const void* a, int64_t abytes, const void* b, int64_t bbytes) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + static_cast<uintptr_t>(bbytes) && b0 < a0 + static_cast<uintptr_t>(abytes);
}

w4_status launch_repack_like(bool restore, const uint8_t* qw, const float* sc, const uint8_t* zp, const void* wr,
                             int64_t K, int64_t N, uint8_t* qw_out, float* sc_out, uint8_t* zp_out, void* wr_out,
                             cudaStream_t st) {
  using namespace w4host;
  RepackGeom g;
  if (!geom_of(K, N, &g))
    return fail(W4_ERR_SHAPE, "streaming layout needs K %% 32 == 0, N %% 8 == 0, 0 < K, N <= 2^30 (K=%lld N=%lld)",
                static_cast<long long>(K), static_cast<long long>(N));
  const DeviceInfo* di = nullptr;
  w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  const int64_t blocks = std::min<int64_t>((g.words + 255) / 256, static_cast<int64_t>(di->sms) * 32);
  if (!restore) {
    w4r_repack_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        reinterpret_cast<const uint32_t*>(qw), reinterpret_cast<const uint32_t*>(sc),
        reinterpret_cast<const uint32_t*>(zp), N, g, static_cast<uint32_t*>(wr_out));
  } else {
    w4r_restore_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const uint32_t*>(wr), N, g, reinterpret_cast<uint32_t*>(qw_out), reinterpret_cast<uint32_t*>(sc_out),
        reinterpret_cast<uint32_t*>(zp_out));
  }
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, restore ? "launch w4r_restore" : "launch w4r_repack");
}

// ---------------------------------------------------------------- GEMV launch

w4_status check_rdesc(const w4r_desc& d, RepackGeom* g) {
  using namespace w4host;
  if (d.M < 0 || d.K < 0 || d.N < 0) return fail(W4_ERR_SHAPE, "negative size");
  if (d.act < W4_ACT_NONE || d.act > W4_ACT_GELU_ERF) return fail(W4_ERR_VALUE, "unknown activation %d", int(d.act));
  if (d.reserved != 0) return fail(W4_ERR_VALUE, "reserved field must be 0");
  if (d.M == 0 || d.N == 0) return W4_OK;
  if (d.N % 8 != 0) return fail(W4_ERR_SHAPE, "streaming layout needs N %% 8 == 0 (N=%lld)", (long long)d.N);
  if (d.K % 32 != 0) return fail(W4_ERR_SHAPE, "K=%lld is not a multiple of 32", (long long)d.K);
  if (d.M != 1) return fail(W4_ERR_SHAPE, "the streaming-layout GEMV takes M = 1 (M=%lld)", (long long)d.M);
  if (d.y == nullptr) return fail(W4_ERR_NULL, "y is NULL");
  if (!aligned_to(d.y, 4)) return fail(W4_ERR_ALIGN, "y must be 4-byte aligned");
  if (d.bias != nullptr && !aligned_to(d.bias, 4)) return fail(W4_ERR_ALIGN, "bias must be 4-byte aligned");
  if (d.residual != nullptr && !aligned_to(d.residual, 4))
    return fail(W4_ERR_ALIGN, "residual must be 4-byte aligned");
  if (d.K == 0) return W4_OK;
  if (d.x == nullptr || d.wr == nullptr) return fail(W4_ERR_NULL, "x and wr must not be NULL");
  if (!aligned_to(d.x, 16)) return fail(W4_ERR_ALIGN, "the streaming-layout GEMV needs x 16-byte aligned");
  if (!aligned_to(d.wr, 16)) return fail(W4_ERR_ALIGN, "the repacked weight must be 16-byte aligned");
  if (d.K > XCAP) return fail(W4_ERR_SHAPE, "the streaming-layout GEMV takes K <= %d (K=%lld)", XCAP, (long long)d.K);
  geom_of(d.K, d.N, g);
  return W4_OK;
}

w4_status check_rdescs(const w4r_desc* descs, int32_t count, int* work) {
  using namespace w4host;
  *work = 0;
  for (int32_t i = 0; i < count; ++i) {
    RepackGeom g;
    const w4_status rc = check_rdesc(descs[i], &g);
    if (rc != W4_OK) {
      char why[256];
      snprintf(why, sizeof(why), "%s", w4_last_error());
      return fail(rc, "descriptor %d: %s", i, why);
    }
    if (descs[i].M != 0 && descs[i].N != 0) ++*work;
  }
  return W4_OK;
}

// x floats that CTA c of G must hold: the sum of K over the matrices its
// range of groups touches.
// cfirst[0 .. G]: CTA c takes body groups [cfirst[c], cfirst[c + 1]), the
// first group whose rounds before it reach c R / G of the launch's R rounds.
void split_by_rounds(const RepackGeom* geo, int count, int G, int32_t* cfirst) {
  int64_t R = 0;
  for (int i = 0; i < count; ++i) R += static_cast<int64_t>(geo[i].ngroups) * geo[i].A;
  int64_t g0 = 0, r0 = 0;  // groups and rounds before matrix i
  int i = 0;
  for (int c = 0; c <= G; ++c) {
    const int64_t t = c * R / G;
    while (i < count && r0 + static_cast<int64_t>(geo[i].ngroups) * geo[i].A < t) {
      r0 += static_cast<int64_t>(geo[i].ngroups) * geo[i].A;
      g0 += geo[i].ngroups;
      ++i;
    }
    cfirst[c] = static_cast<int32_t>(i < count ? g0 + (t - r0 + geo[i].A - 1) / geo[i].A : g0);
  }
}

int64_t max_x_need(const w4r_desc* d, const RepackGeom* geo, int count, const int32_t* cfirst, int G) {
  int64_t worst = 0;
  int64_t g0 = 0;
  int gi = 0;
  for (int c = 0; c < G; ++c) {
    const int64_t lo = cfirst[c], hi = cfirst[c + 1];
    if (hi <= lo) continue;
    while (gi + 1 < count && g0 + geo[gi].ngroups <= lo) g0 += geo[gi++].ngroups;
    int64_t need = 0, gg0 = g0;
    for (int gj = gi; gj < count && gg0 < hi; gg0 += geo[gj++].ngroups) need += d[gj].K;
    worst = std::max(worst, need);
  }
  return worst;
}

// CTAs of a launch of T body groups and TH head groups: each CTA takes an
// equal share of both.
int grid_of(int64_t T, int64_t TH, const w4host::DeviceInfo& di) {
  return static_cast<int>(std::min<int64_t>(std::min(di.sms, GMAX), T + TH));
}

// One launch over the matrices d[0 .. count) and, with hd, the head's TH
// groups (the caller has checked that the step fits one launch).
w4_status launch_rgroup(const w4r_desc* d, const RepackGeom* geo, int count, cudaStream_t st,
                        const w4host::DeviceInfo& di, const RHead* hd = nullptr, int32_t TH = 0) {
  using namespace w4host;
  int64_t T = 0;
  for (int i = 0; i < count; ++i) T += geo[i].ngroups;
  if (hd == nullptr) TH = 0;
  const int G = grid_of(T, TH, di);
  RParams prm;
  std::memset(&prm, 0, sizeof(prm));
  split_by_rounds(geo, count, G, prm.cfirst);
  // every CTA stages the x of each matrix its range touches: split the
  // launch until that fits its shared memory
  if (hd == nullptr && count > 1 && max_x_need(d, geo, count, prm.cfirst, G) > XCAP) {
    const int h = count / 2;
    const w4_status rc = launch_rgroup(d, geo, h, st, di);
    if (rc != W4_OK) return rc;
    return launch_rgroup(d + h, geo + h, count - h, st, di);
  }
  if ((T + TH) * G >= (int64_t(1) << 31))
    return fail(W4_ERR_SHAPE, "too many groups for one launch (%lld)", (long long)(T + TH));
  int g0 = 0;
  for (int i = 0; i < count; ++i) {
    RMat& m = prm.m[i];
    m.wr = static_cast<const uint8_t*>(d[i].wr);
    m.x = d[i].x;
    m.y = d[i].y;
    m.bias = d[i].bias;
    m.res = d[i].residual;
    m.ldr = d[i].ldr;
    m.K = static_cast<int32_t>(d[i].K);
    m.N = static_cast<int32_t>(d[i].N);
    m.g0 = g0;
    m.ngroups = geo[i].ngroups;
    m.act = d[i].act;
    m.gsl = geo[i].gsl;
    g0 += geo[i].ngroups;
  }
  prm.count = count;
  prm.T = static_cast<int32_t>(T);
  prm.TH = TH;
  if (hd != nullptr) prm.hd = *hd;
  prm.err = di.err;
  prm.timeout_ns = wait_timeout_ns();
  const bool step = hd != nullptr;
  static int configured[2][64] = {};
  if (di.dev < 64 && !configured[step][di.dev]) {
    const cudaError_t e =
        step ? cudaFuncSetAttribute(w4r_gemv_m1_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_STEP)
             : cudaFuncSetAttribute(w4r_gemv_m1_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(w4r_gemv)");
    configured[step][di.dev] = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(G));
  cfg.blockDim = dim3(PW * 32);
  cfg.dynamicSmemBytes = static_cast<size_t>(step ? SMEM_STEP : SMEM_BYTES);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = step ? cudaLaunchKernelEx(&cfg, w4r_gemv_m1_kernel<true>, prm)
                             : cudaLaunchKernelEx(&cfg, w4r_gemv_m1_kernel<false>, prm);
  return e == cudaSuccess ? W4_OK : cuda_fail(e, step ? "launch w4r_gemv (decode step)" : "launch w4r_gemv");
}

}  // namespace

extern "C" {

size_t w4_repacked_bytes(int64_t K, int64_t N) {
  RepackGeom g;
  if (!geom_of(K, N, &g)) return 0;
  return static_cast<size_t>(g.words) * 4;
}

w4_status w4_repack(const uint8_t* qw, const float* scales, const uint8_t* zp, int64_t K, int64_t N, void* wr,
                    void* stream) {
  using namespace w4host;
  if (qw == nullptr || scales == nullptr || zp == nullptr || wr == nullptr)
    return fail(W4_ERR_NULL, "qw, scales, zp and wr must not be NULL");
  if (!aligned_to(qw, 16) || !aligned_to(scales, 16) || !aligned_to(zp, 16) || !aligned_to(wr, 16))
    return fail(W4_ERR_ALIGN, "qw, scales, zp and wr must be 16-byte aligned");
  return launch_repack_like(false, qw, scales, zp, nullptr, K, N, nullptr, nullptr, nullptr, wr,
                            static_cast<cudaStream_t>(stream));
}

w4_status w4_repack_restore(const void* wr, int64_t K, int64_t N, uint8_t* qw, float* scales, uint8_t* zp,
                            void* stream) {
  using namespace w4host;
  if (qw == nullptr || scales == nullptr || zp == nullptr || wr == nullptr)
    return fail(W4_ERR_NULL, "qw, scales, zp and wr must not be NULL");
  if (!aligned_to(qw, 16) || !aligned_to(scales, 16) || !aligned_to(zp, 16) || !aligned_to(wr, 16))
    return fail(W4_ERR_ALIGN, "qw, scales, zp and wr must be 16-byte aligned");
  return launch_repack_like(true, nullptr, nullptr, nullptr, wr, K, N, qw, scales, zp, nullptr,
                            static_cast<cudaStream_t>(stream));
}

w4_status w4r_matmul_grouped(const w4r_desc* descs, int32_t count, void* stream) {
  using namespace w4host;
  if (count < 0) return fail(W4_ERR_SHAPE, "negative count");
  if (count == 0) return W4_OK;
  if (descs == nullptr) return fail(W4_ERR_NULL, "descs is NULL");
  static thread_local RepackGeom geo[RCAP];
  static thread_local w4r_desc run[RCAP];
  int work = 0;
  w4_status rc0 = check_rdescs(descs, count, &work);
  if (rc0 != W4_OK) return rc0;
  if (work == 0) return W4_OK;
  const DeviceInfo* di = nullptr;
  w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  int n = 0;
  for (int32_t i = 0; i < count; ++i) {
    const w4r_desc& d = descs[i];
    if (d.M == 0 || d.N == 0) continue;
    if (d.K == 0) {
      w4_desc z = {};
      z.bias = d.bias;
      z.residual = d.residual;
      z.ldr = d.ldr;
      z.act = d.act;
      rc = launch_zero_fill(d.y, d.N, 1, d.N, st, &z);
      if (rc != W4_OK) return rc;
      continue;
    }
    geom_of(d.K, d.N, &geo[n]);
    run[n++] = d;
    if (n == RCAP) {
      rc = launch_rgroup(run, geo, n, st, *di);
      if (rc != W4_OK) return rc;
      n = 0;
    }
  }
  if (n > 0) rc = launch_rgroup(run, geo, n, st, *di);
  return rc;
}

w4_status w4r_matmul(const w4r_desc* d, void* stream) {
  if (d == nullptr) return w4host::fail(W4_ERR_NULL, "descriptor is NULL");
  return w4r_matmul_grouped(d, 1, stream);
}

}  // extern "C"

namespace {

// The step with the head's logits (keys == nullptr) or its greedy token.
w4_status decode_step(const w4r_desc* descs, int32_t count, const float* h, const void* tr, int64_t K, int64_t V,
                      float* logits, unsigned long long* keys, int32_t* token, float* best_logit, void* stream) {
  using namespace w4host;
  if (count < 0) return fail(W4_ERR_SHAPE, "negative count");
  if (count > 0 && descs == nullptr) return fail(W4_ERR_NULL, "descs is NULL");
  int work = 0;
  w4_status rc = count > 0 ? check_rdescs(descs, count, &work) : W4_OK;
  if (rc != W4_OK) return rc;
  rc = check_stream_head(h, tr, K, V);
  if (rc != W4_OK) return rc;
  if (keys == nullptr) {
    if (logits == nullptr) return fail(W4_ERR_NULL, "logits is NULL");
    if (!aligned_to(logits, 4)) return fail(W4_ERR_ALIGN, "logits must be 4-byte aligned");
  } else {
    if (V > 0x7fffffff) return fail(W4_ERR_SHAPE, "V must be below 2^31");
    if (token == nullptr) return fail(W4_ERR_NULL, "token is NULL");
    if (!aligned_to(token, 4) || !aligned_to(best_logit, 4) || !aligned_to(keys, 8))
      return fail(W4_ERR_ALIGN, "token / best 4-byte, keys 8-byte aligned");
  }
  // h is read when the launch starts and the body's outputs are written
  // during it: h must not be one of them
  for (int32_t i = 0; i < count; ++i) {
    const w4r_desc& d = descs[i];
    if (d.M != 0 && d.N != 0 && overlaps(h, K * 4, d.y, d.N * 4))
      return fail(W4_ERR_VALUE, "h overlaps the output of descriptor %d: a step's head reads its input at the start",
                  i);
  }
  const DeviceInfo* di = nullptr;
  rc = current_device(&di);
  if (rc != W4_OK) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the head alone (logits or greedy token), stream-ordered after the body
  auto head = [&]() -> w4_status {
    if (keys == nullptr) return launch_stream_head(h, tr, K, V, logits, st, *di);
    return i8r_head_argmax(h, tr, K, V, token, best_logit, keys, stream);
  };
  static thread_local RepackGeom geo[RCAP];
  static thread_local w4r_desc run[RCAP];
  int n = 0;
  bool one_launch = work <= RCAP && K <= HKS;
  for (int32_t i = 0; i < count && one_launch; ++i) {
    const w4r_desc& d = descs[i];
    if (d.M == 0 || d.N == 0 || d.K == 0) continue;
    geom_of(d.K, d.N, &geo[n]);
    run[n++] = d;
  }
  StreamHeadGeom hg;
  stream_head_geom(K, V, &hg);
  if (one_launch && n > 0) {
    int64_t T = 0;
    for (int i = 0; i < n; ++i) T += geo[i].ngroups;
    const int G = grid_of(T, hg.ngroups, *di);
    static thread_local int32_t cfirst[GMAX + 1];
    split_by_rounds(geo, n, G, cfirst);
    one_launch = max_x_need(run, geo, n, cfirst, G) <= XCAP_STEP;
  }
  if (!one_launch) {
    // more matrices, x or h than one launch holds: the body's launches, then the head's
    rc = w4r_matmul_grouped(descs, count, stream);
    if (rc != W4_OK) return rc;
    return head();
  }
  for (int32_t i = 0; i < count; ++i) {  // K = 0: y is the epilogue of 0
    const w4r_desc& d = descs[i];
    if (d.M == 0 || d.N == 0 || d.K != 0) continue;
    w4_desc z = {};
    z.bias = d.bias;
    z.residual = d.residual;
    z.ldr = d.ldr;
    z.act = d.act;
    rc = launch_zero_fill(d.y, d.N, 1, d.N, st, &z);
    if (rc != W4_OK) return rc;
  }
  if (n == 0) return head();
  RHead hd;
  hd.tr = static_cast<const uint8_t*>(tr);
  hd.h = h;
  hd.logits = keys == nullptr ? logits : nullptr;
  hd.keys = keys;
  hd.group_bytes = hg.group_bytes;
  hd.K = static_cast<int32_t>(K);
  hd.V = static_cast<int32_t>(V);
  hd.gsl = hg.gsl;
  hd.A = hg.A;
  if (keys != nullptr) {
    const cudaError_t e = cudaMemsetAsync(keys, 0, 8, st);
    if (e != cudaSuccess) return cuda_fail(e, "clear argmax key");
  }
  rc = launch_rgroup(run, geo, n, st, *di, &hd, hg.ngroups);
  if (rc != W4_OK || keys == nullptr) return rc;
  return launch_argmax_finish(keys, 1, token, best_logit, st);
}

}  // namespace

extern "C" {

w4_status w4r_decode_step(const w4r_desc* descs, int32_t count, const float* h, const void* tr, int64_t K, int64_t V,
                          float* logits, void* stream) {
  return decode_step(descs, count, h, tr, K, V, logits, nullptr, nullptr, nullptr, stream);
}

w4_status w4r_decode_step_argmax(const w4r_desc* descs, int32_t count, const float* h, const void* tr, int64_t K,
                                 int64_t V, int32_t* token, float* best_logit, void* keys, void* stream) {
  if (keys == nullptr) return w4host::fail(W4_ERR_NULL, "keys is NULL");
  return decode_step(descs, count, h, tr, K, V, nullptr, static_cast<unsigned long long*>(keys), token, best_logit,
                     stream);
}

}  // extern "C"
