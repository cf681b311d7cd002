// Device-side helpers shared by the kernels of libw4b200: shared-memory
// barriers, bounded waits, bulk / tensor copies, the nibble decoder.
//
// Every wait on a barrier is bounded by %globaltimer: when the limit runs
// out the waiting thread records W4_ERR_TIMEOUT in the device error word and
// reports failure to its caller, which stops issuing work and returns. No
// kernel here traps, asserts or spins without limit.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "w4.h"

namespace w4dev {

// Device error word: {status, kernel id, block index, detail}. Only the first
// error is kept (compare-and-swap on the status slot).
struct ErrorWord {
  int32_t status;
  int32_t kernel;
  int32_t block;
  int32_t detail;
};

enum KernelId : int32_t { K_GEMV = 1, K_GENERIC = 2, K_HEAD = 3, K_HEAD_GENERIC = 4, K_TC = 5, K_EMBED = 6, K_GEMVR = 7, K_HEADR = 8, K_DEBUG = 9, K_TILE = 10, K_HEADT = 11, K_GEMVI = 12 };

__device__ __forceinline__ void record_error(ErrorWord* e, int32_t status, int32_t kernel, int32_t detail) {
  if (atomicCAS(&e->status, 0, status) == 0) {
    e->kernel = kernel;
    e->block = static_cast<int32_t>(blockIdx.x);
    e->detail = detail;
    __threadfence();
  }
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: a thread whose phase is not complete is
// suspended (it issues nothing) until the phase completes or about hint_ns
// pass, instead of spinning and taking issue slots from working warps.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Wait until the phase with parity `parity` of `bar` has completed. Returns
// false (after recording the error) when `timeout_ns` passes first, or when
// *abort is set by another thread of the CTA. Each try suspends the thread
// for up to 0.2 ms, so a waiting warp costs almost no issue slots and the
// timer and the abort flag are looked at after every try.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t timeout_ns,
                                                  volatile int* abort, ErrorWord* err, int32_t kernel,
                                                  int32_t detail) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
  while (true) {
    if (mbar_try_wait_sleep(a, parity, 200000u)) return true;
    if (abort != nullptr && *abort) return false;
    if (globaltimer_ns() - t0 > timeout_ns) {
      if (abort != nullptr) *abort = 1;
      record_error(err, W4_ERR_TIMEOUT, kernel, detail);
      return false;
    }
  }
}

// ---------------------------------------------------------------- bulk copies (no multicast)

// Untiled bulk copy global -> this CTA's shared memory; completes `bytes`
// transaction bytes on `bar`. Both addresses 16-B aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 16-byte asynchronous copy global -> shared (L2 only): reads src_bytes
// (0..16) bytes and zero-fills the rest of the 16. Both addresses 16-B aligned.
__device__ __forceinline__ void cp_async_16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Wait until at most N of this thread's committed cp.async groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Arrive on `bar` once every cp.async this thread has issued so far has
// completed (the arrival is counted in the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 2-D tiled tensor copy global -> this CTA's shared memory (box from map).
// c0 is the innermost coordinate in elements (bytes for uint8 maps) and must
// be a multiple of 16 bytes; c1 any row index (rows past the end read zeros).
__device__ __forceinline__ void tma_g2s_2d(void* dst, const CUtensorMap* map, int32_t c0, int32_t c1,
                                           uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------- named barriers

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------- nibble decode
//
// A 32-bit word holds 8 nibbles n0..n7 (n_i in bits 4i..4i+3). For i in 0..3
// the float with bits 0x4B000000 | (word & (0xF << 4i)) equals 2^23 + n_i*16^i
// exactly (the nibble lands inside the 23-bit mantissa of 2^23); for i in
// 4..7 the same holds on word >> 16 with 16^(i-4). Subtracting the float
// built the same way from the zero-point word gives (q - zp) * 16^(i mod 4)
// exactly: both operands are integers in [2^23, 2^24). The power of two is
// folded into the scale, s * 16^-(i mod 4), which is exact too.

// One LOP3: (word & mask) | magic, with the magic exponent word passed in a
// register so that the instruction needs only one immediate (the mask).
__device__ __forceinline__ float magic_nib_r(uint32_t word, uint32_t magic, int slot /*0..3, compile time*/) {
  uint32_t r;
  switch (slot) {
    case 0: asm("lop3.b32 %0, %1, 0xF, %2, 0xEA;" : "=r"(r) : "r"(word), "r"(magic)); break;
    case 1: asm("lop3.b32 %0, %1, 0xF0, %2, 0xEA;" : "=r"(r) : "r"(word), "r"(magic)); break;
    case 2: asm("lop3.b32 %0, %1, 0xF00, %2, 0xEA;" : "=r"(r) : "r"(word), "r"(magic)); break;
    default: asm("lop3.b32 %0, %1, 0xF000, %2, 0xEA;" : "=r"(r) : "r"(word), "r"(magic)); break;
  }
  return __uint_as_float(r);
}

__device__ __forceinline__ float magic_nib(uint32_t word, int slot /*0..3*/) {
  return __uint_as_float(0x4B000000u | (word & (0xFu << (4 * slot))));
}

__device__ __forceinline__ float inv_slot_scale(int slot) {
  return slot == 0 ? 1.0f : (slot == 1 ? 0.0625f : (slot == 2 ? 0.00390625f : 0.000244140625f));
}

// ---------------------------------------------------------------- fused epilogue

// y = act(v + bias[n]) + residual[m * ldr + n] (the MatMul + Add that the
// export's gemm_to_matmul step leaves behind each GPT-2 weight, with the
// activation or residual add that follows it in the model). Zero pointers /
// W4_ACT_NONE switch the parts off. GELU forms as in include/w4.h; tanhf and
// erff are CUDA's single-precision functions.
struct Epi {
  const float* bias;
  const float* res;
  int64_t ldr;
  int32_t act;
  int32_t pad;
};

__device__ __forceinline__ float gelu_tanh_f(float v) {
  const float c0 = 0.7978845608028654f;  // sqrt(2 / pi)
  const float c1 = 0.044715f;
  return 0.5f * v * (1.f + tanhf(c0 * (v + c1 * v * v * v)));
}

__device__ __forceinline__ float gelu_erf_f(float v) { return 0.5f * v * (1.f + erff(v * 0.7071067811865476f)); }

__device__ __forceinline__ bool epi_active(const Epi& e) {
  return e.bias != nullptr || e.res != nullptr || e.act != W4_ACT_NONE;
}

__device__ __forceinline__ float epi_apply(float v, const Epi& e, int64_t m, int64_t n) {
  if (e.bias != nullptr) v += e.bias[n];
  if (e.act == W4_ACT_GELU_TANH) v = gelu_tanh_f(v);
  else if (e.act == W4_ACT_GELU_ERF) v = gelu_erf_f(v);
  if (e.res != nullptr) v += e.res[m * e.ldr + n];
  return v;
}

// ---- the int8 head's streaming-layout atom (shared by the head kernel and
// the fused decode step)

// Byte j of a biased word in the mantissa of 2^23: [byte j, 0, 0, 0x4B].
template <int J>
__device__ __forceinline__ float byte_float(uint32_t w, uint32_t magic) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(w), "r"(magic), "n"(0x7540 | J));
  return __uint_as_float(r);
}

// One 16-row x 8-column atom of this lane into P[0..7] (two running sums per
// column, rows 2c and 2c+1). hb: h of the atom's block, row pair c at
// hb + c * hq floats.
__device__ __forceinline__ void atom_i8(const uint8_t* st, int lane, const float* hb, int hq, uint32_t magic,
                                        float2 nbias, float2 (&P)[8]) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 wv = *reinterpret_cast<const uint4*>(st + c * 512 + lane * 16);
    const float2 hv = *reinterpret_cast<const float2*>(hb + c * hq);
    // wv.x: row 2c cols 0-3, wv.y: row 2c cols 4-7, wv.z / wv.w: row 2c+1
    P[0] = __ffma2_rn(hv, __fadd2_rn(make_float2(byte_float<0>(wv.x, magic), byte_float<0>(wv.z, magic)), nbias), P[0]);
    P[1] = __ffma2_rn(hv, __fadd2_rn(make_float2(byte_float<1>(wv.x, magic), byte_float<1>(wv.z, magic)), nbias), P[1]);
    P[2] = __ffma2_rn(hv, __fadd2_rn(make_float2(byte_float<2>(wv.x, magic), byte_float<2>(wv.z, magic)), nbias), P[2]);
    P[3] = __ffma2_rn(hv, __fadd2_rn(make_float2(byte_float<3>(wv.x, magic), byte_float<3>(wv.z, magic)), nbias), P[3]);
    P[4] = __ffma2_rn(hv, __fadd2_rn(make_float2(byte_float<0>(wv.y, magic), byte_float<0>(wv.w, magic)), nbias), P[4]);
    P[5] = __ffma2_rn(hv, __fadd2_rn(make_float2(byte_float<1>(wv.y, magic), byte_float<1>(wv.w, magic)), nbias), P[5]);
    P[6] = __ffma2_rn(hv, __fadd2_rn(make_float2(byte_float<2>(wv.y, magic), byte_float<2>(wv.w, magic)), nbias), P[6]);
    P[7] = __ffma2_rn(hv, __fadd2_rn(make_float2(byte_float<3>(wv.y, magic), byte_float<3>(wv.w, magic)), nbias), P[7]);
  }
}

// Order-preserving 64-bit key of (logit, token): logit bits made monotonic
// (-0 taken as +0) above the complement of the token id, so the maximum key
// is the largest logit and, among equal logits, the lowest id.
__device__ __forceinline__ unsigned long long head_key(float logit, uint32_t token) {
  uint32_t b = __float_as_uint(logit);
  if (b == 0x80000000u) b = 0u;
  const uint32_t o = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return (static_cast<unsigned long long>(o) << 32) | static_cast<unsigned long long>(0xFFFFFFFFu - token);
}

}  // namespace w4dev
