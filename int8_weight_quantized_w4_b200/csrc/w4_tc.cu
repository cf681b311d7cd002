// w4_tc: y = x . W for large M (prefill) on the 5th-generation tensor cores,
// W in the 4-bit blocked format of "ONNX export, quantization and the browser
// runtime", section "Quantization (train/quantize.py)", step 2 (dq4): blocks
// of 32 along K, fp32 scale and uint4 zero point per (block, column),
// w = (q - zp) * scale. The page's output is fp32 compute, so the products are
// formed as 3xTF32: x = x_hi + x_lo, w = w_hi + w_lo (hi truncated to tf32,
// lo the exact fp32 remainder, which the tensor core reads to tf32
// precision), and D += x_hi w_hi + x_hi w_lo + x_lo w_hi in an fp32
// accumulator. The dropped x_lo w_lo term and the tf32 reading of the lo
// parts are below 2^-19 |x w| per product.
//
// Design (sm_100a):
//  * One CTA per 128 x 256 tile of y (all weights of a grouped launch share
//    one grid), eight warps. The accumulator (128 lanes x 256 fp32 columns)
//    lives in tensor memory, allocated by warp 0.
//  * Per 32-row K-block (one scale / zero-point row): the threads load x and
//    the packed weight slice with plain loads (issued two blocks ahead of
//    the one being converted), dequantise exactly as the oracle does
//    ((q - zp) * s, one fp32 rounding, through the exponent trick of
//    w4_device.cuh), split both into tf32 hi (low 13 mantissa bits cleared)
//    and lo (the exact remainder), and store them in shared memory in the
//    canonical K-major layout
//    without swizzle (core matrices of 8 rows x 16 bytes; the two 16-byte
//    halves of an 8-wide K step are LBO = 128 bytes apart, groups of 8 rows
//    SBO = 256 bytes apart). Two stages: the next block is converted while
//    the tensor core works on the current one.
//  * One thread issues the 12 MMAs of a block (4 K steps x 3 products,
//    M = 128, N = 256, K = 8, kind::tf32) and commits them to the stage's
//    mbarrier; the stage is rewritten only after that commit arrives.
//  * Column 8 l + c of a tile (l = 0..31, c = 0..7) is stored as row 32 c + l
//    of the B operand, so that the 32 lanes of a warp, which convert the
//    8-column groups l = 0..31, store contiguous runs (no bank conflicts);
//    accumulator column j therefore holds y column 8 (j mod 32) + j / 32.
//  * Epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (its rows) and
//    columns 128 (w / 4) .. +127, 32 at a time, and writes y.
// Every wait is bounded; on timeout the kernel records an error and skips
// the remaining work.
#include <cuda_runtime.h>

#include <algorithm>

#include "w4_device.cuh"
#include "w4_internal.h"

namespace {

using namespace w4dev;

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 32;
constexpr int NT = 256;                                 // 8 warps; warp w reads TMEM lanes 32 (w % 4) ..
constexpr int A_PART = BM * BK * 4;                     // 16 KB: x hi or x lo
constexpr int B_PART = BN * BK * 4;                     // 32 KB: w hi or w lo
constexpr int STAGE_BYTES = 2 * A_PART + 2 * B_PART;    // 96 KB
constexpr int NSTAGE = 2;
constexpr int SMEM_BYTES = NSTAGE * STAGE_BYTES + 64;
constexpr uint32_t TMEM_COLS = BN;                      // fp32 accumulator columns

struct TcMat {
  const float* x;
  const uint8_t* qw;
  const float* scales;
  const uint8_t* zp;
  float* y;
  int64_t ldx, ldy;
  int32_t M, K, N, nb;
  int32_t tiles_m, tile_off;  // tiles of this weight: tiles_m x ceil(N / BN), from tile_off on
  Epi epi;                    // fused epilogue of the store
};

struct TcParams {
  TcMat mat[W4_GROUP_MAX];
  int32_t count;
  int32_t total_tiles;
  ErrorWord* err;
  uint64_t timeout_ns;
};

// Byte offset of element (r, k) of an R-row x 32 operand slice in the
// canonical K-major no-swizzle layout, one slab of R x 8 per K step.
__device__ __forceinline__ uint32_t kmaj_off(int r, int k, int R) {
  return static_cast<uint32_t>((k >> 3) * (R * 32) + (r >> 3) * 256 + ((k >> 2) & 1) * 128 + (r & 7) * 16 + (k & 3) * 4);
}

// Shared-memory matrix descriptor (sm_100 format): start address, leading
// byte offset (between the two 16-byte K halves of a core-matrix pair),
// stride byte offset (between groups of 8 rows), version 1, no swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((128u >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((256u >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// Instruction descriptor: fp32 accumulator, tf32 A and B, both K-major,
// N = BN, M = BM.
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                            (static_cast<uint32_t>(BM >> 4) << 24);

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t da, uint64_t db, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(da), "l"(db), "r"(kIdesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// High part of the 3xTF32 split: v with its low 13 mantissa bits cleared (a
// tf32 value); v - hi is then exact in fp32.
__device__ __forceinline__ float tf32_hi(float v) { return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__global__ void __launch_bounds__(NT, 1) w4_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* mma_done = reinterpret_cast<uint64_t*>(smem + NSTAGE * STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + NSTAGE);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // which weight and tile
  int g = 0;
  while (g + 1 < p.count && p.mat[g + 1].tile_off <= static_cast<int>(blockIdx.x)) ++g;
  const TcMat& m = p.mat[g];
  const int local = static_cast<int>(blockIdx.x) - m.tile_off;
  const int m0 = (local % m.tiles_m) * BM;
  const int n0 = (local / m.tiles_m) * BN;
  const int64_t hrow = m.N / 2;  // bytes per row of packed nibbles

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) mbar_init(&mma_done[s], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  bool ok = true;
  int issued = 0;  // K-blocks whose MMAs were issued
  // One K-block's raw inputs for this thread: 4 x (16 bytes of x) and one
  // 8-column x 4-row piece of the weight with its scales and zero points.
  // The loads of the block after the next are issued while the current one
  // is converted (two blocks in flight).
  struct Raw {
    float4 xv[(BM * BK / 4) / NT];
    uint32_t w[4];
    float4 s0, s1;
    uint32_t z;
  };
  const int cg = tid & 31;  // weight: group of 8 columns
  const int kq = tid >> 5;  // weight: group of 4 rows of the K-block
  const int nw = n0 + 8 * cg;
  auto load = [&](int b, Raw& R) {
    const int k0 = b * BK;
#pragma unroll
    for (int i = 0; i < (BM * BK / 4) / NT; ++i) {
      const int r = tid & (BM - 1), q = (tid >> 7) + 2 * i;
      const int row = m0 + r;
      R.xv[i] = row < m.M ? __ldg(reinterpret_cast<const float4*>(m.x + static_cast<int64_t>(row) * m.ldx + k0 + 4 * q))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (nw < m.N) {
#pragma unroll
      for (int t = 0; t < 4; ++t)
        R.w[t] = __ldg(reinterpret_cast<const uint32_t*>(m.qw + static_cast<int64_t>(k0 + 4 * kq + t) * hrow + nw / 2));
      R.s0 = __ldg(reinterpret_cast<const float4*>(m.scales + static_cast<int64_t>(b) * m.N + nw));
      R.s1 = __ldg(reinterpret_cast<const float4*>(m.scales + static_cast<int64_t>(b) * m.N + nw + 4));
      R.z = __ldg(reinterpret_cast<const uint32_t*>(m.zp + (static_cast<int64_t>(b) * m.N + nw) / 2));
    } else {
#pragma unroll
      for (int t = 0; t < 4; ++t) R.w[t] = 0u;
      R.s0 = R.s1 = make_float4(0.f, 0.f, 0.f, 0.f);
      R.z = 0u;
    }
  };
  Raw cur, nxt, nxt2;
  if (m.nb > 0) load(0, cur);
  if (m.nb > 1) load(1, nxt);
  for (int b = 0; b < m.nb; ++b) {
    const int s = b & 1;
    if (b + 2 < m.nb) load(b + 2, nxt2);
    // The stage is free once the MMAs that read it two blocks ago are done.
    // A thread whose bounded wait gives up writes nothing; the barrier below
    // then takes the whole CTA out of the loop together.
    if (b >= NSTAGE && ok)
      ok = mbar_wait_bounded(&mma_done[s], ((b - NSTAGE) >> 1) & 1, p.timeout_ns, abort_flag, p.err, K_TC, 1);
    uint8_t* st = smem + s * STAGE_BYTES;
    uint8_t* a_hi = st;
    uint8_t* a_lo = st + A_PART;
    uint8_t* b_hi = st + 2 * A_PART;
    uint8_t* b_lo = st + 2 * A_PART + B_PART;
    // x: 128 rows x 32, 16 bytes per thread and pass; the 32 lanes of a warp
    // take 32 consecutive rows, so each store is 4 contiguous core-matrix rows
    // groups (conflict-free)
    if (ok) {
#pragma unroll
    for (int i = 0; i < (BM * BK / 4) / NT; ++i) {
      const int r = tid & (BM - 1), q = (tid >> 7) + 2 * i;
      const float4 v = cur.xv[i];
      const float4 h = make_float4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
      const float4 l = make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
      const uint32_t off = kmaj_off(r, 4 * q, BM);
      *reinterpret_cast<float4*>(a_hi + off) = h;
      *reinterpret_cast<float4*>(a_lo + off) = l;
    }
    // weight: w = (q - zp) * s exactly as the oracle rounds it. Nibble c of a
    // 32-bit word sits at slot c % 4 of its half-word: the float with bits
    // 0x4B000000 | (half & (0xF << 4 slot)) is 2^23 + q 16^slot exactly, the
    // difference with the zero point's is (q - zp) 16^slot exactly, and the
    // scale times 16^-slot (exact) makes the product the oracle's w.
    {
      const float sv[8] = {cur.s0.x, cur.s0.y, cur.s0.z, cur.s0.w, cur.s1.x, cur.s1.y, cur.s1.z, cur.s1.w};
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t zh = c < 4 ? cur.z : cur.z >> 16;
        const float zf = magic_nib(zh, c & 3);
        const float sc = sv[c] * inv_slot_scale(c & 3);
        float hv[4], lv[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const uint32_t wh = c < 4 ? cur.w[t] : cur.w[t] >> 16;
          const float wv = (magic_nib(wh, c & 3) - zf) * sc;
          hv[t] = tf32_hi(wv);
          lv[t] = wv - hv[t];
        }
        // column 8 cg + c of the tile is row 32 c + cg of B: a warp's 32
        // lanes (cg = 0..31) then store 4 contiguous 128-byte runs
        const uint32_t off = kmaj_off(32 * c + cg, 4 * kq, BN);
        *reinterpret_cast<float4*>(b_hi + off) = make_float4(hv[0], hv[1], hv[2], hv[3]);
        *reinterpret_cast<float4*>(b_lo + off) = make_float4(lv[0], lv[1], lv[2], lv[3]);
      }
    }
    }  // ok
    fence_async_smem();  // the stores above are read by the tensor core
    tc_fence_before();
    const bool any_failed = __syncthreads_or(!ok) != 0;  // one decision for the whole CTA
    tc_fence_after();
    if (any_failed) {
      ok = false;
      break;
    }
    if (tid == 0) {
      const uint32_t ah = smem_u32(a_hi), al = smem_u32(a_lo), bh = smem_u32(b_hi), bl = smem_u32(b_lo);
#pragma unroll
      for (int ks = 0; ks < BK / 8; ++ks) {
        const uint32_t oa = ks * BM * 32, ob = ks * BN * 32;
        // small terms first, then the main product
        tc_mma(tmem, smem_desc(al + oa), smem_desc(bh + ob), b > 0 || ks > 0);
        tc_mma(tmem, smem_desc(ah + oa), smem_desc(bl + ob), true);
        tc_mma(tmem, smem_desc(ah + oa), smem_desc(bh + ob), true);
      }
      tc_commit(&mma_done[s]);
    }
    issued = b + 1;
    cur = nxt;
    nxt = nxt2;
  }

  // all MMAs done: the last commit covers every earlier one
  if (issued > 0) {
    const int b = issued - 1;
    const bool done = mbar_wait_bounded(&mma_done[b & 1], (b >> 1) & 1, p.timeout_ns, abort_flag, p.err, K_TC, 2);
    ok = ok && done;
  }
  // the epilogue's tensor-memory loads are warp-collective: every thread
  // takes the same decision
  ok = __syncthreads_and(ok) != 0;
  tc_fence_after();
  if (ok && issued == m.nb) {
    const int quad = warp & 3;  // TMEM lanes 32 quad .. 32 quad + 31 = rows of the tile
    const int half = warp >> 2; // columns 128 half .. 128 half + 127
    const int row = m0 + 32 * quad + lane;
#pragma unroll 1
    for (int ch = 4 * half; ch < 4 * half + 4; ++ch) {
      uint32_t v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * quad) << 16) + 32 * ch, v);
      // accumulator column 32 ch + i holds y column 8 i + ch of the tile
      if (row < m.M) {
        float* yr = m.y + static_cast<int64_t>(row) * m.ldy + n0 + ch;
        const int ncol = m.N - n0;
        if (epi_active(m.epi)) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (8 * i + ch < ncol) yr[8 * i] = epi_apply(__uint_as_float(v[i]), m.epi, row, n0 + ch + 8 * i);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (8 * i + ch < ncol) yr[8 * i] = __uint_as_float(v[i]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
}

}  // namespace

namespace w4host {

bool tc_eligible(const w4_desc& d, const char** why) {
  if (d.N % 32 != 0) {
    *why = "the tensor-core path needs N % 32 == 0";
    return false;
  }
  if ((reinterpret_cast<uintptr_t>(d.x) & 15) != 0 || (d.ldx % 4) != 0) {
    *why = "the tensor-core path needs x 16-byte aligned and ldx % 4 == 0";
    return false;
  }
  if (d.M > (int64_t(1) << 30) || d.K > (int64_t(1) << 30) || d.N > (int64_t(1) << 30)) {
    *why = "the tensor-core path needs M, K and N below 2^30";
    return false;
  }
  return true;
}

w4_status launch_tc(const w4_desc* d, int count, cudaStream_t st, const DeviceInfo& di) {
  if (count > W4_GROUP_MAX) return fail(W4_ERR_SHAPE, "at most %d matrices per tensor-core launch", W4_GROUP_MAX);
  static thread_local TcParams prm;
  std::memset(&prm, 0, sizeof(prm));
  int g = 0;
  int64_t tiles = 0;
  for (int i = 0; i < count; ++i) {
    const w4_desc& s = d[i];
    if (s.M == 0 || s.N == 0 || s.K == 0) continue;
    TcMat& m = prm.mat[g];
    m.x = s.x;
    m.qw = s.qw;
    m.scales = s.scales;
    m.zp = s.zp;
    m.y = s.y;
    m.ldx = s.ldx;
    m.ldy = s.ldy;
    m.epi = Epi{s.bias, s.residual, s.ldr, s.act, 0};
    m.M = static_cast<int32_t>(s.M);
    m.K = static_cast<int32_t>(s.K);
    m.N = static_cast<int32_t>(s.N);
    m.nb = static_cast<int32_t>(s.K / BK);
    m.tiles_m = static_cast<int32_t>((s.M + BM - 1) / BM);
    m.tile_off = static_cast<int32_t>(tiles);
    tiles += static_cast<int64_t>(m.tiles_m) * ((s.N + BN - 1) / BN);
    ++g;
  }
  if (g == 0) return W4_OK;
  if (tiles > 0x7fffffff) return fail(W4_ERR_SHAPE, "too many tiles for one tensor-core launch");
  prm.count = g;
  prm.total_tiles = static_cast<int32_t>(tiles);
  prm.err = di.err;
  prm.timeout_ns = wait_timeout_ns();
  static int configured[64] = {};
  if (di.dev < 64 && !configured[di.dev]) {
    const cudaError_t e = cudaFuncSetAttribute(w4_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(w4_tc)");
    configured[di.dev] = 1;
  }
  w4_tc_kernel<<<static_cast<unsigned>(tiles), NT, SMEM_BYTES, st>>>(prm);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch w4_tc");
}

}  // namespace w4host
