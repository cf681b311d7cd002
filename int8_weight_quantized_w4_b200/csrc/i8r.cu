// i8r: the streaming layout of the int8 tied LM head, and the M = 1 head
// GEMV (logits, or the greedy token) that reads it.
//
// The head is the one of "ONNX export, quantization and the browser
// runtime", section "Quantization (train/quantize.py)", steps 3
// (embedding_int8: int8 [K, V] table, one fp32 scale per token column) and 4
// (last_token_logits: only the last position's row h is multiplied):
// logits[v] = s_v * sum_k h_k T[k, v].
//
// Layout (K % 16 == 0; nb = K / 16 blocks of 16 rows):
//   gs = 32 / gcd(nb, 32) strips of 8 token columns form a group (8 gs
//   columns, all K rows); A = gs * nb / 32 rounds of 4096 bytes make a group,
//   followed by the group's 8 gs scales (fp32). In round r of group G, lane l
//   (0..31) owns strip s = l % gs (columns c0 = 8 (G gs + s) .. c0 + 7) and
//   block b = l / gs + r * (32 / gs): 16 rows x 8 columns, 128 bytes, at
//   c * 512 + l * 16 + w * 4 for row pair c (rows 16 b + 2c, +1) and word w:
//   w = 2 e + h holds columns c0 + 4h .. c0 + 4h + 3 of row 16 b + 2c + e,
//   one byte each, stored as (q XOR 0x80) (the int8 code biased to
//   unsigned). Columns at or past V hold code 0 and scale 0 and are never
//   written. The bytes are the page's bytes, reordered and biased; nothing is
//   rounded, so restoring gives the page's table and scales back exactly.
//
// GEMV design (sm_100a, M = 1), the body's (w4r.cu) with the int8 decode:
//  * One persistent CTA per SM takes an equal share of the groups; each of
//    its 12 warps streams its own groups through a ring of 3 stages (one bulk
//    copy per round, the group's scales riding on its last round).
//  * Decode: one PRMT places a biased byte in the mantissa of 2^23, so the
//    float is 2^23 + 128 + q exactly; rows 2c and 2c+1 are taken together so
//    that one FADD2 removes 2^23 + 128 from both (exact) and one FFMA2
//    accumulates with (h_2c, h_2c+1). The scale is applied once per column at
//    the end: s_v * sum_k h_k q_kv.
//  * h is staged in shared memory as [row pair c][block b][2 floats].
//  * With a key buffer instead of logits, each column's logit is folded into
//    a 64-bit key (order-preserving logit bits above the complement of the
//    token id) and one atomicMax per warp keeps the maximum: the greedy
//    token, ties to the lowest id, without writing the logits.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "w4_device.cuh"
#include "w4_internal.h"

namespace {

using namespace w4dev;

constexpr int HROUND = w4host::kStreamHeadRound;  // table bytes of a round
constexpr int HSTAGE = HROUND + 1024;   // a round plus up to 32 * 8 scales
constexpr int HW = 12;                  // warps per CTA
constexpr int HST = 3;                  // stages per warp
constexpr int HKCAP = w4host::kStreamHeadKCap;    // rows of h a CTA can hold
constexpr int HSTAGE_SMEM = HW * HST * HSTAGE;
constexpr int HSMEM_BYTES = HSTAGE_SMEM + HKCAP * 4 + HW * HST * 8 + HW * 4;

struct HParams {
  const uint8_t* tr;
  const float* h;
  float* logits;               // or nullptr
  unsigned long long* keys;    // or nullptr: greedy decoding
  int32_t K, V, ngroups, gsl;
  int64_t group_bytes;
  ErrorWord* err;
  uint64_t timeout_ns;
};

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__global__ void __launch_bounds__(HW * 32, 1) i8r_head_kernel(const __grid_constant__ HParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int T = p.ngroups;
  const int lo = static_cast<int>(static_cast<int64_t>(blockIdx.x) * T / G);
  const int hi = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * T / G);
  const int ngw = hi - lo > warp ? (hi - lo - warp + HW - 1) / HW : 0;
  const int nb = p.K >> 4;
  const int gsl = p.gsl;
  const int gs = 1 << gsl;
  const int A = (nb << gsl) >> 5;
  const int sc_bytes = 32 * gs;

  uint8_t* stg = smem + warp * (HST * HSTAGE);
  float* hs = reinterpret_cast<float*>(smem + HSTAGE_SMEM);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + HSTAGE_SMEM + HKCAP * 4) + warp * HST;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + HSTAGE_SMEM + HKCAP * 4 + HW * HST * 8) + warp;

  // the warp's rounds in order: group lo + warp + HW t, rounds 0 .. A-1 of it
  int it = 0, ir = 0;  // issue cursor (group ordinal, round)
  int issued = 0;
  auto issue = [&](int stage) {
    const int gg = lo + warp + HW * it;
    const uint8_t* src = p.tr + static_cast<int64_t>(gg) * p.group_bytes + static_cast<int64_t>(ir) * HROUND;
    const uint32_t bytes = ir == A - 1 ? HROUND + sc_bytes : HROUND;  // the scales ride on the last round
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar[stage], bytes);
      bulk_g2s(stg + stage * HSTAGE, src, bytes, &bar[stage]);
    }
    ++issued;
    if (++ir == A) {
      ir = 0;
      ++it;
    }
  };

  if (threadIdx.x == 0) asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.h), "r"(p.K * 4) : "memory");
  if (ngw > 0) {
    if (lane == 0) {
      for (int s = 0; s < HST; ++s) mbar_init(&bar[s], 1);
      *abort_flag = 0;
      fence_mbar_init();
    }
    __syncwarp();
    issue(0);  // the table does not depend on the previous launch
  }
  pdl_launch_dependents();
  pdl_wait();  // h may be the previous launch's output, the outputs its inputs

  // h into shared memory as [row pair c][block b][2]
  for (int i = threadIdx.x; i < (p.K >> 2); i += HW * 32) {
    const int b = i >> 2, q = i & 3;  // floats 16 b + 4 q .. +3: row pairs 2q, 2q+1
    const float4 v = __ldg(reinterpret_cast<const float4*>(p.h) + i);
    *reinterpret_cast<float2*>(hs + ((2 * q) * nb + b) * 2) = make_float2(v.x, v.y);
    *reinterpret_cast<float2*>(hs + ((2 * q + 1) * nb + b) * 2) = make_float2(v.z, v.w);
  }
  __syncthreads();
  if (ngw == 0) return;
  for (int s = 1; s < HST && it < ngw; ++s) issue(s);

  uint32_t magic;
  asm("mov.b32 %0, 0x4B000000;" : "=r"(magic));
  const float2 nbias = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
  const int phase = lane >> gsl;
  const int pstride = 32 >> gsl;
  const float* hw = hs + phase * 2;
  const int hq = nb * 2;

  bool ok = true;
  int s = 0;
  uint32_t par = 0;
#pragma unroll 1
  for (int t = 0; t < ngw && ok; ++t) {
    const int gg = lo + warp + HW * t;
    float2 P[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) P[i] = make_float2(0.f, 0.f);
    float sv[8];
#pragma unroll 1
    for (int r = 0; r < A; ++r) {
      ok = mbar_wait_bounded(&bar[s], par, p.timeout_ns, abort_flag, p.err, K_HEADR, 1);
      if (__any_sync(0xffffffffu, !ok)) {
        ok = false;
        break;
      }
      const uint8_t* st = stg + s * HSTAGE;
      atom_i8(st, lane, hw + r * pstride * 2, hq, magic, nbias, P);
      if (r == A - 1) {
        const float4* sp = reinterpret_cast<const float4*>(st + HROUND + (lane & (gs - 1)) * 32);
        const float4 s0 = sp[0], s1 = sp[1];
        sv[0] = s0.x; sv[1] = s0.y; sv[2] = s0.z; sv[3] = s0.w;
        sv[4] = s1.x; sv[5] = s1.y; sv[6] = s1.z; sv[7] = s1.w;
      }
      __syncwarp();
      if (it < ngw) {
        if (lane == 0) fence_proxy_async_smem();
        issue(s);
      }
      if (++s == HST) {
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
    const int col = (((gg << gsl) + (lane & (gs - 1))) * 8);
    if (p.keys != nullptr) {
      unsigned long long best = 0ull;
      if (phase == 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (col + i < p.V) best = max(best, head_key(acc[i] * sv[i], static_cast<uint32_t>(col + i)));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
      if (lane == 0 && best != 0ull) atomicMax(p.keys, best);
    } else if (phase == 0) {
      float* lp = p.logits + col;
      if (col + 8 <= p.V) {
#pragma unroll
        for (int i = 0; i < 8; ++i) lp[i] = acc[i] * sv[i];
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (col + i < p.V) lp[i] = acc[i] * sv[i];
      }
    }
  }

  if (!ok && lane == 0) {
    for (int st = 0; st < HST; ++st) {
      const int fills = issued > st ? (issued - st + HST - 1) / HST : 0;
      if (fills > 0) mbar_wait_bounded(&bar[st], (fills - 1) & 1, p.timeout_ns, nullptr, p.err, K_HEADR, 2);
    }
  }
}

// ---------------------------------------------------------------- repacking

// Source of byte-word o of the repacked head: kind 0 a table word (4
// columns of one row), 1 a scale; fills *row / *col (first column).
__device__ __forceinline__ int head_source(int64_t o, const w4host::StreamHeadGeom& g, int* row, int64_t* col) {
  const int64_t gw = g.group_bytes / 4;
  const int64_t G = o / gw;
  const int w = static_cast<int>(o - G * gw);
  const int gs = 1 << g.gsl;
  if (w >= g.A * (HROUND / 4)) {  // scales
    *col = G * 8 * gs + (w - g.A * (HROUND / 4));
    return 1;
  }
  const int r = w / (HROUND / 4);
  const int v = w - r * (HROUND / 4);
  const int c = v >> 7, lane = (v >> 2) & 31, ww = v & 3;
  const int strip = lane & (gs - 1), phase = lane >> g.gsl;
  const int b = phase + r * (32 >> g.gsl);
  *row = 16 * b + 2 * c + (ww >> 1);
  *col = (G * gs + strip) * 8 + 4 * (ww & 1);
  return 0;
}

__global__ void i8r_repack_kernel(const int8_t* __restrict__ table, int64_t ldt, const float* __restrict__ scales,
                                  int64_t V, w4host::StreamHeadGeom g, uint32_t* __restrict__ out) {
  const int64_t words = g.bytes / 4;
  for (int64_t o = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; o < words;
       o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int row = 0;
    int64_t col = 0;
    uint32_t v = 0;
    if (head_source(o, g, &row, &col) == 1) {
      v = col < V ? __float_as_uint(scales[col]) : 0u;
    } else {
      const int8_t* src = table + row * ldt + col;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t q = col + i < V ? static_cast<uint32_t>(static_cast<uint8_t>(src[i])) : 0u;
        v |= ((q ^ 0x80u) & 0xFFu) << (8 * i);
      }
    }
    out[o] = v;
  }
}

__global__ void i8r_restore_kernel(const uint32_t* __restrict__ in, int64_t V, w4host::StreamHeadGeom g, int8_t* __restrict__ table,
                                   int64_t ldt, float* __restrict__ scales) {
  const int64_t words = g.bytes / 4;
  for (int64_t o = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; o < words;
       o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int row = 0;
    int64_t col = 0;
    const uint32_t v = in[o];
    if (head_source(o, g, &row, &col) == 1) {
      if (col < V) scales[col] = __uint_as_float(v);
    } else {
      int8_t* dst = table + row * ldt + col;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (col + i < V) dst[i] = static_cast<int8_t>(((v >> (8 * i)) & 0xFFu) ^ 0x80u);
    }
  }
}

bool aligned_to(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

w4_status launch_i8r(const float* h, const void* tr, int64_t K, int64_t V, float* logits, unsigned long long* keys,
                     cudaStream_t st, const w4host::DeviceInfo& di) {
  using namespace w4host;
  w4host::StreamHeadGeom g;
  w4host::stream_head_geom(K, V, &g);
  HParams prm = {};
  prm.tr = static_cast<const uint8_t*>(tr);
  prm.h = h;
  prm.logits = logits;
  prm.keys = keys;
  prm.K = static_cast<int32_t>(K);
  prm.V = static_cast<int32_t>(V);
  prm.ngroups = g.ngroups;
  prm.gsl = g.gsl;
  prm.group_bytes = g.group_bytes;
  prm.err = di.err;
  prm.timeout_ns = wait_timeout_ns();
  static int configured[64] = {};
  if (di.dev < 64 && !configured[di.dev]) {
    const cudaError_t e = cudaFuncSetAttribute(i8r_head_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, HSMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(i8r_head)");
    configured[di.dev] = 1;
  }
  const int grid = std::min(di.sms, g.ngroups);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(HW * 32);
  cfg.dynamicSmemBytes = static_cast<size_t>(HSMEM_BYTES);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, i8r_head_kernel, prm);
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch i8r_head");
}

w4_status check_head_args(const float* h, const void* tr, int64_t K, int64_t V) {
  using namespace w4host;
  w4host::StreamHeadGeom g;
  if (!w4host::stream_head_geom(K, V, &g))
    return fail(W4_ERR_SHAPE, "the streaming head takes K %% 16 == 0, 0 < K <= %d and 0 < V <= 2^30 (K=%lld V=%lld)",
                HKCAP, static_cast<long long>(K), static_cast<long long>(V));
  if (h == nullptr || tr == nullptr) return fail(W4_ERR_NULL, "h and the repacked table must not be NULL");
  if (!aligned_to(h, 16)) return fail(W4_ERR_ALIGN, "h must be 16-byte aligned");
  if (!aligned_to(tr, 16)) return fail(W4_ERR_ALIGN, "the repacked table must be 16-byte aligned");
  return W4_OK;
}

}  // namespace

namespace w4host {

namespace {
int gcd32(int a) {
  int b = 32;
  while (b != 0) {
    const int t = a % b;
    a = b;
    b = t;
  }
  return a;
}
}  // namespace

bool stream_head_geom(int64_t K, int64_t V, StreamHeadGeom* g) {
  if (K <= 0 || V <= 0 || K % 16 != 0 || K > kStreamHeadKCap || V > (int64_t(1) << 30)) return false;
  g->nb = static_cast<int32_t>(K / 16);
  const int gs = 32 / gcd32(g->nb);
  g->gsl = __builtin_ctz(gs);
  g->A = g->nb / gcd32(g->nb);
  const int64_t strips = (V + 7) / 8;
  g->ngroups = static_cast<int32_t>((strips + gs - 1) / gs);
  g->group_bytes = static_cast<int64_t>(g->A) * kStreamHeadRound + 32 * gs;
  g->bytes = g->ngroups * g->group_bytes;
  return true;
}

w4_status check_stream_head(const float* h, const void* tr, int64_t K, int64_t V) { return check_head_args(h, tr, K, V); }

w4_status launch_stream_head(const float* h, const void* tr, int64_t K, int64_t V, float* logits, cudaStream_t st,
                             const DeviceInfo& di) {
  return launch_i8r(h, tr, K, V, logits, nullptr, st, di);
}

}  // namespace w4host

extern "C" {

size_t i8_head_repacked_bytes(int64_t K, int64_t V) {
  w4host::StreamHeadGeom g;
  return w4host::stream_head_geom(K, V, &g) ? static_cast<size_t>(g.bytes) : 0;
}

w4_status i8_head_repack(const int8_t* table, int64_t ldt, const float* scales, int64_t K, int64_t V, void* tr,
                         void* stream) {
  using namespace w4host;
  w4host::StreamHeadGeom g;
  if (!w4host::stream_head_geom(K, V, &g))
    return fail(W4_ERR_SHAPE, "the streaming head takes K %% 16 == 0, 0 < K <= %d and 0 < V <= 2^30", HKCAP);
  if (ldt < V) return fail(W4_ERR_SHAPE, "ldt < V");
  if (table == nullptr || scales == nullptr || tr == nullptr) return fail(W4_ERR_NULL, "NULL buffer");
  if (!aligned_to(scales, 4) || !aligned_to(tr, 16)) return fail(W4_ERR_ALIGN, "scales 4-byte, tr 16-byte aligned");
  const DeviceInfo* di = nullptr;
  w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  const int64_t blocks = std::min<int64_t>((g.bytes / 4 + 255) / 256, static_cast<int64_t>(di->sms) * 32);
  i8r_repack_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      table, ldt, scales, V, g, static_cast<uint32_t*>(tr));
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch i8r_repack");
}

w4_status i8_head_repack_restore(const void* tr, int64_t K, int64_t V, int8_t* table, int64_t ldt, float* scales,
                                 void* stream) {
  using namespace w4host;
  w4host::StreamHeadGeom g;
  if (!w4host::stream_head_geom(K, V, &g))
    return fail(W4_ERR_SHAPE, "the streaming head takes K %% 16 == 0, 0 < K <= %d and 0 < V <= 2^30", HKCAP);
  if (ldt < V) return fail(W4_ERR_SHAPE, "ldt < V");
  if (table == nullptr || scales == nullptr || tr == nullptr) return fail(W4_ERR_NULL, "NULL buffer");
  if (!aligned_to(scales, 4) || !aligned_to(tr, 16)) return fail(W4_ERR_ALIGN, "scales 4-byte, tr 16-byte aligned");
  const DeviceInfo* di = nullptr;
  w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  const int64_t blocks = std::min<int64_t>((g.bytes / 4 + 255) / 256, static_cast<int64_t>(di->sms) * 32);
  i8r_restore_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint32_t*>(tr), V, g, table, ldt, scales);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "launch i8r_restore");
}

w4_status i8r_head_logits(const float* h, const void* tr, int64_t K, int64_t V, float* logits, void* stream) {
  using namespace w4host;
  w4_status rc = check_head_args(h, tr, K, V);
  if (rc != W4_OK) return rc;
  if (logits == nullptr) return fail(W4_ERR_NULL, "logits is NULL");
  if (!aligned_to(logits, 4)) return fail(W4_ERR_ALIGN, "logits must be 4-byte aligned");
  const DeviceInfo* di = nullptr;
  rc = current_device(&di);
  if (rc != W4_OK) return rc;
  return launch_i8r(h, tr, K, V, logits, nullptr, static_cast<cudaStream_t>(stream), *di);
}

w4_status i8r_head_argmax(const float* h, const void* tr, int64_t K, int64_t V, int32_t* token, float* best_logit,
                          void* keys, void* stream) {
  using namespace w4host;
  w4_status rc = check_head_args(h, tr, K, V);
  if (rc != W4_OK) return rc;
  if (V > 0x7fffffff) return fail(W4_ERR_SHAPE, "V must be below 2^31");
  if (token == nullptr || keys == nullptr) return fail(W4_ERR_NULL, "token and keys must not be NULL");
  if (!aligned_to(token, 4) || !aligned_to(best_logit, 4) || !aligned_to(keys, 8))
    return fail(W4_ERR_ALIGN, "token / best 4-byte, keys 8-byte aligned");
  const DeviceInfo* di = nullptr;
  rc = current_device(&di);
  if (rc != W4_OK) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto* k = static_cast<unsigned long long*>(keys);
  cudaError_t e = cudaMemsetAsync(k, 0, 8, st);
  if (e != cudaSuccess) return cuda_fail(e, "clear argmax key");
  rc = launch_i8r(h, tr, K, V, nullptr, k, st, *di);
  if (rc != W4_OK) return rc;
  return launch_argmax_finish(k, 1, token, best_logit, st);
}

}  // extern "C"
