// extern "C" boundary of libw4b200: argument checks, kernel choice, device
// properties, tensor-map encoding, host-side nibble packing, diagnostics.
// Every check runs before any launch; a failed check launches nothing.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <unordered_map>

#include "w4_device.cuh"
#include "w4_internal.h"

// One error word per device that loads the library (see w4_device_error).
__device__ w4dev::ErrorWord g_w4_error_word;

namespace w4host {

namespace {

thread_local char t_detail[512] = "";
std::atomic<uint64_t> g_timeout_ns{2000000000ull};

constexpr int kMaxDev = 64;
DeviceInfo g_dev[kMaxDev];
std::once_flag g_dev_once[kMaxDev];
w4_status g_dev_status[kMaxDev];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

void init_device(int dev) {
  DeviceInfo& d = g_dev[dev];
  d.dev = dev;
  cudaDeviceProp prop;
  cudaError_t e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) {
    g_dev_status[dev] = W4_ERR_CUDA;
    return;
  }
  d.sms = prop.multiProcessorCount;
  d.major = prop.major;
  d.minor = prop.minor;
  d.smem_optin = prop.sharedMemPerBlockOptin;
  if (!(prop.major == 10 && prop.minor == 0)) {
    g_dev_status[dev] = W4_ERR_DEVICE;
    return;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_w4_error_word);
  if (e != cudaSuccess) {
    g_dev_status[dev] = W4_ERR_CUDA;
    return;
  }
  d.err = static_cast<w4dev::ErrorWord*>(p);
  g_dev_status[dev] = W4_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

w4_status fail(w4_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_detail, sizeof(t_detail), fmt, ap);
  va_end(ap);
  return s;
}

w4_status cuda_fail(cudaError_t e, const char* what) {
  return fail(W4_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

uint64_t wait_timeout_ns() { return g_timeout_ns.load(std::memory_order_relaxed); }

w4_status current_device(const DeviceInfo** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(W4_ERR_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDev) return fail(W4_ERR_DEVICE, "device index %d out of range", dev);
  std::call_once(g_dev_once[dev], init_device, dev);
  if (g_dev_status[dev] == W4_ERR_DEVICE)
    return fail(W4_ERR_DEVICE, "device %d is sm_%d%d; this library is built for sm_100a (B200) only", dev,
                g_dev[dev].major, g_dev[dev].minor);
  if (g_dev_status[dev] != W4_OK) return fail(g_dev_status[dev], "device %d could not be queried", dev);
  *out = &g_dev[dev];
  return W4_OK;
}

static w4_status encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                           uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows) {
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(W4_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d): dims %llu x %llu, box %u x %u", int(r),
                (unsigned long long)inner, (unsigned long long)rows, box_inner, box_rows);
  return W4_OK;
}

namespace {
struct MapKey {
  const void* qw;
  int64_t K, N;
  bool operator==(const MapKey& o) const { return qw == o.qw && K == o.K && N == o.N; }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    size_t h = reinterpret_cast<size_t>(k.qw) * 0x9E3779B97F4A7C15ull;
    h ^= static_cast<size_t>(k.K) * 31 + static_cast<size_t>(k.N) + (h << 6) + (h >> 2);
    return h;
  }
};
struct MapSet {
  CUtensorMap m[4];
};
std::mutex g_map_mu;
std::unordered_map<MapKey, MapSet, MapKeyHash> g_map_cache;
constexpr size_t kMapCacheMax = 4096;
}  // namespace

// The four tensor maps of one packed weight, all over the [K rows][N/2 bytes]
// nibble matrix: 256-byte-wide boxes of 128 and 16 rows (wide tiles) and
// 128-byte-wide boxes of 256 and 32 rows (narrow tiles). A map is a pure
// function of (pointer, K, N), so the cache can never return a stale one:
// reusing freed memory for another weight of the same shape yields the same
// map.
w4_status encode_w4_maps(CUtensorMap* wide_full, CUtensorMap* wide_unit, CUtensorMap* narrow_full,
                         CUtensorMap* narrow_unit, const uint8_t* qw, int64_t K, int64_t N) {
  const MapKey key{qw, K, N};
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    auto itc = g_map_cache.find(key);
    if (itc != g_map_cache.end()) {
      *wide_full = itc->second.m[0];
      *wide_unit = itc->second.m[1];
      *narrow_full = itc->second.m[2];
      *narrow_unit = itc->second.m[3];
      return W4_OK;
    }
  }
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (g_encode == nullptr) return fail(W4_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const uint64_t half = static_cast<uint64_t>(N / 2);
  MapSet ms;
  w4_status rc;
  if ((rc = encode_2d(&ms.m[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, qw, half, K, half, 256, 128)) != W4_OK) return rc;
  if ((rc = encode_2d(&ms.m[1], CU_TENSOR_MAP_DATA_TYPE_UINT8, qw, half, K, half, 256, 16)) != W4_OK) return rc;
  if ((rc = encode_2d(&ms.m[2], CU_TENSOR_MAP_DATA_TYPE_UINT8, qw, half, K, half, 128, 256)) != W4_OK) return rc;
  if ((rc = encode_2d(&ms.m[3], CU_TENSOR_MAP_DATA_TYPE_UINT8, qw, half, K, half, 128, 32)) != W4_OK) return rc;
  *wide_full = ms.m[0];
  *wide_unit = ms.m[1];
  *narrow_full = ms.m[2];
  *narrow_unit = ms.m[3];
  std::lock_guard<std::mutex> lk(g_map_mu);
  if (g_map_cache.size() >= kMapCacheMax) g_map_cache.clear();
  g_map_cache.emplace(key, ms);
  return W4_OK;
}

// ------------------------------------------------------------------ validation

static w4_status check_desc(const w4_desc& d) {
  if (d.M < 0 || d.K < 0 || d.N < 0) return fail(W4_ERR_SHAPE, "negative size (M=%lld K=%lld N=%lld)",
                                                 (long long)d.M, (long long)d.K, (long long)d.N);
  if (d.K % 32 != 0) return fail(W4_ERR_SHAPE, "K=%lld is not a multiple of 32", (long long)d.K);
  if (d.N % 2 != 0) return fail(W4_ERR_SHAPE, "N=%lld is odd", (long long)d.N);
  if (d.act < W4_ACT_NONE || d.act > W4_ACT_GELU_ERF) return fail(W4_ERR_VALUE, "unknown activation %d", int(d.act));
  if (d.reserved != 0) return fail(W4_ERR_VALUE, "reserved field must be 0");
  if (d.M == 0 || d.N == 0) return W4_OK;
  if (d.y == nullptr) return fail(W4_ERR_NULL, "y is NULL");
  if (d.ldy < d.N) return fail(W4_ERR_SHAPE, "ldy=%lld < N=%lld", (long long)d.ldy, (long long)d.N);
  if (!aligned(d.y, 4)) return fail(W4_ERR_ALIGN, "y must be 4-byte aligned");
  if (d.bias != nullptr && !aligned(d.bias, 4)) return fail(W4_ERR_ALIGN, "bias must be 4-byte aligned");
  if (d.residual != nullptr) {
    if (d.ldr < d.N) return fail(W4_ERR_SHAPE, "ldr=%lld < N=%lld", (long long)d.ldr, (long long)d.N);
    if (!aligned(d.residual, 4)) return fail(W4_ERR_ALIGN, "residual must be 4-byte aligned");
    if (d.residual == d.y && d.ldr != d.ldy)
      return fail(W4_ERR_SHAPE, "an in-place residual (residual == y) needs ldr == ldy");
  }
  if (d.K == 0) return W4_OK;
  if (d.x == nullptr || d.qw == nullptr || d.scales == nullptr || d.zp == nullptr)
    return fail(W4_ERR_NULL, "x, qw, scales and zp must not be NULL");
  if (d.ldx < d.K) return fail(W4_ERR_SHAPE, "ldx=%lld < K=%lld", (long long)d.ldx, (long long)d.K);
  if (!aligned(d.qw, 16) || !aligned(d.scales, 16) || !aligned(d.zp, 16))
    return fail(W4_ERR_ALIGN, "qw, scales and zp must be 16-byte aligned");
  if (!aligned(d.x, 4)) return fail(W4_ERR_ALIGN, "x must be 4-byte aligned");
  return W4_OK;
}

}  // namespace w4host

using namespace w4host;

extern "C" {

int32_t w4_abi_version(void) { return W4_ABI_VERSION; }

const char* w4_status_string(w4_status s) {
  switch (s) {
    case W4_OK: return "W4_OK";
    case W4_ERR_NULL: return "W4_ERR_NULL";
    case W4_ERR_SHAPE: return "W4_ERR_SHAPE";
    case W4_ERR_ALIGN: return "W4_ERR_ALIGN";
    case W4_ERR_DEVICE: return "W4_ERR_DEVICE";
    case W4_ERR_CUDA: return "W4_ERR_CUDA";
    case W4_ERR_TIMEOUT: return "W4_ERR_TIMEOUT";
    case W4_ERR_WORKSPACE: return "W4_ERR_WORKSPACE";
    case W4_ERR_VALUE: return "W4_ERR_VALUE";
  }
  return "W4_ERR_UNKNOWN";
}

const char* w4_last_error(void) { return t_detail; }

w4_status w4_set_wait_timeout_ns(uint64_t ns) {
  if (ns == 0) return fail(W4_ERR_VALUE, "timeout must be positive");
  g_timeout_ns.store(ns);
  return W4_OK;
}

// ------------------------------------------------------------------ packing

w4_status w4_pack_nibbles(const uint8_t* q, int64_t n, uint8_t* out) {
  if (n < 0) return fail(W4_ERR_SHAPE, "negative count");
  if (n == 0) return W4_OK;
  if (q == nullptr || out == nullptr) return fail(W4_ERR_NULL, "NULL buffer");
  for (int64_t i = 0; i < n; ++i)
    if (q[i] > 15) return fail(W4_ERR_VALUE, "value %u at %lld exceeds 15", unsigned(q[i]), (long long)i);
  for (int64_t i = 0; i + 1 < n; i += 2) out[i / 2] = static_cast<uint8_t>(q[i] | (q[i + 1] << 4));
  if (n & 1) out[n / 2] = q[n - 1];
  return W4_OK;
}

w4_status w4_unpack_nibbles(const uint8_t* packed, int64_t n, uint8_t* q) {
  if (n < 0) return fail(W4_ERR_SHAPE, "negative count");
  if (n == 0) return W4_OK;
  if (q == nullptr || packed == nullptr) return fail(W4_ERR_NULL, "NULL buffer");
  for (int64_t i = 0; i < n; ++i) q[i] = (i & 1) ? (packed[i / 2] >> 4) : (packed[i / 2] & 0x0F);
  return W4_OK;
}

// ------------------------------------------------------------------ body

size_t w4_matmul_workspace_size(int64_t M, int64_t K, int64_t N) {
  const DeviceInfo* di = nullptr;
  if (current_device(&di) != W4_OK || M <= 0 || K <= 0 || N <= 0 || K % 32 || N % 2) return 0;
  // the GEMV's need (a call may force the GEMV for any M; the tensor-core and
  // plain kernels need none)
  w4_desc d = {};
  d.M = M;
  d.K = K;
  d.N = N;
  return gemv_workspace_bytes(&d, 1, di->sms);
}

static w4_status matmul_one(const w4_desc& d, void* ws, size_t wsb, w4_path path, cudaStream_t st) {
  w4_status rc = check_desc(d);
  if (rc != W4_OK) return rc;
  if (path < W4_PATH_AUTO || path > W4_PATH_TC) return fail(W4_ERR_VALUE, "unknown path %d", int(path));
  if (d.M == 0 || d.N == 0) return W4_OK;
  const DeviceInfo* di = nullptr;
  rc = current_device(&di);
  if (rc != W4_OK) return rc;
  if (d.K == 0) return launch_zero_fill(d.y, d.ldy, d.M, d.N, st, &d);
  const char* why = "";
  const char* why_tc = "";
  const bool gemv_ok = gemv_eligible(d, &why);
  const bool tc_ok = tc_eligible(d, &why_tc);
  switch (path) {
    case W4_PATH_GENERIC: return launch_generic(d, st, *di);
    case W4_PATH_GEMV:
      if (!gemv_ok) return fail(W4_ERR_ALIGN, "%s", why);
      return launch_gemv(&d, 1, ws, wsb, st, *di);
    case W4_PATH_TC:
      if (!tc_ok) return fail(W4_ERR_ALIGN, "%s", why_tc);
      return launch_tc(&d, 1, st, *di);
    default:
      if (d.M > kTcMinM) return tc_ok ? launch_tc(&d, 1, st, *di) : launch_generic(d, st, *di);
      return gemv_ok ? launch_gemv(&d, 1, ws, wsb, st, *di) : launch_generic(d, st, *di);
  }
}

w4_status w4_matmul_desc(const w4_desc* d, void* workspace, size_t workspace_bytes, w4_path path, void* stream) {
  if (d == nullptr) return fail(W4_ERR_NULL, "descriptor is NULL");
  return matmul_one(*d, workspace, workspace_bytes, path, static_cast<cudaStream_t>(stream));
}

w4_status w4_matmul_path(const float* x, int64_t ldx, const uint8_t* qw, const float* scales, const uint8_t* zp,
                         float* y, int64_t ldy, int64_t M, int64_t K, int64_t N, void* workspace,
                         size_t workspace_bytes, w4_path path, void* stream) {
  const w4_desc d = {x, ldx, qw, scales, zp, y, ldy, M, K, N};
  return matmul_one(d, workspace, workspace_bytes, path, static_cast<cudaStream_t>(stream));
}

w4_status w4_matmul(const float* x, int64_t ldx, const uint8_t* qw, const float* scales, const uint8_t* zp, float* y,
                    int64_t ldy, int64_t M, int64_t K, int64_t N, void* workspace, size_t workspace_bytes,
                    void* stream) {
  return w4_matmul_path(x, ldx, qw, scales, zp, y, ldy, M, K, N, workspace, workspace_bytes, W4_PATH_AUTO, stream);
}

size_t w4_matmul_grouped_workspace_size(const w4_desc* descs, int32_t count) {
  const DeviceInfo* di = nullptr;
  if (descs == nullptr || count <= 0 || current_device(&di) != W4_OK) return 0;
  size_t best = 0;
  // the GEMV takes the descriptors with M <= kTcMinM, W4_GROUP_MAX per launch
  static thread_local w4_desc small[W4_GROUP_MAX];
  int n = 0;
  for (int32_t i = 0; i < count; ++i) {
    if (descs[i].M > kTcMinM) continue;
    small[n++] = descs[i];
    if (n == W4_GROUP_MAX || i == count - 1) {
      const size_t b = gemv_workspace_bytes(small, n, di->sms);
      best = b > best ? b : best;
      n = 0;
    }
  }
  if (n > 0) {
    const size_t b = gemv_workspace_bytes(small, n, di->sms);
    best = b > best ? b : best;
  }
  return best;
}

w4_status w4_matmul_grouped(const w4_desc* descs, int32_t count, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (count < 0) return fail(W4_ERR_SHAPE, "negative count");
  if (count == 0) return W4_OK;
  if (descs == nullptr) return fail(W4_ERR_NULL, "descs is NULL");
  for (int32_t i = 0; i < count; ++i) {
    const w4_status rc = check_desc(descs[i]);
    if (rc != W4_OK) {
      char why[sizeof(t_detail)];
      snprintf(why, sizeof(why), "%s", t_detail);
      return fail(rc, "descriptor %d: %s", i, why);
    }
  }
  const DeviceInfo* di = nullptr;
  w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Split: descriptors with M <= kTcMinM that the GEMV can take go into
  // grouped GEMV launches, larger M into grouped tensor-core launches; the
  // rest (K = 0, odd layouts) run one by one on their own kernels.
  static thread_local w4_desc fast[W4_GROUP_MAX];
  static thread_local w4_desc tc[W4_GROUP_MAX];
  int nfast = 0, ntc = 0;
  for (int32_t i = 0; i < count; ++i) {
    const w4_desc& d = descs[i];
    if (d.M == 0 || d.N == 0) continue;
    const char* why = "";
    if (d.K == 0) {
      rc = launch_zero_fill(d.y, d.ldy, d.M, d.N, st, &d);
    } else if (d.M > kTcMinM) {
      if (!tc_eligible(d, &why)) {
        rc = launch_generic(d, st, *di);
      } else {
        tc[ntc++] = d;
        if (ntc == W4_GROUP_MAX) {
          rc = launch_tc(tc, ntc, st, *di);
          ntc = 0;
        }
      }
    } else if (!gemv_eligible(d, &why)) {
      rc = launch_generic(d, st, *di);
    } else {
      fast[nfast++] = d;
      if (nfast == W4_GROUP_MAX) {
        rc = launch_gemv(fast, nfast, workspace, workspace_bytes, st, *di);
        nfast = 0;
      }
    }
    if (rc != W4_OK) return rc;
  }
  if (nfast > 0) rc = launch_gemv(fast, nfast, workspace, workspace_bytes, st, *di);
  if (rc != W4_OK) return rc;
  if (ntc > 0) rc = launch_tc(tc, ntc, st, *di);
  return rc;
}

// ------------------------------------------------------------------ head

static w4_status head_impl(const HeadArgs& a, void* ws, size_t wsb, w4_path path, cudaStream_t st) {
  if (a.M < 0 || a.K < 0 || a.V < 0) return fail(W4_ERR_SHAPE, "negative size");
  if (path != W4_PATH_AUTO && path != W4_PATH_GEMV && path != W4_PATH_GENERIC)
    return fail(W4_ERR_VALUE, "path %d is not a head path", int(path));
  if (a.M == 0 || a.V == 0) return W4_OK;
  if (a.logits == nullptr) return fail(W4_ERR_NULL, "logits is NULL");
  if (a.ldl < a.V) return fail(W4_ERR_SHAPE, "ldl < V");
  if (!aligned(a.logits, 4)) return fail(W4_ERR_ALIGN, "logits must be 4-byte aligned");
  if (a.K > 0) {
    if (a.h == nullptr || a.table == nullptr || a.scales == nullptr)
      return fail(W4_ERR_NULL, "h, table and scales must not be NULL");
    if (a.ldh < a.K) return fail(W4_ERR_SHAPE, "ldh < K");
    if (a.ldt < a.V) return fail(W4_ERR_SHAPE, "ldt < V");
    if (!aligned(a.h, 4) || !aligned(a.scales, 4)) return fail(W4_ERR_ALIGN, "h and scales must be 4-byte aligned");
    if (!aligned(a.table, 16)) return fail(W4_ERR_ALIGN, "table must be 16-byte aligned");
  }
  const DeviceInfo* di = nullptr;
  w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  if (a.K == 0) return launch_zero_fill(a.logits, a.ldl, a.M, a.V, st);
  if (path == W4_PATH_GENERIC) return launch_head_generic(a, st, *di);
  return launch_head(a, ws, wsb, st, *di);
}

// Greedy decoding: when the rows kernel folds the logits itself the workspace
// is [64-bit keys, M of them]; otherwise [the head's own workspace, so that
// its counter block sits at the start as always][keys][logits M x V], each
// part 256-byte aligned.
static size_t round256(size_t b) { return (b + 255) / 256 * 256; }

static size_t argmax_head_ws(int64_t M, int64_t K, int64_t V, int sms) {
  return head_rows_path(M, K) ? 0 : round256(head_workspace_bytes(M, K, V, sms));
}

static size_t argmax_ws_bytes(int64_t M, int64_t K, int64_t V, int sms) {
  size_t b = argmax_head_ws(M, K, V, sms) + round256(static_cast<size_t>(M) * 8);
  if (!head_rows_path(M, K)) b += static_cast<size_t>(M) * static_cast<size_t>(V) * 4;
  return b;
}

size_t i8_head_argmax_workspace_size(int64_t M, int64_t K, int64_t V) {
  const DeviceInfo* di = nullptr;
  if (current_device(&di) != W4_OK || M <= 0 || K < 0 || V <= 0) return 0;
  return argmax_ws_bytes(M, K, V, di->sms);
}

w4_status i8_head_argmax(const float* h, int64_t ldh, const int8_t* table, int64_t ldt, const float* scales,
                         int64_t M, int64_t K, int64_t V, int32_t* tokens, float* best_logits, void* workspace,
                         size_t workspace_bytes, void* stream) {
  if (M < 0 || K < 0 || V < 0) return fail(W4_ERR_SHAPE, "negative size");
  if (M == 0) return W4_OK;
  if (V == 0) return fail(W4_ERR_SHAPE, "V == 0: no token to choose");
  if (V > 0x7fffffff || M > 65535) return fail(W4_ERR_SHAPE, "V must be below 2^31 and M at most 65535");
  if (tokens == nullptr) return fail(W4_ERR_NULL, "tokens is NULL");
  if (!aligned(tokens, 4) || !aligned(best_logits, 4)) return fail(W4_ERR_ALIGN, "tokens and best must be 4-byte aligned");
  if (K > 0) {
    if (h == nullptr || table == nullptr || scales == nullptr)
      return fail(W4_ERR_NULL, "h, table and scales must not be NULL");
    if (ldh < K) return fail(W4_ERR_SHAPE, "ldh < K");
    if (ldt < V) return fail(W4_ERR_SHAPE, "ldt < V");
    if (!aligned(h, 4) || !aligned(scales, 4)) return fail(W4_ERR_ALIGN, "h and scales must be 4-byte aligned");
    if (!aligned(table, 16)) return fail(W4_ERR_ALIGN, "table must be 16-byte aligned");
  }
  const DeviceInfo* di = nullptr;
  w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  const size_t need = argmax_ws_bytes(M, K, V, di->sms);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(W4_ERR_WORKSPACE, "argmax workspace of %zu bytes needed, %zu given", need,
                workspace == nullptr ? size_t(0) : workspace_bytes);
  if (!aligned(workspace, 16)) return fail(W4_ERR_WORKSPACE, "workspace must be 16-byte aligned");
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t hws_bytes = argmax_head_ws(M, K, V, di->sms);
  auto* keys = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(workspace) + hws_bytes);
  cudaError_t e = cudaMemsetAsync(keys, 0, static_cast<size_t>(M) * 8, st);
  if (e != cudaSuccess) return cuda_fail(e, "clear argmax keys");
  if (head_rows_path(M, K)) {
    const HeadArgs a = {h, ldh, table, ldt, scales, nullptr, V, M, K, V};
    rc = launch_head_keys(a, keys, st, *di);
  } else {
    float* logits = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(keys) + round256(static_cast<size_t>(M) * 8));
    if (K == 0) {
      rc = launch_zero_fill(logits, V, M, V, st);
    } else {
      const HeadArgs a = {h, ldh, table, ldt, scales, logits, V, M, K, V};
      rc = launch_head(a, hws_bytes > 0 ? workspace : nullptr, hws_bytes, st, *di);
    }
    if (rc == W4_OK) rc = launch_argmax_rows(logits, V, M, V, keys, st);
  }
  if (rc != W4_OK) return rc;
  rc = launch_argmax_finish(keys, M, tokens, best_logits, st);
  if (rc != W4_OK) return rc;
  // the keys may lie in the block where other calls keep their counters:
  // leave them zero, as every call of this library leaves that block
  e = cudaMemsetAsync(keys, 0, static_cast<size_t>(M) * 8, st);
  return e == cudaSuccess ? W4_OK : cuda_fail(e, "clear argmax keys");
}

size_t i8_head_workspace_size(int64_t M, int64_t K, int64_t V) {
  const DeviceInfo* di = nullptr;
  if (current_device(&di) != W4_OK) return 0;
  return head_workspace_bytes(M, K, V, di->sms);
}

w4_status i8_head_logits_path(const float* h, int64_t ldh, const int8_t* table, int64_t ldt, const float* scales,
                              float* logits, int64_t ldl, int64_t M, int64_t K, int64_t V, void* workspace,
                              size_t workspace_bytes, w4_path path, void* stream) {
  const HeadArgs a = {h, ldh, table, ldt, scales, logits, ldl, M, K, V};
  return head_impl(a, workspace, workspace_bytes, path, static_cast<cudaStream_t>(stream));
}

w4_status i8_head_logits(const float* h, int64_t ldh, const int8_t* table, int64_t ldt, const float* scales,
                         float* logits, int64_t ldl, int64_t M, int64_t K, int64_t V, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return i8_head_logits_path(h, ldh, table, ldt, scales, logits, ldl, M, K, V, workspace, workspace_bytes,
                             W4_PATH_AUTO, stream);
}

// ------------------------------------------------------------------ diagnostics

w4_status w4_device_error(int32_t* info4, int32_t clear) {
  const DeviceInfo* di = nullptr;
  w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  w4dev::ErrorWord w = {};
  cudaError_t e = cudaMemcpyFromSymbol(&w, g_w4_error_word, sizeof(w));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (info4 != nullptr) {
    info4[0] = w.status;
    info4[1] = w.kernel;
    info4[2] = w.block;
    info4[3] = w.detail;
  }
  if (clear) {
    const w4dev::ErrorWord z = {};
    e = cudaMemcpyToSymbol(g_w4_error_word, &z, sizeof(z));
    if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
  }
  return static_cast<w4_status>(w.status);
}

w4_status w4_debug_wait_timeout(uint64_t timeout_ns, void* stream) {
  const DeviceInfo* di = nullptr;
  w4_status rc = current_device(&di);
  if (rc != W4_OK) return rc;
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return fail(W4_ERR_VALUE, "timeout must be in (0, 10 s]");
  return launch_debug_wait(timeout_ns, static_cast<cudaStream_t>(stream), *di);
}

}  // extern "C"
