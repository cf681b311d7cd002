/*
 * w4.h — C ABI of the B200 quantised-weight matmul library (libw4b200.so).
 *
 * Two operations, both fp32 in and out, both hand-written CUDA for sm_100a:
 *
 *  w4_matmul       y = x . W, W[K, N] stored 4-bit asymmetric in blocks of 32
 *                  along K with one fp32 scale and one uint4 zero point per
 *                  (block, column), dequantised as w = (q - zp) * scale.
 *                  Source: "ONNX export, quantization and the browser runtime"
 *                  (tokenling docs), section "Quantization (train/quantize.py)",
 *                  steps 1 (gemm_to_matmul: plain [K, N] weights, K = in,
 *                  N = out) and 2 (dq4: 4-bit asymmetric, blocks of 32 along K,
 *                  fp32 scale + uint4 zero point per block, raw packed UINT4,
 *                  restored by one blocked DequantizeLinear).
 *
 *  i8_head_logits  logits = h . (T * s), T[K, V] int8 with one fp32 scale per
 *                  token column, applied to the last position only.
 *                  Source: same page and section, steps 3 (embedding_int8: the
 *                  tied embedding / LM head stored once as int8, one scale per
 *                  token, in the head's [768, V] layout) and 4
 *                  (last_token_logits: the head reads the last position only).
 *
 * Data layouts (all row-major):
 *   x       fp32 [M, K], row stride ldx >= K (elements).
 *   qw      uint8 [K * N / 2]: element (k, n) of the [K, N] nibble tensor is
 *           flat index i = k*N + n, stored in byte i >> 1, low nibble when i is
 *           even ("raw packed UINT4", low nibble first).
 *   scales  fp32 [K/32, N]; row b holds the scales of rows 32b .. 32b+31.
 *   zp      uint8 [(K/32) * N / 2]: the [K/32, N] zero-point tensor packed by
 *           the same rule as qw.
 *   y       fp32 [M, N], row stride ldy >= N; fully overwritten.
 *   table   int8 [K, V] with row stride ldt >= V (bytes); row k starts at byte
 *           k * ldt, which need not be aligned (V = 50257 is odd).
 *   logits  fp32 [M, V], row stride ldl >= V; fully overwritten.
 *
 * Conventions shared by every entry point:
 *   - All array pointers are DEVICE pointers owned by the caller (for example
 *     torch tensors). The library allocates no device memory and keeps no
 *     per-call state.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Calls are asynchronous and stream-ordered: nothing inside
 *     synchronises with the host, except the functions marked SYNCHRONOUS.
 *   - Every argument check runs before any launch. On failure the call
 *     returns the status, launches nothing and records a one-line reason that
 *     w4_last_error() returns on the same host thread.
 *   - There is no CPU fallback: every result is computed by this library's
 *     kernels on the GPU, or the call fails.
 *   - Sizes are int64_t; M = 0 or N = 0 (V = 0) is a valid no-op; K = 0 writes
 *     zeros (the empty sum).
 */
#ifndef W4_B200_H
#define W4_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define W4_ABI_VERSION 6

#if defined(__GNUC__)
#define W4_API __attribute__((visibility("default")))
#else
#define W4_API
#endif

typedef enum w4_status {
  W4_OK = 0,
  W4_ERR_NULL = 1,      /* a required pointer is NULL                                */
  W4_ERR_SHAPE = 2,     /* K % 32 != 0, N odd, negative size, ld < row length, ...   */
  W4_ERR_ALIGN = 3,     /* qw / scales / zp not 16-byte aligned; fp32 not 4-byte     */
  W4_ERR_DEVICE = 4,    /* current device is not sm_100 (B200), or no device          */
  W4_ERR_CUDA = 5,      /* a CUDA runtime call or launch failed (detail in last_error) */
  W4_ERR_TIMEOUT = 6,   /* a bounded device-side wait ran out (see w4_device_error)  */
  W4_ERR_WORKSPACE = 7, /* workspace missing, too small or misaligned                */
  W4_ERR_VALUE = 8      /* a host-side value out of range (e.g. a nibble > 15)       */
} w4_status;

/* Kernel choice. W4_PATH_AUTO picks by shape, alignment and M; the others
 * force one of this library's own kernels (for tests and benchmarks) and
 * fail with W4_ERR_SHAPE / W4_ERR_ALIGN when that kernel cannot take the
 * call. */
typedef enum w4_path {
  W4_PATH_AUTO = 0,
  W4_PATH_GEMV = 1,    /* TMA-fed stream-K GEMV: N % 32 == 0, x 16-B aligned, ldx % 4 == 0 */
  W4_PATH_GENERIC = 2, /* plain-load kernel: any even N, any 4-B aligned x / y                */
  W4_PATH_TC = 3       /* tcgen05 3xTF32 tile GEMM (large M)                                  */
} w4_path;

/* Activation of the fused epilogue (see w4_desc). GPT-2's MLP uses the
 * tanh form ("gelu_new"); the erf form is the exact GELU. */
typedef enum w4_act {
  W4_ACT_NONE = 0,      /* identity                                                   */
  W4_ACT_GELU_TANH = 1, /* 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3)))            */
  W4_ACT_GELU_ERF = 2   /* 0.5 v (1 + erf(v / sqrt(2)))                                */
} w4_act;

/* One matmul: the fields x .. N as in w4_matmul, then an optional fused
 * epilogue. The pages' export step "gemm_to_matmul" ("ONNX export,
 * quantization and the browser runtime", section "Quantization
 * (train/quantize.py)", step 1) splits every GPT-2 Conv1D into MatMul + Add;
 * the epilogue folds that Add, and the activation or residual add that
 * follows it in the model, into the kernel's final store:
 *   y[m, n] = act(x.W[m, n] + bias[n]) + residual[m * ldr + n]
 * all in fp32, in that order.
 * - bias: NULL or [N] fp32, 4-byte aligned.
 * - residual: NULL or [M, N] fp32 with row stride ldr >= N, 4-byte aligned.
 *   It may be y itself (same pointer and ldr == ldy: an in-place residual
 *   update); any other overlap with y or the inputs is not allowed.
 * - act: a w4_act value; anything else is refused with W4_ERR_VALUE.
 * - reserved: must be 0.
 * All-zero epilogue fields (what a zero-initialised struct holds) mean plain
 * y = x.W. */
typedef struct w4_desc {
  const float* x;
  int64_t ldx;
  const uint8_t* qw;
  const float* scales;
  const uint8_t* zp;
  float* y;
  int64_t ldy;
  int64_t M;
  int64_t K;
  int64_t N;
  const float* bias;
  const float* residual;
  int64_t ldr;
  int32_t act;
  int32_t reserved;
} w4_desc;

/* ------------------------------------------------------------------ body */

/* Bytes of workspace w4_matmul needs for this shape on the current device
 * (0 when none is needed). The workspace starts with a fixed block of
 * 32-bit split-K counters followed by partial sums. It must be device memory,
 * 16-byte aligned,
 * and ZERO-FILLED before its first use; every successful call leaves the
 * counter block zero again (the partial sums need no zeroing), so one
 * zeroing at allocation suffices. Two calls that
 * may run at the same time must not share a workspace. After a call that
 * reported W4_ERR_TIMEOUT, zero it again before reuse. */
W4_API size_t w4_matmul_workspace_size(int64_t M, int64_t K, int64_t N);

/* y[M, N] = x[M, K] . W[K, N] with W in the 4-bit blocked format above.
 * Requires K % 32 == 0, N even, ldx >= K, ldy >= N, qw / scales / zp 16-byte
 * aligned, x / y 4-byte aligned. workspace may be NULL only when
 * w4_matmul_workspace_size() returns 0. */
W4_API w4_status w4_matmul(const float* x, int64_t ldx, const uint8_t* qw, const float* scales,
                    const uint8_t* zp, float* y, int64_t ldy, int64_t M, int64_t K, int64_t N,
                    void* workspace, size_t workspace_bytes, void* stream);

/* One matmul described by a w4_desc (epilogue included), with a kernel
 * choice; the workspace rules are w4_matmul's. `d` is a HOST pointer read
 * during the call only. */
W4_API w4_status w4_matmul_desc(const w4_desc* d, void* workspace, size_t workspace_bytes, w4_path path,
                                void* stream);

/* As w4_matmul with an explicit kernel choice. */
W4_API w4_status w4_matmul_path(const float* x, int64_t ldx, const uint8_t* qw, const float* scales,
                         const uint8_t* zp, float* y, int64_t ldy, int64_t M, int64_t K,
                         int64_t N, void* workspace, size_t workspace_bytes, w4_path path,
                         void* stream);

/* Allocation-free form of w4_matmul. The pages describe no such entry point;
 * it exists for callers that cannot allocate device memory where they
 * multiply (for example a plugin inside a framework that owns every device
 * allocation, or a process that forbids allocation after start-up). Inputs
 * and outputs are the caller's, exactly as for w4_matmul; the split-K scratch
 * comes from one array of W4_NOALLOC_SCRATCH_BYTES inside this library,
 * which every GPU that loads the library keeps until the process exits.
 * - The scratch is the split-K GEMV's (M <= 16); a call that w4_matmul sends
 *   to the tensor-core kernel (M > 16) or to the plain kernel needs none.
 *   Shapes whose scratch need (w4_matmul_workspace_size) exceeds the array
 *   are refused with W4_ERR_WORKSPACE. The need grows with M and with the
 *   number of SMs the call keeps busy (4 KB + SMs x M' x 4 KB, M' = M rounded
 *   up to 1, 2, 4 or 8): on a 148-SM B200 every M <= 2 fits (at most
 *   1.2 MB), while M from 3 to 16 fits only for weights too small to fill
 *   the GPU.
 * - Each call that needs scratch first clears the split-K counters at its
 *   start, then runs as w4_matmul. Calls share the array, so calls that
 *   overlap on the GPU (other streams, other host threads on the same
 *   device) race: serialise them.
 * - The first call on a device looks up the array's device address; make
 *   that first call before any stream capture.
 * Calls no allocating routine. */
#define W4_NOALLOC_SCRATCH_BYTES (2u << 20)
W4_API w4_status w4_matmul_noalloc(const float* x, int64_t ldx, const uint8_t* qw, const float* scales,
                                   const uint8_t* zp, float* y, int64_t ldy, int64_t M, int64_t K,
                                   int64_t N, void* stream);

/* Many independent matmuls (for example the 48 weights of a decoder stack)
 * in as few launches as possible: up to W4_GROUP_MAX descriptors share one
 * persistent launch whose work is split evenly over the SMs. `descs` is a
 * HOST array read during the call only. The outputs must not overlap each
 * other or any input. */
#define W4_GROUP_MAX 48
W4_API size_t w4_matmul_grouped_workspace_size(const w4_desc* descs, int32_t count);
W4_API w4_status w4_matmul_grouped(const w4_desc* descs, int32_t count, void* workspace,
                            size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------ streaming layout (decode) */

/* The streaming layout of one W4 weight: the same 32-bit words as the three
 * page-format buffers above (nibble words of 8 consecutive columns of one
 * row, fp32 scales, zero-point words of 8 columns; "ONNX export, quantization
 * and the browser runtime", section "Quantization (train/quantize.py)",
 * step 2), reordered once at load time into the order in which the decode
 * GEMV streams them, so that each of its warps reads one contiguous run of
 * bytes. Nothing is added, rounded or dropped: w4_repack_restore gives back
 * the page-format buffers bit for bit.
 *
 * Layout, K % 32 == 0, N % 8 == 0, nb = K / 32, gs = 32 / gcd(nb, 32),
 * A = gs * nb / 32: groups of 8 gs columns (all K rows) in column order, each
 * group A rounds of 5248 bytes. In round r of group G, lane l (0..31) owns
 * strip s = l % gs (columns c0 = 8 (G gs + s) .. c0 + 7) and block
 * b = l / gs + r * (32 / gs); its bytes are
 *   nibble word of row 32 b + 4 c + j (c, j in 0..7, 0..3) at c*512 + l*16 + j*4
 *     (the page's 4-byte word of row 32 b + 4 c + j, columns c0..c0+7),
 *   scale of column c0 + i (i in 0..7) at 4096 + (i/4)*512 + l*16 + (i%4)*4,
 *   zero-point word of block b, columns c0..c0+7, at 5120 + l*4.
 * Strips at or past N (N not a multiple of 8 gs) hold zeros.
 * w4_repacked_bytes() is the buffer size: K*N/2 + (K/32)*N*4 + (K/32)*N/2
 * bytes (the page-format total) when N is a multiple of 8 gs, a little more
 * otherwise; 0 for a shape the layout does not take. */
W4_API size_t w4_repacked_bytes(int64_t K, int64_t N);

/* Page format -> streaming layout, on the GPU. qw / scales / zp as for
 * w4_matmul, wr: w4_repacked_bytes(K, N) bytes of device memory; all four
 * 16-byte aligned. Asynchronous, stream-ordered. W4_ERR_SHAPE unless
 * K % 32 == 0, N % 8 == 0 and 0 < K, N <= 2^30. */
W4_API w4_status w4_repack(const uint8_t* qw, const float* scales, const uint8_t* zp, int64_t K, int64_t N,
                           void* wr, void* stream);

/* Streaming layout -> page format (the exact inverse of w4_repack). */
W4_API w4_status w4_repack_restore(const void* wr, int64_t K, int64_t N, uint8_t* qw, float* scales, uint8_t* zp,
                                   void* stream);

/* One decode matmul on a repacked weight: y[1, N] = act(x[1, K] . W + bias)
 * + residual, the fields and the epilogue as in w4_desc (ldx / ldy / ldr are
 * not used: one row). Requires M == 1 (W4_ERR_SHAPE otherwise), K % 32 == 0,
 * K <= 14336, N % 8 == 0, x and wr 16-byte aligned, y / bias / residual
 * 4-byte aligned. No workspace: every output column is summed inside one
 * warp. reserved must be 0. */
typedef struct w4r_desc {
  const float* x;
  int64_t ldx;
  const void* wr;
  float* y;
  int64_t ldy;
  int64_t M;
  int64_t K;
  int64_t N;
  const float* bias;
  const float* residual;
  int64_t ldr;
  int32_t act;
  int32_t reserved;
} w4r_desc;

/* Many independent decode matmuls on repacked weights in as few launches as
 * possible (128 per launch; a launch whose CTAs would each stage more than
 * 14336 floats of x is split). `descs` is a HOST array read during the call
 * only; outputs must not overlap each other or any input. The launch lets the
 * next launch on the stream begin streaming its weights while this one
 * finishes (programmatic dependent launch); x is read and y written only
 * after the previous work on the stream has completed, so the usual stream
 * order holds for every input and output. */
W4_API w4_status w4r_matmul_grouped(const w4r_desc* descs, int32_t count, void* stream);
W4_API w4_status w4r_matmul(const w4r_desc* d, void* stream);

/* ------------------------------------------------------------------ tile layout (prefill) */

/* The tile layout of one W4 weight, read by the tensor-core tile GEMM: the
 * page-format nibbles, scales and zero points ("ONNX export, quantization and
 * the browser runtime", section "Quantization (train/quantize.py)", step 2)
 * reordered once at load time, nothing rounded (w4t_repack_restore gives the
 * page buffers back bit for bit). K % 32 == 0, N % 8 == 0, K <= 2^24,
 * N <= 2^23; tiles of 128 columns (the last padded with zero weights) in
 * column order, each K / 32 blocks of 2624 bytes:
 *   block b of tile T: [0, 2048) column c (0..127) at c * 16, four words;
 *     word j holds rows 32 b + 8 j + r (r = 0..7) of column 128 T + c with
 *     row r in bits {0-3, 16-19, 4-7, 20-23, 8-11, 24-27, 12-15, 28-31}[r];
 *   [2048, 2560) the block's scales, column c at 2048 + 4 c;
 *   [2560, 2624) its zero points packed as the page packs them (word w:
 *     columns 8 w .. 8 w + 7, nibble i = column 8 w + i).
 * w4t_repacked_bytes() is the size (the page-format total when N % 128 == 0;
 * 0 for a shape the layout does not take). Repack and restore: as
 * w4_repack / w4_repack_restore (device buffers, 16-byte aligned,
 * asynchronous). */
W4_API size_t w4t_repacked_bytes(int64_t K, int64_t N);
W4_API w4_status w4t_repack(const uint8_t* qw, const float* scales, const uint8_t* zp, int64_t K, int64_t N,
                            void* wt, void* stream);
W4_API w4_status w4t_repack_restore(const void* wt, int64_t K, int64_t N, uint8_t* qw, float* scales, uint8_t* zp,
                                    void* stream);

/* Matmuls y = act(x . W + bias) + residual on weights in the tile layout, for
 * any M (built for prefill, M > 16), on the tensor cores. Per K-block the
 * weights' (q - zp) are exact in bf16; each x is split exactly into three
 * bf16 pieces (x = p0 + p1 + p2, 8 + 8 + 8 significant bits), so every
 * product is exact; tcgen05.mma sums a block's products in fp32 and the
 * block's scale is applied in fp32 (y += s * sum). Non-finite x give NaN.
 * - descs: HOST array of w4t_desc (the w4r_desc fields; wr = the tile-layout
 *   weight), read during the call only. Any M >= 0 up to 131072, K % 32 == 0,
 *   N % 8 == 0, ldx >= K, ldy >= N, ldr >= N when residual is set; x / y /
 *   bias / residual 4-byte aligned, wr 16-byte aligned. K = 0 writes the
 *   epilogue of 0. Outputs must not overlap each other or any input.
 * - workspace: device memory of at least w4t_workspace_size(descs, count)
 *   bytes, 16-byte aligned (NULL when that is 0); it receives the pieces of
 *   each distinct x (same x pointer, ldx, M and K share them) and needs no
 *   zeroing. Calls that may run at the same time must not share it.
 * - The pieces are written by one launch, then the tile GEMM runs (a second
 *   launch per class of rows-per-tile: 16, 32, 64 or 128 by M); both start
 *   early on the stream (programmatic dependent launch) and read x, bias and
 *   the residual and write y only after the previous work on the stream has
 *   completed. */
typedef w4r_desc w4t_desc;
W4_API size_t w4t_workspace_size(const w4t_desc* descs, int32_t count);
W4_API w4_status w4t_matmul_grouped(const w4t_desc* descs, int32_t count, void* workspace, size_t workspace_bytes,
                                    void* stream);
W4_API w4_status w4t_matmul(const w4t_desc* d, void* workspace, size_t workspace_bytes, void* stream);

/* Decode matmuls (one row of x) on weights in the tile layout, on the tensor
 * cores with integer MMAs: y[1, N] = act(x[1, K] . W + bias) + residual.
 * x is written in fixed point against its largest magnitude, as 8 signed
 * 7-bit digits per element (exact for every element within 2^31 of the
 * largest, within 2^-55 of it otherwise); the MMA multiplies the digits by
 * the stored codes q exactly in int32, the zero point enters exactly as
 * D - zp * (block sum of the digits), and each block's integer sums are
 * weighed and scaled by s in fp32 and summed over the blocks in fp32.
 * Non-finite x give NaN.
 * - descs: HOST array of w4t_desc (wr = the tile-layout weight), read during
 *   the call only. M must be 1 (0 skips the descriptor), K % 32 == 0,
 *   K <= 3072, N % 8 == 0; x / y / bias / residual 4-byte aligned, wr
 *   16-byte aligned; ldx / ldy / ldr are not used. K = 0 writes the
 *   epilogue of 0. Outputs must not overlap each other or any input.
 * - workspace: device memory of at least w4i_workspace_size(descs, count)
 *   bytes (about 8.5 K per distinct x), 16-byte aligned; it receives the
 *   digits of each distinct x and needs no zeroing. Calls that may run at the
 *   same time must not share it.
 * - The digits are written by one launch, then the GEMV runs (a second
 *   launch); both start early on the stream (programmatic dependent launch)
 *   and read x, bias and the residual and write y only after the previous
 *   work on the stream has completed. */
W4_API size_t w4i_workspace_size(const w4t_desc* descs, int32_t count);
W4_API w4_status w4i_matmul_grouped(const w4t_desc* descs, int32_t count, void* workspace, size_t workspace_bytes,
                                    void* stream);
W4_API w4_status w4i_matmul(const w4t_desc* d, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------ head */

/* Bytes of workspace i8_head_logits needs for this shape on the current
 * device (same rules as w4_matmul's workspace: zero-filled before first use,
 * counter block left zero by every successful call, not shared by calls that may run
 * at the same time). One workspace of the larger size can serve both ops on
 * one stream. */
W4_API size_t i8_head_workspace_size(int64_t M, int64_t K, int64_t V);

/* logits[M, V] = h[M, K] . (T[K, V] * s[V]); the M rows of h are the last
 * positions of M sequences (pass h = hidden + (T_len - 1) * ldh for one
 * sequence). Requires ldh >= K, ldt >= V, ldl >= V, h / scales / logits
 * 4-byte aligned, table 16-byte aligned. workspace may be NULL only when
 * i8_head_workspace_size() returns 0. */
W4_API w4_status i8_head_logits(const float* h, int64_t ldh, const int8_t* table, int64_t ldt,
                                const float* scales, float* logits, int64_t ldl, int64_t M, int64_t K,
                                int64_t V, void* workspace, size_t workspace_bytes, void* stream);

/* As i8_head_logits with an explicit kernel choice (AUTO, GEMV or GENERIC;
 * the GENERIC kernel needs no workspace). */
W4_API w4_status i8_head_logits_path(const float* h, int64_t ldh, const int8_t* table, int64_t ldt,
                                     const float* scales, float* logits, int64_t ldl, int64_t M,
                                     int64_t K, int64_t V, void* workspace, size_t workspace_bytes,
                                     w4_path path, void* stream);

/* The streaming layout of the int8 head: the page's table bytes and scales
 * ("ONNX export, quantization and the browser runtime", section
 * "Quantization (train/quantize.py)", step 3) reordered once at load time
 * into the order in which the M = 1 head GEMV streams them, one contiguous
 * run of bytes per warp, and biased to unsigned (code XOR 0x80). Nothing is
 * rounded: i8_head_repack_restore gives back the page's table and scales
 * exactly.
 *
 * Layout, K % 16 == 0, nb = K / 16, gs = 32 / gcd(nb, 32), A = gs * nb / 32:
 * groups of 8 gs token columns (all K rows) in column order; a group is A
 * rounds of 4096 bytes followed by its 8 gs scales (fp32). In round r of
 * group G, lane l owns strip s = l % gs (columns c0 = 8 (G gs + s) ..
 * c0 + 7) and block b = l / gs + r * (32 / gs) (rows 16 b .. 16 b + 15);
 * the byte of row 16 b + 2 c + e, column c0 + 4 h + i sits at
 * c * 512 + l * 16 + (2 e + h) * 4 + i. Columns at or past V hold code 0 and
 * scale 0. i8_head_repacked_bytes() is the size (0 for a shape the layout
 * does not take: K % 16 != 0, K > 8192, V < 1). */
W4_API size_t i8_head_repacked_bytes(int64_t K, int64_t V);

/* Page format (table [K, V] with row stride ldt >= V, any alignment;
 * scales [V] fp32, 4-byte aligned) -> streaming layout tr
 * (i8_head_repacked_bytes(K, V) bytes, 16-byte aligned), on the GPU. */
W4_API w4_status i8_head_repack(const int8_t* table, int64_t ldt, const float* scales, int64_t K, int64_t V,
                                void* tr, void* stream);

/* Streaming layout -> page format (the exact inverse of i8_head_repack). */
W4_API w4_status i8_head_repack_restore(const void* tr, int64_t K, int64_t V, int8_t* table, int64_t ldt,
                                        float* scales, void* stream);

/* logits[v] = s_v * sum_k h[k] T[k, v] for ONE last-position row h (K fp32,
 * 16-byte aligned) on a repacked head; logits: V fp32, 4-byte aligned, fully
 * overwritten. No workspace. Like w4r_matmul_grouped, the launch may start
 * streaming the table before the previous work on the stream has finished;
 * h is read and the logits written only after it has. */
W4_API w4_status i8r_head_logits(const float* h, const void* tr, int64_t K, int64_t V, float* logits,
                                 void* stream);

/* Greedy decoding on a repacked head: *token = argmax_v of exactly the
 * logits i8r_head_logits computes (ties to the lowest id; -0 equals +0),
 * *best_logit (may be NULL) = that logit; the logits are not written. keys:
 * 8 bytes of device memory (8-byte aligned) that the call clears and uses. */
W4_API w4_status i8r_head_argmax(const float* h, const void* tr, int64_t K, int64_t V, int32_t* token,
                                 float* best_logit, void* keys, void* stream);

/* One decode step in one launch: the matmuls of `descs` (as
 * w4r_matmul_grouped: repacked weights, M = 1) and the int8 head's logits
 * (as i8r_head_logits: logits[v] = s_v * sum_k h_k T[k, v] on the head in its
 * streaming layout), streamed by the same persistent CTAs, each of which takes
 * an equal share of the head's column groups and of the body's bytes (the
 * head's first), so that the step pays one launch's start and tail ("ONNX export, quantization and the
 * browser runtime", section "Quantization (train/quantize.py)", steps 2 to
 * 4). Every output is bit-identical to the two separate calls.
 * - descs / count: as for w4r_matmul_grouped (a HOST array, read during the
 *   call only; count may be 0).
 * - h, tr, K, V, logits: as for i8r_head_logits. h is read when the launch
 *   starts, so it must not overlap any y of `descs` (W4_ERR_VALUE): within a
 *   step the head's input is not one of the body's outputs.
 * - A step that one launch cannot hold (more than 128 weights, K of the head
 *   above 2048, or more x than a CTA stages) runs as the body's launches
 *   followed by the head's, with the same results.
 * - The launch starts streaming while the previous work on the stream
 *   finishes (programmatic dependent launch); x and h are read and y and the
 *   logits written only after that work has completed. */
W4_API w4_status w4r_decode_step(const w4r_desc* descs, int32_t count, const float* h, const void* tr, int64_t K,
                                 int64_t V, float* logits, void* stream);

/* The same step with greedy decoding instead of the logits (as
 * i8r_head_argmax): *token = argmax_v of exactly the logits w4r_decode_step
 * computes (ties to the lowest id; -0 equals +0), *best_logit (may be NULL)
 * = that logit; the logits are not written. keys: 8 bytes of device memory
 * (8-byte aligned) that the call clears and uses. One launch for the step
 * and one small launch that turns the key into the token. */
W4_API w4_status w4r_decode_step_argmax(const w4r_desc* descs, int32_t count, const float* h, const void* tr,
                                        int64_t K, int64_t V, int32_t* token, float* best_logit, void* keys,
                                        void* stream);

/* The tile layout of the int8 head, read by the tensor-core head
 * (i8t_head_logits / i8t_head_argmax) for 1 to 8 last-position rows. The
 * page's table bytes and scales ("ONNX export, quantization and the browser
 * runtime", section "Quantization (train/quantize.py)", step 3) reordered
 * once at load time into the tensor core's int8 operand layout; nothing is
 * changed or rounded: i8t_head_repack_restore gives back the page's table
 * and scales exactly.
 *
 * Layout, K % 32 == 0, 32 <= K <= 1024: tiles of 128 tokens in token order,
 * each K / 32 units of 4096 bytes and then the tile's 128 scales (fp32). In
 * unit u of tile t the code of row 32 u + 16 h + i (h in 0..1, i in 0..15)
 * and token 128 t + c sits at byte (c / 8) * 256 + h * 128 + (c % 8) * 16 + i;
 * the scale of token 128 t + c at byte K * 128 + 4 c of the tile. Tokens at
 * or past V hold code 0 and scale 0. i8t_head_repacked_bytes() is the size
 * (0 for a shape the layout does not take). */
W4_API size_t i8t_head_repacked_bytes(int64_t K, int64_t V);

/* Page format (table [K, V] with row stride ldt >= V, any alignment;
 * scales [V] fp32, 4-byte aligned) -> tile layout (i8t_head_repacked_bytes
 * bytes, 16-byte aligned), on the GPU. W4_ERR_SHAPE for a shape the layout
 * does not take. */
W4_API w4_status i8t_head_repack(const int8_t* table, int64_t ldt, const float* scales, int64_t K, int64_t V,
                                 void* tiles, void* stream);

/* Tile layout -> page format (the exact inverse of i8t_head_repack). */
W4_API w4_status i8t_head_repack_restore(const void* tiles, int64_t K, int64_t V, int8_t* table, int64_t ldt,
                                         float* scales, void* stream);

/* logits[m, v] = s_v * sum_k h[m, k] T[k, v] for M <= 8 last-position rows
 * h [M, K] (row stride ldh >= K when M > 1, 4-byte aligned) on a head in the
 * tile layout; logits [M, V] with row stride ldl >= V when M > 1, 4-byte
 * aligned, fully overwritten. The tensor cores multiply the codes by h
 * written per row in fixed point (8 signed 7-bit digits against the row's
 * largest magnitude: exact for every element within 2^31 of it, within
 * 2^-55 of it otherwise) with exact integer sums, and the digits are weighed
 * and scaled in fp64: each logit is the dot product rounded about once, and
 * deterministic. A row holding an Inf or NaN gives NaN logits. No workspace.
 * The launch may start streaming the table before the previous work on the
 * stream has finished; h is read and the logits written only after it has.
 * W4_ERR_SHAPE for M > 8 or a shape the layout does not take; M = 0 or
 * V = 0 is a no-op. */
W4_API w4_status i8t_head_logits(const float* h, int64_t ldh, const void* tiles, int64_t K, int64_t V, int64_t M,
                                 float* logits, int64_t ldl, void* stream);

/* Greedy decoding with the tensor-core head: tokens[m] = argmax_v of exactly
 * the logits i8t_head_logits computes (ties to the lowest id; -0 equals +0),
 * best_logits[m] (may be NULL) = that logit; the logits are not written.
 * keys: 8 M bytes of device memory (8-byte aligned) that the call clears and
 * uses. tokens / best_logits: M entries on the device. */
W4_API w4_status i8t_head_argmax(const float* h, int64_t ldh, const void* tiles, int64_t K, int64_t V, int64_t M,
                                 int32_t* tokens, float* best_logits, void* keys, void* stream);

/* Greedy decoding on the head: tokens[m] = argmax_v logits[m, v] (ties to
 * the lowest token id), best_logits[m] = that logit when best_logits is not
 * NULL; the logits are exactly those i8_head_logits computes. The pages
 * measure greedy decoding ("ONNX export, quantization and the browser
 * runtime", section "Quantization (train/quantize.py)", measurements: 32
 * greedy tokens); folding the argmax into the head avoids writing and
 * re-reading the [M, V] logits. tokens / best_logits: device, M entries.
 * workspace: i8_head_argmax_workspace_size() bytes, 16-byte aligned, with
 * the same rules as the other workspaces (zero-filled before first use; every
 * successful call leaves its leading counter block zero); other rules as
 * i8_head_logits. */
W4_API size_t i8_head_argmax_workspace_size(int64_t M, int64_t K, int64_t V);
W4_API w4_status i8_head_argmax(const float* h, int64_t ldh, const int8_t* table, int64_t ldt,
                                const float* scales, int64_t M, int64_t K, int64_t V, int32_t* tokens,
                                float* best_logits, void* workspace, size_t workspace_bytes, void* stream);

/* Token lookup from the tied int8 table: out[i, k] = T[k, tokens[i]] *
 * s[tokens[i]] (fp32, one rounding per element). "ONNX export, quantization
 * and the browser runtime", section "Quantization (train/quantize.py)",
 * step 3: the tied table is stored once, [K, V], and the lookup is
 * Gather(axis=1) + Transpose on it, dequantized. tokens is a DEVICE int32
 * array of ntok ids; out is device fp32 [ntok, ldo] with ldo >= K, fully
 * overwritten. A token id outside [0, V) makes its row zero and records
 * W4_ERR_VALUE in the device error word (read with w4_device_error). Table
 * 1-byte aligned (any ldt >= V), scales / out 4-byte aligned. */
W4_API w4_status i8_embed_lookup(const int8_t* table, int64_t ldt, const float* scales, const int32_t* tokens,
                                 int64_t ntok, float* out, int64_t ldo, int64_t K, int64_t V, void* stream);

/* ------------------------------------------------------------------ quantisers */

/* Scale storage of w4_quantize: fp32 (the shipped format, the one every
 * matmul here reads) or fp16 (the "fp16 scales" variant the page measures;
 * widen it to fp32, exactly, before a matmul). */
typedef enum w4_scale_type { W4_SCALE_F32 = 0, W4_SCALE_F16 = 1 } w4_scale_type;

/* The export's dq4 step ("ONNX export, quantization and the browser
 * runtime", section "Quantization (train/quantize.py)", step 2) on the GPU:
 * w [K, N] fp32 (row stride ldw >= N, 4-byte aligned, finite values) ->
 *   qw [K*N/2] packed nibbles (flat [K, N] order, low nibble first),
 *   scales [K/block, N] (fp32, or fp16 with W4_SCALE_F16; aligned to the
 *   element size), zp [(K/block)*N/2] packed nibbles.
 * block is 32 (the shipped format) or 64 (the group size of the page's MLX
 * comparison); K % block == 0 and N even (else W4_ERR_SHAPE / W4_ERR_VALUE).
 * The page gives no formula; this is the min/max reading, in fp64 with one
 * rounding per division: lo = min(min w, 0) and hi = max(max w, 0) over the
 * block of one column; s = (hi - lo) / 15 rounded once to the stored type;
 * a stored s of 0 becomes s = 1, zp = 0; zp = rint(-lo / s) and
 * q = rint(w / s) + zp, clamped to 0..15, rint rounding half to even.
 * Buffers are the caller's device memory; the call is asynchronous and
 * stream-ordered. */
W4_API w4_status w4_quantize(const float* w, int64_t ldw, int64_t K, int64_t N, int32_t block, int32_t scale_type,
                             uint8_t* qw, void* scales, uint8_t* zp, void* stream);

/* The export's embedding_int8 step (same section, step 3) on the GPU:
 * w [K, V] fp32 (row stride ldw >= V) -> table [K, V] int8 (row stride
 * ldt >= V) and scales [V] fp32, one per token (column): in fp64,
 * s = max|w| / 127 rounded once to fp32 (an all-zero column takes s = 1),
 * q = rint(w / s) clamped to -127..127. */
W4_API w4_status i8_quantize_head(const float* w, int64_t ldw, int64_t K, int64_t V, int8_t* table, int64_t ldt,
                                  float* scales, void* stream);

/* ------------------------------------------------------------------ host packing */

/* Pack n uint4 values (each 0..15) into (n + 1) / 2 bytes, low nibble first;
 * an odd n leaves the last high nibble 0. Host memory. W4_ERR_VALUE if a
 * value exceeds 15 (nothing is written then). */
W4_API w4_status w4_pack_nibbles(const uint8_t* q, int64_t n, uint8_t* out);

/* Unpack the first n nibbles of `packed` (host memory) into q[n]. */
W4_API w4_status w4_unpack_nibbles(const uint8_t* packed, int64_t n, uint8_t* q);

/* ------------------------------------------------------------------ diagnostics */

W4_API const char* w4_status_string(w4_status s);

/* One-line reason for the last non-OK status returned on this host thread. */
W4_API const char* w4_last_error(void);

/* SYNCHRONOUS. Reads the current device's error word, which a kernel sets
 * when one of its bounded waits runs out (kernels never trap, assert or spin
 * without limit). info (may be NULL) receives {status, kernel id, block
 * index, detail}. With clear != 0 the word is reset to 0. Returns the
 * recorded status (W4_OK if none) or W4_ERR_CUDA if the read itself failed. */
W4_API w4_status w4_device_error(int32_t* info4, int32_t clear);

/* Limit of every bounded device wait, in nanoseconds (default 2e9). */
W4_API w4_status w4_set_wait_timeout_ns(uint64_t ns);

/* Launches a kernel that waits, through the same bounded-wait code the
 * matmul kernels use, on a barrier nothing ever completes, with the given
 * limit. It records W4_ERR_TIMEOUT in the device error word and returns;
 * used to test the timeout path without hanging a GPU. */
W4_API w4_status w4_debug_wait_timeout(uint64_t timeout_ns, void* stream);

W4_API int32_t w4_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* W4_B200_H */
