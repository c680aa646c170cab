/*
 * qgemm.h -- C ABI of the B200 (sm_100a) FP4 quantized linear layer.
 *
 * The layer is the forward pass of the FP4 training method summarised in the
 * QbitAI write-up "微软首创FP4训练框架，训练效果媲美BF16" (news.movedaos.com/post/4103;
 * arXiv 2501.17116, "Optimizing Large Language Model Training Using FP4
 * Quantization"), cited below as [FP4-writeup] with the paragraph:
 *
 *     Y = dequant( Q(A_clamped) . Q(W) ) + dA . W
 *
 *   A  (M x K, row-major, tokens x in-features), fp32 or bf16
 *   W  (K x N, row-major), fp32 or bf16
 *   Q  E2M1 FP4 codes {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6}
 *      ([FP4-writeup], E2M1 paragraph), one fp32 scale per row of A
 *      (token-wise) and per column of W (channel-wise) ([FP4-writeup],
 *      granularity paragraph), ScaleShift calibration r = 6/amax, s = amax/6,
 *      round to nearest, ties to the even code ([FP4-writeup], ScaleShift
 *      paragraph)
 *   A_clamped = clamp(A, -T, T), T = the alpha-quantile of |A| over the whole
 *      tensor (order statistic of rank ceil(alpha * M * K) - 1), and the sparse
 *      compensation dA = A - A_clamped ([FP4-writeup], outlier clamping and
 *      compensation paragraph)
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers, owned by the caller; the
 *     library allocates no device memory.  Calls are asynchronous on the
 *     given stream; argument checks happen on the host before anything is
 *     enqueued, and a failed check enqueues nothing.
 *   - Packed codes hold two 4-bit codes per byte, the even k in the low
 *     nibble; code bit 3 is the sign, bits 2..0 index the magnitude grid.
 *     Row codes of A are M x K/2 bytes; column codes of W are stored
 *     transposed, N x K/2 bytes, so both GEMM operands have K contiguous.
 *   - Shapes: K % 32 == 0 and 0 < K <= 16384 (else QG_ERR_UNSUPPORTED_SHAPE);
 *     M, N >= 1 arbitrary.  Row strides (lda, ldw) are in elements, at least
 *     the row length; lda keeps every row start of A 16-byte aligned (checked).
 *     ldw may be any value >= N: rows of W that are not 16-byte multiples
 *     are read element by element (slower).  Base pointers are 16-byte
 *     aligned.
 *   - Workspace: calls that take (ws, ws_bytes) use a caller-allocated device
 *     buffer of at least qg_workspace_size(...) bytes, 256-byte aligned.  Its
 *     first bytes hold a sticky device status word; initialise a new
 *     workspace once with qg_workspace_init().  Calls on one workspace must
 *     not overlap in time (use one stream, or one workspace per stream).
 *   - Errors: nothing aborts, traps or throws.  Host-side argument errors are
 *     returned immediately.  Device-side conditions (non-finite input, a
 *     bounded wait that timed out, an internal capacity overflow) set bits in
 *     the status word; qg_sync_status() synchronises the stream, returns the
 *     condition and clears it.
 *   - Environment: QGEMM_NO_COOPERATIVE=1 (read when the library first sets up
 *     a device) makes it use the multi-kernel sequences of the bf16 activation
 *     and column quantizers instead of their single cooperative kernels: the
 *     same results, slower; meant for testing those paths.
 *   - Inputs must be finite.  Calls that scan all of A for the threshold
 *     (quantize_act, clamp_compensate, fp4_linear) report NaN/Inf as
 *     QG_ERR_NONFINITE; the other calls give unspecified codes for them.
 */
#ifndef QGEMM_H
#define QGEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same definition as the CUDA runtime's; 0 / NULL is the legacy stream. */
typedef struct CUstream_st* cudaStream_t;

typedef enum { QG_F32 = 0, QG_BF16 = 1 } qg_dtype;

typedef enum {
    QG_OK = 0,
    QG_ERR_INVALID_ARG = 1,       /* null pointer, bad stride, alpha out of (0, 1], ... */
    QG_ERR_UNSUPPORTED_SHAPE = 2, /* K % 32 != 0, K > 16384, non-positive sizes */
    QG_ERR_WORKSPACE = 3,         /* workspace missing, misaligned or too small */
    QG_ERR_CUDA = 4,              /* a CUDA runtime call failed (launch, no device, ...) */
    QG_ERR_NONFINITE = 5,         /* NaN or Inf found in A (device-side) */
    QG_ERR_TIMEOUT = 6,           /* a bounded device wait gave up (device-side) */
    QG_ERR_INTERNAL = 7           /* device-side capacity check failed */
} qg_status;

/* CSR form of dA (device arrays, caller-owned).  Rows ascending, columns
 * ascending within a row; val holds a - sign(a) * T in double (exact for
 * bf16 input).  nnz_capacity must be at least qg_nnz_capacity(M * K, alpha);
 * *nnz_out (device int64) receives the count. */
typedef struct {
    int32_t* row_ptr;     /* M + 1 */
    int32_t* col;         /* nnz_capacity */
    double* val;          /* nnz_capacity */
    int64_t nnz_capacity;
    int64_t* nnz_out;     /* device, 1 element */
} qg_csr;

/* Which call a workspace is sized for. */
typedef enum {
    QG_OP_QUANTIZE_ROWS = 0,
    QG_OP_QUANTIZE_COLS = 1,
    QG_OP_CLAMP_COMPENSATE = 2,
    QG_OP_QUANTIZE_ACT = 3,
    QG_OP_SPMM = 4,
    QG_OP_FP4_GEMM = 5,
    QG_OP_FP4_LINEAR = 6,
    QG_OP_FP4_DGRAD = 7,    /* sized with (M, K, N) of the forward layer */
    QG_OP_FP4_WGRAD = 8,    /* sized with (M, K, N) of the forward layer */
    QG_OP_FP4_GEMM_COMPENSATED = 9
} qg_op;

const char* qg_status_string(qg_status s);
const char* qg_version(void);

/* Number of kernel launches this library has enqueued in this process (all
 * devices, all streams); graph replays of captured launches are not counted. */
uint64_t qg_launch_count(void);

/* Rank of the threshold in sorted |A|: ceil(alpha * n) - 1 evaluated in
 * double, clamped to [0, n - 1].  ([FP4-writeup], outlier paragraph; the
 * order-statistic reading of "quantile".) */
int64_t qg_quantile_rank(double alpha, int64_t n);

/* Upper bound on the clamped entries: n - (qg_quantile_rank(alpha, n) + 1). */
int64_t qg_nnz_capacity(int64_t n, double alpha);

/* Bytes of workspace that `op` needs for these sizes (N is ignored by the
 * activation-only calls; alpha by the calls without a threshold).  Always a
 * multiple of 256 and at least 256. */
size_t qg_workspace_size(qg_op op, int64_t M, int64_t K, int64_t N, qg_dtype dtype,
                         double alpha);

/* Zero the workspace's status word and counters (enqueued on `stream`). */
qg_status qg_workspace_init(void* ws, size_t ws_bytes, cudaStream_t stream);

/* Synchronise `stream`, then return and clear the workspace's device status
 * (QG_OK when nothing was flagged; QG_ERR_CUDA when the stream had failed). */
qg_status qg_sync_status(void* ws, cudaStream_t stream);

/* Elementwise E2M1 encoding ([FP4-writeup], E2M1 + ScaleShift paragraphs,
 * rounding only, no scaling): x (n fp32, n even) -> packed (n/2 bytes). */
qg_status qg_e2m1_encode(const float* x, int64_t n, uint8_t* packed, void* ws,
                         size_t ws_bytes, cudaStream_t stream);

/* Token-wise (row) quantization of A without clamping ([FP4-writeup],
 * granularity + ScaleShift paragraphs).  amax_i = max_k |A_ik|;
 * r_i = fp32(6 / amax_i), s_i = fp32(amax_i / 6) (both 0 when amax_i is 0 or
 * 6 / amax_i overflows); codes_ik = E2M1(fp32(A_ik * r_i)).
 * A: M x K (stride lda elements) -> codes M x K/2, scales M (fp32). */
qg_status qg_quantize_rows(const void* A, qg_dtype dtype, int64_t M, int64_t K, int64_t lda,
                           uint8_t* codes, float* scales, void* ws, size_t ws_bytes,
                           cudaStream_t stream);

/* Channel-wise (column) quantization of W ([FP4-writeup], granularity
 * paragraph), same arithmetic as qg_quantize_rows over the columns of W.
 * W: K x N (stride ldw elements) -> codesT N x K/2 (transposed), scales N. */
qg_status qg_quantize_cols(const void* W, qg_dtype dtype, int64_t K, int64_t N, int64_t ldw,
                           uint8_t* codesT, float* scales, void* ws, size_t ws_bytes,
                           cudaStream_t stream);

/* The same computation as qg_quantize_cols, for callers that cannot
 * allocate device memory: code running under a fixed memory plan (an
 * inference engine that has handed all device memory to its own pool and
 * forbids further allocation while serving), or code that must not call
 * cudaMalloc because it synchronises the device.  No workspace is taken and
 * nothing is allocated: the column maxima live in a fixed array inside the
 * library, sized for N <= 65536 columns (256 KB, held on every GPU that loads
 * the library until the process exits).  The pages have no counterpart for
 * this entry point; it is a deployment convenience.
 *   - N > 65536 returns QG_ERR_UNSUPPORTED_SHAPE before anything is enqueued;
 *     other argument checks are those of qg_quantize_cols.
 *   - The first call on a device looks up the array's device address (a CUDA
 *     runtime query); make that first call before any stream capture.  The
 *     address is kept for the life of the process: after a cudaDeviceReset
 *     it is stale, so do not call this entry point again after a reset.
 *   - For either dtype it runs the two-pass kernels (column maxima, then the
 *     codes) rather than the single cooperative bf16 kernel of
 *     qg_quantize_cols: same results, 12-22 % slower on bf16 weights
 *     (measured on a B200 from 2048 x 5504 to 4096 x 22016).
 *   - Every call on a GPU uses that GPU's one array and zeroes what it needs
 *     at the start; it keeps the last call's contents in between.  Calls
 *     whose executions overlap on the same GPU (for example on two streams)
 *     race on it: serialise them. */
qg_status qg_quantize_cols_static(const void* W, qg_dtype dtype, int64_t K, int64_t N,
                                  int64_t ldw, uint8_t* codesT, float* scales,
                                  cudaStream_t stream);

/* Outlier clamping and compensation ([FP4-writeup], outlier paragraph):
 * T = alpha-quantile of |A| (whole tensor), A_clamped = clamp(A, -T, T) in the
 * input dtype (M x K, contiguous, may be NULL), dA in CSR, T_out (device fp32,
 * 1 element).  0 < alpha <= 1. */
qg_status qg_clamp_compensate(const void* A, qg_dtype dtype, int64_t M, int64_t K, int64_t lda,
                              double alpha, void* A_clamped, const qg_csr* dA, float* T_out,
                              void* ws, size_t ws_bytes, cudaStream_t stream);

/* Fused activation quantizer: threshold, clamp, dA (CSR) and token-wise
 * quantization of A_clamped (amax_i = min(max_k |A_ik|, T)), in two passes
 * over A for bf16 input (one cooperative launch) and three for fp32
 * ([FP4-writeup], outlier + granularity + ScaleShift paragraphs).
 * Outputs as qg_quantize_rows plus dA and T_out. */
qg_status qg_quantize_act(const void* A, qg_dtype dtype, int64_t M, int64_t K, int64_t lda,
                          double alpha, uint8_t* codes, float* scales, const qg_csr* dA,
                          float* T_out, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Compensation product C = dA . W (M x N, fp32, fully written), products and
 * sums in fp32 with W in its stored dtype ([FP4-writeup], outlier paragraph:
 * the compensation is kept in higher precision).  W: K x N, stride ldw. */
qg_status qg_spmm_correction(const qg_csr* dA, int64_t M, const void* W, qg_dtype w_dtype,
                             int64_t K, int64_t N, int64_t ldw, float* C, void* ws,
                             size_t ws_bytes, cudaStream_t stream);

/* The compensation added into an existing fp32 output ([FP4-writeup],
 * outlier clamping and compensation paragraph): Y += dA . W (M x N,
 * row pitch N), with each row's sum formed as in qg_spmm_correction (fp32
 * FMA chain in CSR order) and then added to Y by the memory system
 * (red.global.add: fp32 round to nearest; a sum that is subnormal is
 * flushed to zero).  Rows of dA without entries leave Y untouched.  With Y
 * holding qg_fp4_gemm's output without C, the result is the layer's Y.
 * Same arguments and errors as qg_spmm_correction. */
qg_status qg_spmm_accumulate(const qg_csr* dA, int64_t M, const void* W, qg_dtype w_dtype,
                             int64_t K, int64_t N, int64_t ldw, float* Y, void* ws,
                             size_t ws_bytes, cudaStream_t stream);

/* FP4 GEMM on tcgen05 tensor cores ([FP4-writeup], FP4 GEMM paragraph, with
 * the row and column scales of the granularity paragraph applied after the
 * contraction): acc_ij = sum_k e2m1(codesA_ik) *
 * e2m1(codesWT_jk) accumulated in fp32 (exact for K <= 16384), then
 * Y_ij = acc_ij * sA_i * sW_j (+ C_ij when C != NULL), stored as fp32 or bf16
 * (round to nearest even).  raw_acc (nullable, M x N fp32) receives acc itself.
 * Y may be NULL when only raw_acc is wanted.  C may be the same memory as an
 * fp32 Y (Y += the scaled product, in place): every element of C is read
 * before the same element of Y is written. */
qg_status qg_fp4_gemm(const uint8_t* codesA, const float* sA, const uint8_t* codesWT,
                      const float* sW, int64_t M, int64_t N, int64_t K, const float* C,
                      void* Y, qg_dtype y_dtype, float* raw_acc, void* ws, size_t ws_bytes,
                      cudaStream_t stream);

/* The FP4 GEMM's scaled product added into an existing fp32 output
 * ([FP4-writeup], FP4 GEMM paragraph; the sum with the compensation of the
 * outlier paragraph): Y_ij += acc_ij * sA_i * sW_j (the product rounded to fp32 as in qg_fp4_gemm,
 * then added by the memory system's bulk reduction, fp32 round to nearest).
 * Y: M x N fp32, contiguous, N a multiple of 4 (else
 * QG_ERR_UNSUPPORTED_SHAPE).  With Y holding qg_spmm_correction's output,
 * the result is the layer's Y.  Workspace and other arguments as
 * qg_fp4_gemm. */
qg_status qg_fp4_gemm_accumulate(const uint8_t* codesA, const float* sA, const uint8_t* codesWT,
                                 const float* sW, int64_t M, int64_t N, int64_t K, float* Y,
                                 void* ws, size_t ws_bytes, cudaStream_t stream);

/* The compensated FP4 GEMM, the layer's product in one kernel:
 *   Y_ij = acc_ij * sA_i * sW_j + sum over the entries (i, k) of dA of
 *          dA_ik * W_kj
 * ([FP4-writeup], FP4 GEMM + outlier clamping and compensation paragraphs),
 * with acc the FP4 product as in qg_fp4_gemm and the compensation summed in
 * fp32 (one fused multiply-add per entry, in the row's CSR order, W read in
 * its stored dtype): the same arithmetic as qg_spmm_correction followed by
 * qg_fp4_gemm with that C, bit for bit, but the compensation is computed by
 * extra warps of the GEMM kernel while the tensor cores run, tile by tile, and
 * no M x N correction matrix is written to or read from memory.
 *   dA: CSR over M rows with column indices < K (as qg_quantize_act leaves it);
 *   W: K x N, row pitch ldw >= N elements, 16-byte aligned, dtype w_dtype;
 *   Y: M x N, fp32 or bf16 (y_dtype), contiguous.
 * Workspace: qg_workspace_size(QG_OP_FP4_GEMM_COMPENSATED, M, K, N, any, 1.0)
 * (a fixed ~37 MB of scratch slots: two 128 x 224 fp32 tiles per CTA).
 * Errors as qg_fp4_gemm. */
qg_status qg_fp4_gemm_compensated(const uint8_t* codesA, const float* sA, const uint8_t* codesWT,
                                  const float* sW, int64_t M, int64_t N, int64_t K,
                                  const qg_csr* dA, const void* W, qg_dtype w_dtype, int64_t ldw,
                                  void* Y, qg_dtype y_dtype, void* ws, size_t ws_bytes,
                                  cudaStream_t stream);

/* The whole layer into Y (M x N, fp32 or bf16), Y = dequant(Q(A_clamped)
 * Q(W)) + dA . W ([FP4-writeup], outlier clamping and compensation, FP4
 * GEMM and granularity paragraphs): qg_quantize_act(A), then
 *   fp32 Y: qg_spmm_correction(dA, W) written into Y itself, then
 *           qg_fp4_gemm_accumulate adding the scaled FP4 product into it (for
 *           N not a multiple of 4: qg_fp4_gemm(..., C = Y, Y) in place, the
 *           epilogue reading every sub-tile of C before it writes that
 *           sub-tile of Y); or, when alpha leaves at least 10 clamped entries
 *           per row possible for every 4096 of K (n - ceil(alpha n) >=
 *           10 M K / 4096), the other order:
 *           qg_fp4_gemm(..., C = NULL, Y), then qg_spmm_accumulate;
 *   bf16 Y: the rows in chunks of R (the largest multiple of 256 with
 *           R x N x 4 <= 128 MiB, but at least 256 -- more bytes only when
 *           N > 131072 -- and at most M): qg_spmm_correction of the chunk
 *           into an fp32
 *           scratch of R x N in the workspace, then qg_fp4_gemm(..., C =
 *           scratch, the chunk of Y) -- the same bytes as
 *           qg_fp4_gemm_compensated, which computes the compensation inside
 *           the GEMM kernel but runs 1.3-3.8x slower at the 7B block's shapes.
 * All give Y_ij = fp32(acc_ij * sA_i * sW_j) + C_ij with C the fp32 FMA chain
 * of row i's entries (rounded to bf16 last for bf16 Y).  codesWT / sW come
 * from qg_quantize_cols(W); W is the unquantized weight used by the
 * compensation, K x N row-major and contiguous, stored in the SAME dtype as A
 * (`dtype` describes both; the call has no separate weight dtype, so a weight
 * in the other dtype is read wrongly without an error).  The activation
 * codes, dA and the bf16 chunk scratch live in the workspace
 * (qg_workspace_size(QG_OP_FP4_LINEAR, ...)); besides Y, the activation codes
 * and dA, no buffer grows with M: the chunk stays at its R rows.  Errors: QG_ERR_INVALID_ARG (bad dtype or
 * alpha, a NULL or misaligned pointer), the shape and workspace errors of
 * qg_quantize_act and qg_fp4_gemm, QG_ERR_UNSUPPORTED_SHAPE when the dA
 * capacity exceeds INT32_MAX entries, QG_ERR_CUDA; device conditions (NaN or
 * Inf in A, a bounded wait that ran out) go to the workspace's status word. */
qg_status qg_fp4_linear(const void* A, qg_dtype dtype, int64_t M, int64_t K,
                        const uint8_t* codesWT, const float* sW, const void* W, int64_t N,
                        double alpha, void* Y, qg_dtype y_dtype, void* ws, size_t ws_bytes,
                        cudaStream_t stream);

/* Where qg_fp4_linear leaves its intermediate results inside a workspace
 * sized for (M, K, N, dtype, alpha), as byte offsets from the workspace base
 * (each a multiple of 256), for a caller that wants to inspect them after the
 * call: parts[0] activation codes (M x K/2 bytes), parts[1] activation scales
 * (M fp32), parts[2] dA row_ptr (M + 1 int32), parts[3] dA col (int32),
 * parts[4] dA val (double), parts[5] the dA entry count (int64), parts[6] the
 * threshold T (fp32).  `parts` is a host array of 7 elements.  Nothing is
 * enqueued.  Errors: QG_ERR_INVALID_ARG (null parts, bad dtype or alpha),
 * QG_ERR_UNSUPPORTED_SHAPE (as qg_fp4_linear). */
qg_status qg_fp4_linear_parts(int64_t M, int64_t K, int64_t N, qg_dtype dtype, double alpha,
                              size_t* parts);

/* Backward GEMMs of the layer with FP4 operands (the training method also
 * runs the gradient GEMMs in FP4: [FP4-writeup], the paragraphs on the FP4
 * GEMM and on the differentiable gradient estimator).  The pages do not state
 * how gradients are quantized; the reading used here is the forward's rule:
 * each operand is quantized along the contraction dimension with one fp32
 * scale per outer index (ScaleShift, E2M1, ties to the even code), no clamp.
 *
 * dgrad: dA (M x K) = sum over n of Q(dY)[m, n] * Q(W)[k, n], with dY (M x N)
 *   quantized per row m and W (K x N, the forward weight) per row k; the
 *   contraction is over N, so N % 32 == 0 and N <= 16384.
 * wgrad: dW (K x N) = sum over m of Q(A)[m, k] * Q(dY)[m, n], with A (M x K)
 *   quantized per column k and dY per column n; the contraction is over the
 *   M tokens, so M % 32 == 0 and M <= 16384.
 * All matrices row-major and contiguous (16-byte aligned); output fp32 or
 * bf16 (out_dtype).  The codes and scales of both operands live in the
 * workspace (qg_workspace_size(QG_OP_FP4_DGRAD / QG_OP_FP4_WGRAD, M, K, N,
 * any dtype, 1.0); the size does not depend on the dtype).  Errors: as
 * qg_fp4_gemm, plus QG_ERR_UNSUPPORTED_SHAPE when the contraction dimension
 * breaks the rule above. */
qg_status qg_fp4_dgrad(const void* dY, qg_dtype dy_dtype, int64_t M, int64_t N, const void* W,
                       qg_dtype w_dtype, int64_t K, void* dA, qg_dtype out_dtype, void* ws,
                       size_t ws_bytes, cudaStream_t stream);
qg_status qg_fp4_wgrad(const void* A, qg_dtype a_dtype, int64_t M, int64_t K, const void* dY,
                       qg_dtype dy_dtype, int64_t N, void* dW, qg_dtype out_dtype, void* ws,
                       size_t ws_bytes, cudaStream_t stream);

/* MXFP4 block-scaled variant: E2M1 codes with one E8M0 scale per 32
 * consecutive elements along K (the micro-scaling section of the lecture page
 * "FP4量化训练的硬件挑战：NVIDIA Blackwell架构上的微缩放格式（Micro-scaling）实现",
 * zyxy.net/?p=24232: group, scale by the group's max, divide, round to FP4;
 * the E8M0 block scale from the micro-scaling paragraph of the low-precision
 * training survey at 10100.com/article/123065115).  Reading: the block scale
 * is 2^e with e the smallest exponent such that 6 * 2^e >= the block's largest
 * magnitude (no clipping), e in [-127, 126] stored as the byte e + 127 (a zero
 * block gets e = -127); codes E2M1(fp32(x * 2^-e)), ties to the even code.
 *
 * Codes: row-major, two codes per byte (even k in the low nibble): rows of A
 * as M x K/2, columns of W transposed as N x K/2.  Scales: the layout the GEMM
 * reads, in 512-byte atoms: rows in blocks of 128, K in groups of 128 (four
 * 32-blocks); one atom per (row block, k group), k group fastest, with
 * 2 * ceil(K / 256) groups per row block; in an atom, row r (0..127 inside its
 * block) and 32-block j (0..3 inside the group) sit at byte
 * (r % 32) * 16 + (r / 32) * 4 + j.  Padding rows and blocks hold 127 (2^0).
 * qg_mx_scale_bytes(rows, K) = ceil(rows / 128) * ceil(K / 256) * 1024 is the
 * buffer size (0 for an invalid K).  K % 32 == 0 and K <= 16384; all pointers
 * 16-byte aligned; A row pitch lda (elements) with lda * element size a
 * multiple of 16; W row pitch ldw >= N.  Non-finite inputs set the workspace
 * status (QG_ERR_NONFINITE from qg_sync_status) and give unspecified codes.
 * Workspace: qg_workspace_size(QG_OP_QUANTIZE_ROWS, ...) for the quantizers,
 * qg_workspace_size(QG_OP_FP4_GEMM, M, K, N, ...) for the GEMM.
 *
 * qg_mx_gemm: Y = sum over 32-blocks b of 2^(eA_ib + eW_jb) * sum_{k in b}
 * e2m1(qA_ik) * e2m1(qW_jk) (+ C), on the block-scaled FP4 tensor-core MMA
 * with the scales applied by the hardware; fp32 accumulation; Y fp32 or bf16,
 * raw_acc (nullable) receives the fp32 accumulator instead of / besides Y. */
size_t qg_mx_scale_bytes(int64_t rows, int64_t K);
qg_status qg_mx_quantize_rows(const void* A, qg_dtype dtype, int64_t M, int64_t K, int64_t lda,
                              uint8_t* codes, uint8_t* scales, void* ws, size_t ws_bytes,
                              cudaStream_t stream);
qg_status qg_mx_quantize_cols(const void* W, qg_dtype dtype, int64_t K, int64_t N, int64_t ldw,
                              uint8_t* codesT, uint8_t* scalesT, void* ws, size_t ws_bytes,
                              cudaStream_t stream);
qg_status qg_mx_gemm(const uint8_t* codesA, const uint8_t* sA, const uint8_t* codesWT,
                     const uint8_t* sW, int64_t M, int64_t N, int64_t K, const float* C, void* Y,
                     qg_dtype y_dtype, float* raw_acc, void* ws, size_t ws_bytes,
                     cudaStream_t stream);

/* ---- tensor-pipe E2M1 rate (measurement) -----------------------------------
 * The ceiling of qg_fp4_gemm's mainloop ([FP4-writeup], FP4 GEMM paragraph:
 * the matrix product is the part FP4 accelerates).  One launch over the whole
 * GPU: every SM (pair != 0: every 2-SM cluster that can be resident, 2-SM MMA)
 * issues iters x 4 block-scaled E2M1 MMAs of the GEMM's shape, 128 x 224 x 64
 * per SM (256 x 224 x 64 per pair), on operands that stay in shared memory,
 * accumulating in TMEM; no global memory is read or written besides the
 * status word.  Time the launch with CUDA events on `stream`; *flops_out
 * (host pointer) receives the MMA flops of the launch, 2 x 128 x 224 x 64 x 4
 * x iters per CTA.  1 <= iters <= 2^20 (else QG_ERR_INVALID_ARG; 2^20 takes
 * about a quarter of a second).  ws: qg_workspace_size(QG_OP_FP4_GEMM, 1, 32,
 * 1, QG_F32, 1.0) bytes at least; a completion wait that runs out (~2 s of SM
 * clocks) sets the timeout bit (QG_ERR_TIMEOUT from qg_sync_status), and the
 * kernel then waits once more (bounded) before it releases its TMEM.
 * acc_out (nullable device pointer, 16-byte aligned, 128 x 224 fp32,
 * row-major) receives CTA 0's accumulator after the last MMA, for checking the
 * loop's products: the operand tiles are fixed functions of the CTA index
 * (32-bit words h(i) = ((i * 2654435761 + cta) ^ (. >> 15)) * 2246822519 over
 * the A tile, 128 rows of 128 bytes, then the W^T tile, 224 rows; 128-byte
 * swizzle; a pair takes W^T rows 0..111 of CTA 0 and 0..111 of CTA 1), so
 * acc = iters x (A tile . W^T tile^T) over their 256 E2M1 values per row. */
qg_status qg_fp4_mma_loop(int64_t iters, int pair, double* flops_out, float* acc_out, void* ws,
                          size_t ws_bytes, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QGEMM_H */
