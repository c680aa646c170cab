// api.cu -- the C ABI (include/qgemm.h): argument checks, workspace layout
// and the launch sequences of each call.  No device memory is allocated here.
#include <math.h>

#include <atomic>
#include <mutex>

#include "qg_internal.cuh"

namespace qg {

static const int kMaxDevices = 64;
static int g_sms[kMaxDevices];
static bool g_ready[kMaxDevices];
static std::mutex g_mu;
static std::atomic<unsigned long long> g_launches{0};

void count_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

// One-time per-device setup (kernel attributes), with that device current.
static cudaError_t ensure_device(int* dev_out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_ready[dev]) {
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        e = act_setup();
        if (e != cudaSuccess) return e;
        e = cols_setup();
        if (e != cudaSuccess) return e;
        e = gemm_setup();
        if (e != cudaSuccess) return e;
        e = spmm_setup();
        if (e != cudaSuccess) return e;
        g_sms[dev] = sms;
        g_ready[dev] = true;
    }
    if (dev_out) *dev_out = dev;
    return cudaSuccess;
}

cudaError_t device_setup() { return ensure_device(nullptr); }

int num_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices || g_sms[dev] <= 0)
        return 148;
    return g_sms[dev];
}

static size_t elsize(qg_dtype d) { return d == QG_BF16 ? 2 : 4; }

static qg_status check_ld(const void* A, qg_dtype dt, int64_t K, int64_t ld) {
    if (A == nullptr || !aligned16(A)) return QG_ERR_INVALID_ARG;
    if (ld < K || ((size_t)ld * elsize(dt)) % 16 != 0) return QG_ERR_INVALID_ARG;
    return QG_OK;
}

static qg_status check_ws(void* ws, size_t ws_bytes, size_t need) {
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return QG_ERR_WORKSPACE;
    if (ws_bytes < need) return QG_ERR_WORKSPACE;
    return QG_OK;
}

static bool alpha_ok(double a) { return a > 0.0 && a <= 1.0; }


template <class T>
static T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

static ActBuffers act_buffers(void* ws, const WsLayout& L) {
    ActBuffers b;
    b.status = at<uint32_t>(ws, L.status);
    b.gsync = at<GridSync>(ws, L.gsync);
    b.ctr = at<Counters>(ws, L.counters);
    b.hist1 = at<uint32_t>(ws, L.hist1);
    b.hist2 = L.hist2 ? at<uint32_t>(ws, L.hist2) : nullptr;
    b.rowmax = at<uint32_t>(ws, L.rowmax);
    b.rowcnt = at<uint32_t>(ws, L.rowcnt);
    b.rowpre = at<uint32_t>(ws, L.rowpre);
    b.st_row = at<int32_t>(ws, L.st_row);
    b.st_rank = at<int32_t>(ws, L.st_rank);
    b.st_col = at<int32_t>(ws, L.st_col);
    b.st_val = at<double>(ws, L.st_val);
    b.cap = L.cap;
    b.row_slots = L.row_slots;
    return b;
}

static qg_status check_csr(const qg_csr* dA, int64_t n, double alpha) {
    if (dA == nullptr || dA->row_ptr == nullptr || dA->nnz_out == nullptr) return QG_ERR_INVALID_ARG;
    int64_t k = (int64_t)ceil(alpha * (double)n) - 1;
    if (k < 0) k = 0;
    if (k > n - 1) k = n - 1;
    const int64_t cap = n - (k + 1);
    if (cap > 0 && (dA->col == nullptr || dA->val == nullptr)) return QG_ERR_INVALID_ARG;
    if (dA->nnz_capacity < cap) return QG_ERR_INVALID_ARG;
    if (cap > (int64_t)INT32_MAX) return QG_ERR_UNSUPPORTED_SHAPE;
    return QG_OK;
}

}  // namespace qg

using namespace qg;

extern "C" {

const char* qg_status_string(qg_status s) {
    switch (s) {
        case QG_OK: return "ok";
        case QG_ERR_INVALID_ARG: return "invalid argument";
        case QG_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (need K % 32 == 0, 0 < K <= 16384, M, N >= 1)";
        case QG_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case QG_ERR_CUDA: return "CUDA runtime error";
        case QG_ERR_NONFINITE: return "non-finite value (NaN/Inf) in the input";
        case QG_ERR_TIMEOUT: return "a bounded device wait timed out";
        case QG_ERR_INTERNAL: return "internal capacity check failed";
    }
    return "unknown status";
}

const char* qg_version(void) { return "qgemm 0.1 sm_100a"; }

uint64_t qg_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int64_t qg_quantile_rank(double alpha, int64_t n) {
    int64_t k = (int64_t)ceil(alpha * (double)n) - 1;
    if (k < 0) k = 0;
    if (k > n - 1) k = n - 1;
    return k;
}

int64_t qg_nnz_capacity(int64_t n, double alpha) {
    if (n <= 0) return 0;
    return n - (qg_quantile_rank(alpha, n) + 1);
}

size_t qg_workspace_size(qg_op op, int64_t M, int64_t K, int64_t N, qg_dtype dtype, double alpha) {
    if (M < 1) M = 1;
    if (K < 2) K = 2;
    if (N < 1) N = 1;
    if (!(alpha > 0.0 && alpha <= 1.0)) alpha = 1.0;
    return ws_layout(op, M, K, N, dtype, alpha).total;
}

qg_status qg_workspace_init(void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0 || ws_bytes < 2 * kAlign)
        return QG_ERR_WORKSPACE;
    cudaError_t e = ensure_device(nullptr);
    if (e != cudaSuccess) return QG_ERR_CUDA;
    return cuda_status(cudaMemsetAsync(ws, 0, 2 * kAlign, stream));
}

qg_status qg_sync_status(void* ws, cudaStream_t stream) {
    if (ws == nullptr) return QG_ERR_WORKSPACE;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return QG_ERR_CUDA;
    uint32_t st = 0;
    if (cudaMemcpy(&st, ws, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return QG_ERR_CUDA;
    if (st == 0) return QG_OK;
    if (cudaMemset(ws, 0, sizeof(uint32_t)) != cudaSuccess) return QG_ERR_CUDA;
    if (st & kStatusTimeout) {
        // a wait that gave up may have left a grid barrier half-counted
        if (cudaMemset(static_cast<uint8_t*>(ws) + kGridSyncOffset, 0, sizeof(GridSync)) != cudaSuccess)
            return QG_ERR_CUDA;
    }
    if (st & kStatusNonFinite) return QG_ERR_NONFINITE;
    if (st & kStatusTimeout) return QG_ERR_TIMEOUT;
    return QG_ERR_INTERNAL;
}

qg_status qg_e2m1_encode(const float* x, int64_t n, uint8_t* packed, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
    if (n < 0 || (n % 2) != 0) return QG_ERR_INVALID_ARG;
    if (n == 0) return QG_OK;
    if (!x || !packed || !aligned16(x) || !aligned16(packed)) return QG_ERR_INVALID_ARG;
    qg_status st = check_ws(ws, ws_bytes, ws_layout(QG_OP_QUANTIZE_ROWS, 1, 32, 1, QG_F32, 1.0).total);
    if (st != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    launch_e2m1_encode(x, n, packed, stream);
    return cuda_status(cudaGetLastError());
}

qg_status qg_quantize_rows(const void* A, qg_dtype dtype, int64_t M, int64_t K, int64_t lda,
                           uint8_t* codes, float* scales, void* ws, size_t ws_bytes,
                           cudaStream_t stream) {
    if (!dtype_ok(dtype)) return QG_ERR_INVALID_ARG;
    qg_status st = check_mk(M, K);
    if (st != QG_OK) return st;
    if ((st = check_ld(A, dtype, K, lda)) != QG_OK) return st;
    if (!codes || !scales || !aligned16(codes)) return QG_ERR_INVALID_ARG;
    if ((st = check_ws(ws, ws_bytes, ws_layout(QG_OP_QUANTIZE_ROWS, M, K, 1, dtype, 1.0).total)) != QG_OK)
        return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    launch_quantize_rows(A, dtype, M, K, lda, codes, scales, stream);
    return cuda_status(cudaGetLastError());
}

qg_status qg_quantize_cols(const void* W, qg_dtype dtype, int64_t K, int64_t N, int64_t ldw,
                           uint8_t* codesT, float* scales, void* ws, size_t ws_bytes,
                           cudaStream_t stream) {
    if (!dtype_ok(dtype)) return QG_ERR_INVALID_ARG;
    qg_status st = check_mk(N, K);
    if (st != QG_OK) return st;
    if (W == nullptr || !aligned16(W) || ldw < N) return QG_ERR_INVALID_ARG;
    if (!codesT || !scales || !aligned16(codesT)) return QG_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(QG_OP_QUANTIZE_COLS, 1, K, N, dtype, 1.0);
    if ((st = check_ws(ws, ws_bytes, L.total)) != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    if (dtype == QG_BF16 &&
        launch_quantize_cols_fused(W, K, N, ldw, codesT, scales, at<uint32_t>(ws, L.colmax),
                                   at<GridSync>(ws, L.gsync), at<uint32_t>(ws, L.status), stream))
        return cuda_status(cudaGetLastError());
    launch_quantize_cols(W, dtype, K, N, ldw, codesT, scales, at<uint32_t>(ws, L.colmax), stream);
    return cuda_status(cudaGetLastError());
}

qg_status qg_clamp_compensate(const void* A, qg_dtype dtype, int64_t M, int64_t K, int64_t lda,
                              double alpha, void* A_clamped, const qg_csr* dA, float* T_out,
                              void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (!dtype_ok(dtype) || !alpha_ok(alpha)) return QG_ERR_INVALID_ARG;
    qg_status st = check_mk(M, K);
    if (st != QG_OK) return st;
    if ((st = check_ld(A, dtype, K, lda)) != QG_OK) return st;
    if (A_clamped && !aligned16(A_clamped)) return QG_ERR_INVALID_ARG;
    if (T_out == nullptr) return QG_ERR_INVALID_ARG;
    if ((st = check_csr(dA, M * K, alpha)) != QG_OK) return st;
    const WsLayout L = ws_layout(QG_OP_CLAMP_COMPENSATE, M, K, 1, dtype, alpha);
    if ((st = check_ws(ws, ws_bytes, L.total)) != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    const int64_t rank = qg_quantile_rank(alpha, M * K);
    return cuda_status(run_clamp_compensate(A, dtype, M, K, lda, rank, act_buffers(ws, L), A_clamped,
                                            dA, T_out, stream));
}

qg_status qg_quantize_act(const void* A, qg_dtype dtype, int64_t M, int64_t K, int64_t lda,
                          double alpha, uint8_t* codes, float* scales, const qg_csr* dA,
                          float* T_out, void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (!dtype_ok(dtype) || !alpha_ok(alpha)) return QG_ERR_INVALID_ARG;
    qg_status st = check_mk(M, K);
    if (st != QG_OK) return st;
    if ((st = check_ld(A, dtype, K, lda)) != QG_OK) return st;
    if (!codes || !scales || !aligned16(codes) || T_out == nullptr) return QG_ERR_INVALID_ARG;
    if ((st = check_csr(dA, M * K, alpha)) != QG_OK) return st;
    const WsLayout L = ws_layout(QG_OP_QUANTIZE_ACT, M, K, 1, dtype, alpha);
    if ((st = check_ws(ws, ws_bytes, L.total)) != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    const int64_t rank = qg_quantile_rank(alpha, M * K);
    return cuda_status(run_quantize_act(A, dtype, M, K, lda, rank, act_buffers(ws, L), codes, scales,
                                        dA, T_out, stream));
}

qg_status qg_spmm_correction(const qg_csr* dA, int64_t M, const void* W, qg_dtype w_dtype,
                             int64_t K, int64_t N, int64_t ldw, float* C, void* ws,
                             size_t ws_bytes, cudaStream_t stream) {
    if (!dtype_ok(w_dtype)) return QG_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || K < 1) return QG_ERR_UNSUPPORTED_SHAPE;
    if (dA == nullptr || dA->row_ptr == nullptr) return QG_ERR_INVALID_ARG;
    if (W == nullptr || !aligned16(W) || ldw < N || C == nullptr || !aligned16(C)) return QG_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(QG_OP_SPMM, M, K, N, w_dtype, 1.0);
    qg_status st = check_ws(ws, ws_bytes, L.total);
    if (st != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    launch_spmm(dA, M, W, w_dtype, N, ldw, C, at<uint32_t>(ws, L.status), stream);
    return cuda_status(cudaGetLastError());
}

qg_status qg_spmm_accumulate(const qg_csr* dA, int64_t M, const void* W, qg_dtype w_dtype,
                             int64_t K, int64_t N, int64_t ldw, float* Y, void* ws,
                             size_t ws_bytes, cudaStream_t stream) {
    if (!dtype_ok(w_dtype)) return QG_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || K < 1) return QG_ERR_UNSUPPORTED_SHAPE;
    if (dA == nullptr || dA->row_ptr == nullptr) return QG_ERR_INVALID_ARG;
    if (W == nullptr || !aligned16(W) || ldw < N || Y == nullptr || !aligned16(Y)) return QG_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(QG_OP_SPMM, M, K, N, w_dtype, 1.0);
    qg_status st = check_ws(ws, ws_bytes, L.total);
    if (st != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    launch_spmm(dA, M, W, w_dtype, N, ldw, Y, at<uint32_t>(ws, L.status), stream, true);
    return cuda_status(cudaGetLastError());
}

qg_status qg_fp4_gemm(const uint8_t* codesA, const float* sA, const uint8_t* codesWT,
                      const float* sW, int64_t M, int64_t N, int64_t K, const float* C, void* Y,
                      qg_dtype y_dtype, float* raw_acc, void* ws, size_t ws_bytes,
                      cudaStream_t stream) {
    if (!dtype_ok(y_dtype)) return QG_ERR_INVALID_ARG;
    qg_status st = check_mk(M, K);
    if (st != QG_OK) return st;
    if ((st = check_mk(N, K)) != QG_OK) return st;
    if (!codesA || !codesWT || !sA || !sW || !aligned16(codesA) || !aligned16(codesWT) ||
        !aligned16(sW))
        return QG_ERR_INVALID_ARG;
    if (Y == nullptr && raw_acc == nullptr) return QG_ERR_INVALID_ARG;
    if ((Y && !aligned16(Y)) || (C && !aligned16(C)) || (raw_acc && !aligned16(raw_acc)))
        return QG_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(QG_OP_FP4_GEMM, M, K, N, y_dtype, 1.0);
    if ((st = check_ws(ws, ws_bytes, L.total)) != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    return cuda_status(launch_fp4_gemm(codesA, sA, codesWT, sW, M, N, K, C, Y, y_dtype, raw_acc,
                                       at<uint32_t>(ws, L.status), stream));
}

qg_status qg_fp4_gemm_accumulate(const uint8_t* codesA, const float* sA, const uint8_t* codesWT,
                                 const float* sW, int64_t M, int64_t N, int64_t K, float* Y,
                                 void* ws, size_t ws_bytes, cudaStream_t stream) {
    qg_status st = check_mk(M, K);
    if (st != QG_OK) return st;
    if ((st = check_mk(N, K)) != QG_OK) return st;
    if (!codesA || !codesWT || !sA || !sW || !Y || !aligned16(codesA) || !aligned16(codesWT) ||
        !aligned16(sW) || !aligned16(Y))
        return QG_ERR_INVALID_ARG;
    if (N % 4 != 0) return QG_ERR_UNSUPPORTED_SHAPE;   // Y rows in whole 16-byte units for TMA
    const WsLayout L = ws_layout(QG_OP_FP4_GEMM, M, K, N, QG_F32, 1.0);
    if ((st = check_ws(ws, ws_bytes, L.total)) != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    return cuda_status(launch_fp4_gemm(codesA, sA, codesWT, sW, M, N, K, nullptr, Y, QG_F32,
                                       nullptr, at<uint32_t>(ws, L.status), stream, true));
}

qg_status qg_fp4_linear(const void* A, qg_dtype dtype, int64_t M, int64_t K,
                        const uint8_t* codesWT, const float* sW, const void* W, int64_t N,
                        double alpha, void* Y, qg_dtype y_dtype, void* ws, size_t ws_bytes,
                        cudaStream_t stream) {
    if (!dtype_ok(dtype) || !dtype_ok(y_dtype) || !alpha_ok(alpha)) return QG_ERR_INVALID_ARG;
    qg_status st = check_mk(M, K);
    if (st != QG_OK) return st;
    if ((st = check_mk(N, K)) != QG_OK) return st;
    if ((st = check_ld(A, dtype, K, K)) != QG_OK) return st;
    if (!codesWT || !sW || !W || !Y || !aligned16(codesWT) || !aligned16(sW) || !aligned16(W) ||
        !aligned16(Y))
        return QG_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(QG_OP_FP4_LINEAR, M, K, N, dtype, alpha);
    if ((st = check_ws(ws, ws_bytes, L.total)) != QG_OK) return st;
    if (L.cap > (int64_t)INT32_MAX) return QG_ERR_UNSUPPORTED_SHAPE;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    qg_csr csr;
    csr.row_ptr = at<int32_t>(ws, L.csr_row_ptr);
    csr.col = at<int32_t>(ws, L.csr_col);
    csr.val = at<double>(ws, L.csr_val);
    csr.nnz_capacity = L.cap;
    csr.nnz_out = at<int64_t>(ws, L.csr_nnz);
    uint8_t* codes = at<uint8_t>(ws, L.act_codes);
    float* scales = at<float>(ws, L.act_scales);
    const int64_t rank = qg_quantile_rank(alpha, M * K);
    uint32_t* status = at<uint32_t>(ws, L.status);
    cudaError_t e = run_quantize_act(A, dtype, M, K, K, rank, act_buffers(ws, L), codes, scales, &csr,
                                     at<float>(ws, L.thr), stream);
    if (e != cudaSuccess) return QG_ERR_CUDA;
    if (y_dtype == QG_F32) {
        // fp32 Y, no M x N buffer besides Y, in one of two orders with the same
        // result: with many entries per row (linear_gemm_first: at least
        // kAddOrderEntriesPer4096K possible per 4096 of K) the GEMM writes the scaled product and the SpMM
        // adds the compensation into Y, the SpMM's gathers hiding its reads of
        // Y; otherwise the compensation is written into Y first and the GEMM
        // adds its product into it through the memory system's bulk reduction
        // (or, where the TMA epilogue cannot describe Y, reads each 32 x 32
        // sub-tile of Y as C before it overwrites it in place)
        float* Yf = static_cast<float*>(Y);
        if (linear_gemm_first(L.cap, M, K)) {
            e = launch_fp4_gemm(codes, scales, codesWT, sW, M, N, K, nullptr, Y, QG_F32, nullptr,
                                status, stream);
            if (e != cudaSuccess) return QG_ERR_CUDA;
            launch_spmm(&csr, M, W, dtype, N, N, Yf, status, stream, true);
            return cuda_status(cudaGetLastError());
        }
        launch_spmm(&csr, M, W, dtype, N, N, Yf, status, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return QG_ERR_CUDA;
        e = launch_fp4_gemm(codes, scales, codesWT, sW, M, N, K, nullptr, Y, QG_F32, nullptr,
                            status, stream, true);
        if (e != cudaErrorInvalidValue) return cuda_status(e);
        (void)cudaGetLastError();   // nothing was launched: add in place instead
        return cuda_status(launch_fp4_gemm(codes, scales, codesWT, sW, M, N, K, Yf, Y, QG_F32,
                                           nullptr, status, stream));
    }
    // bf16 Y has no room for the fp32 compensation, so the rows go in chunks
    // of R: the SpMM writes a chunk's dA . W into an fp32 scratch of R x N (at
    // most kLinearScratchMaxBytes, much of it still in L2 when it is read) and
    // the GEMM reads it as C while it writes the chunk's Y.  Every element is
    // bf16(acc s_i t_j + c_ij) with c_ij its row's fp32 FMA chain, as when the
    // compensated GEMM computes c inside the kernel (qg_fp4_gemm_compensated),
    // which is 1.3-3.8x slower at the 7B block's shapes.
    const int64_t R = linear_chunk_rows(M, N);
    float* scratch = at<float>(ws, L.linear_scratch);
    for (int64_t r0 = 0; r0 < M; r0 += R) {
        const int64_t rows = std::min<int64_t>(R, M - r0);
        qg_csr chunk = csr;
        chunk.row_ptr = csr.row_ptr + r0;   // entries are indexed absolutely
        launch_spmm(&chunk, rows, W, dtype, N, N, scratch, status, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return QG_ERR_CUDA;
        e = launch_fp4_gemm(codes + r0 * (K / 2), scales + r0, codesWT, sW, rows, N, K, scratch,
                            static_cast<uint16_t*>(Y) + r0 * N, y_dtype, nullptr, status, stream);
        if (e != cudaSuccess) return QG_ERR_CUDA;
    }
    return QG_OK;
}

qg_status qg_fp4_gemm_compensated(const uint8_t* codesA, const float* sA, const uint8_t* codesWT,
                                  const float* sW, int64_t M, int64_t N, int64_t K,
                                  const qg_csr* dA, const void* W, qg_dtype w_dtype, int64_t ldw,
                                  void* Y, qg_dtype y_dtype, void* ws, size_t ws_bytes,
                                  cudaStream_t stream) {
    if (!dtype_ok(y_dtype) || !dtype_ok(w_dtype)) return QG_ERR_INVALID_ARG;
    qg_status st = check_mk(M, K);
    if (st != QG_OK) return st;
    if ((st = check_mk(N, K)) != QG_OK) return st;
    if (!codesA || !codesWT || !sA || !sW || !aligned16(codesA) || !aligned16(codesWT) ||
        !aligned16(sW))
        return QG_ERR_INVALID_ARG;
    if (Y == nullptr || !aligned16(Y)) return QG_ERR_INVALID_ARG;
    if (dA == nullptr || dA->row_ptr == nullptr || dA->col == nullptr || dA->val == nullptr)
        return QG_ERR_INVALID_ARG;
    if (W == nullptr || !aligned16(W) || ldw < N) return QG_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(QG_OP_FP4_GEMM_COMPENSATED, M, K, N, y_dtype, 1.0);
    if ((st = check_ws(ws, ws_bytes, L.total)) != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    return cuda_status(launch_fp4_gemm_corr(codesA, sA, codesWT, sW, M, N, K, dA, W, w_dtype, ldw,
                                            at<float>(ws, L.corr_scratch), Y, y_dtype,
                                            at<uint32_t>(ws, L.status), stream));
}

qg_status qg_fp4_linear_parts(int64_t M, int64_t K, int64_t N, qg_dtype dtype, double alpha,
                              size_t* parts) {
    if (parts == nullptr || !dtype_ok(dtype) || !alpha_ok(alpha)) return QG_ERR_INVALID_ARG;
    qg_status st = check_mk(M, K);
    if (st != QG_OK) return st;
    if ((st = check_mk(N, K)) != QG_OK) return st;
    const WsLayout L = ws_layout(QG_OP_FP4_LINEAR, M, K, N, dtype, alpha);
    parts[0] = L.act_codes;
    parts[1] = L.act_scales;
    parts[2] = L.csr_row_ptr;
    parts[3] = L.csr_col;
    parts[4] = L.csr_val;
    parts[5] = L.csr_nnz;
    parts[6] = L.thr;
    return QG_OK;
}

// Column quantization of a whole row-major matrix X (rows x cols) into
// codesT (cols x rows/2) + scales (cols): the cooperative bf16 kernel or the
// multi-kernel sequence (colmax: 32 * cols words of scratch).
static cudaError_t quantize_cols_any(const void* X, qg_dtype dt, int64_t rows, int64_t cols,
                                     uint8_t* codesT, float* scales, uint32_t* colmax, void* ws,
                                     const WsLayout& L, cudaStream_t stream) {
    if (dt == QG_BF16 &&
        launch_quantize_cols_fused(X, rows, cols, cols, codesT, scales, colmax,
                                   at<GridSync>(ws, L.gsync), at<uint32_t>(ws, L.status), stream))
        return cudaGetLastError();
    launch_quantize_cols(X, dt, rows, cols, cols, codesT, scales, colmax, stream);
    return cudaGetLastError();
}

qg_status qg_fp4_dgrad(const void* dY, qg_dtype dy_dtype, int64_t M, int64_t N, const void* W,
                       qg_dtype w_dtype, int64_t K, void* dA, qg_dtype out_dtype, void* ws,
                       size_t ws_bytes, cudaStream_t stream) {
    if (!dtype_ok(dy_dtype) || !dtype_ok(w_dtype) || !dtype_ok(out_dtype)) return QG_ERR_INVALID_ARG;
    qg_status st = check_mk(M, N);              // contraction over N
    if (st != QG_OK) return st;
    if ((st = check_mk(K, N)) != QG_OK) return st;
    if ((st = check_ld(dY, dy_dtype, N, N)) != QG_OK) return st;
    if ((st = check_ld(W, w_dtype, N, N)) != QG_OK) return st;
    if (dA == nullptr || !aligned16(dA)) return QG_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(QG_OP_FP4_DGRAD, M, K, N, QG_F32, 1.0);
    if ((st = check_ws(ws, ws_bytes, L.total)) != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    uint8_t* ca = at<uint8_t>(ws, L.g_codes_a);
    float* sa = at<float>(ws, L.g_scales_a);
    uint8_t* cb = at<uint8_t>(ws, L.g_codes_b);
    float* sb = at<float>(ws, L.g_scales_b);
    launch_quantize_rows(dY, dy_dtype, M, N, N, ca, sa, stream);
    launch_quantize_rows(W, w_dtype, K, N, N, cb, sb, stream);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return QG_ERR_CUDA;
    return cuda_status(launch_fp4_gemm(ca, sa, cb, sb, M, K, N, nullptr, dA, out_dtype, nullptr,
                                       at<uint32_t>(ws, L.status), stream));
}

qg_status qg_fp4_wgrad(const void* A, qg_dtype a_dtype, int64_t M, int64_t K, const void* dY,
                       qg_dtype dy_dtype, int64_t N, void* dW, qg_dtype out_dtype, void* ws,
                       size_t ws_bytes, cudaStream_t stream) {
    if (!dtype_ok(a_dtype) || !dtype_ok(dy_dtype) || !dtype_ok(out_dtype)) return QG_ERR_INVALID_ARG;
    qg_status st = check_mk(K, M);              // contraction over the M tokens
    if (st != QG_OK) return st;
    if ((st = check_mk(N, M)) != QG_OK) return st;
    if (A == nullptr || dY == nullptr || !aligned16(A) || !aligned16(dY)) return QG_ERR_INVALID_ARG;
    if (dW == nullptr || !aligned16(dW)) return QG_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(QG_OP_FP4_WGRAD, M, K, N, QG_F32, 1.0);
    if ((st = check_ws(ws, ws_bytes, L.total)) != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    uint8_t* ca = at<uint8_t>(ws, L.g_codes_a);
    float* sa = at<float>(ws, L.g_scales_a);
    uint8_t* cb = at<uint8_t>(ws, L.g_codes_b);
    float* sb = at<float>(ws, L.g_scales_b);
    uint32_t* colmax = at<uint32_t>(ws, L.colmax);
    cudaError_t e = quantize_cols_any(A, a_dtype, M, K, ca, sa, colmax, ws, L, stream);
    if (e != cudaSuccess) return QG_ERR_CUDA;
    e = quantize_cols_any(dY, dy_dtype, M, N, cb, sb, colmax, ws, L, stream);
    if (e != cudaSuccess) return QG_ERR_CUDA;
    return cuda_status(launch_fp4_gemm(ca, sa, cb, sb, K, N, M, nullptr, dW, out_dtype, nullptr,
                                       at<uint32_t>(ws, L.status), stream));
}

size_t qg_mx_scale_bytes(int64_t rows, int64_t K) {
    if (rows < 1 || K < 32 || K % 32 != 0) return 0;
    return (size_t)((rows + 127) / 128) * (size_t)((K + 255) / 256) * 1024u;
}

qg_status qg_mx_quantize_rows(const void* A, qg_dtype dtype, int64_t M, int64_t K, int64_t lda,
                              uint8_t* codes, uint8_t* scales, void* ws, size_t ws_bytes,
                              cudaStream_t stream) {
    if (!dtype_ok(dtype)) return QG_ERR_INVALID_ARG;
    qg_status st = check_mk(M, K);
    if (st != QG_OK) return st;
    if ((st = check_ld(A, dtype, K, lda)) != QG_OK) return st;
    if (!codes || !scales || !aligned16(codes) || !aligned16(scales)) return QG_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(QG_OP_QUANTIZE_ROWS, M, K, 1, dtype, 1.0);
    if ((st = check_ws(ws, ws_bytes, L.total)) != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    launch_mx_quantize_rows(A, dtype, M, K, lda, codes, scales, at<uint32_t>(ws, L.status), stream);
    return cuda_status(cudaGetLastError());
}

qg_status qg_mx_quantize_cols(const void* W, qg_dtype dtype, int64_t K, int64_t N, int64_t ldw,
                              uint8_t* codesT, uint8_t* scalesT, void* ws, size_t ws_bytes,
                              cudaStream_t stream) {
    if (!dtype_ok(dtype)) return QG_ERR_INVALID_ARG;
    qg_status st = check_mk(N, K);
    if (st != QG_OK) return st;
    if (W == nullptr || ldw < N) return QG_ERR_INVALID_ARG;
    if (!codesT || !scalesT || !aligned16(codesT) || !aligned16(scalesT)) return QG_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(QG_OP_QUANTIZE_ROWS, 1, K, 1, dtype, 1.0);
    if ((st = check_ws(ws, ws_bytes, L.total)) != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    launch_mx_quantize_cols(W, dtype, K, N, ldw, codesT, scalesT, at<uint32_t>(ws, L.status), stream);
    return cuda_status(cudaGetLastError());
}

qg_status qg_mx_gemm(const uint8_t* codesA, const uint8_t* sA, const uint8_t* codesWT,
                     const uint8_t* sW, int64_t M, int64_t N, int64_t K, const float* C, void* Y,
                     qg_dtype y_dtype, float* raw_acc, void* ws, size_t ws_bytes,
                     cudaStream_t stream) {
    if (!dtype_ok(y_dtype)) return QG_ERR_INVALID_ARG;
    qg_status st = check_mk(M, K);
    if (st != QG_OK) return st;
    if ((st = check_mk(N, K)) != QG_OK) return st;
    if (!codesA || !codesWT || !sA || !sW || !aligned16(codesA) || !aligned16(codesWT) ||
        !aligned16(sA) || !aligned16(sW))
        return QG_ERR_INVALID_ARG;
    if (Y == nullptr && raw_acc == nullptr) return QG_ERR_INVALID_ARG;
    if ((Y && !aligned16(Y)) || (C && !aligned16(C)) || (raw_acc && !aligned16(raw_acc)))
        return QG_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(QG_OP_FP4_GEMM, M, K, N, y_dtype, 1.0);
    if ((st = check_ws(ws, ws_bytes, L.total)) != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    return cuda_status(launch_fp4_gemm_mx(codesA, sA, codesWT, sW, M, N, K, C, Y, y_dtype, raw_acc,
                                          at<uint32_t>(ws, L.status), stream));
}

qg_status qg_fp4_mma_loop(int64_t iters, int pair, double* flops_out, float* acc_out, void* ws,
                          size_t ws_bytes, cudaStream_t stream) {
    if (iters < 1 || iters > ((int64_t)1 << 20) || flops_out == nullptr) return QG_ERR_INVALID_ARG;
    if (acc_out != nullptr && !aligned16(acc_out)) return QG_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(QG_OP_FP4_GEMM, 1, 32, 1, QG_F32, 1.0);
    qg_status st = check_ws(ws, ws_bytes, L.total);
    if (st != QG_OK) return st;
    if (ensure_device(nullptr) != cudaSuccess) return QG_ERR_CUDA;
    return cuda_status(launch_fp4_mma_loop(iters, pair != 0, flops_out, acc_out,
                                           at<uint32_t>(ws, L.status), stream));
}

}  // extern "C"
