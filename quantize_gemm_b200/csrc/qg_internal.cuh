// qg_internal.cuh -- device helpers and workspace layout shared by the
// kernels of the FP4 linear-layer library (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <stdlib.h>

#include <algorithm>

#include "../../include/qgemm.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a (B200) only"
#endif

namespace qg {

// ---------------------------------------------------------------- status word
// Sticky device status bits, OR-ed into the first word of the workspace.
enum : uint32_t {
    kStatusNonFinite = 1u << 0,
    kStatusTimeout = 1u << 1,
    kStatusOverflow = 1u << 2,
};

// Counters that live right after the status word.
struct Counters {
    unsigned long long nnz;        // dA entries that overflowed their row region
    unsigned long long sel_below;  // entries strictly below the selected bin
    uint32_t nonfinite;            // set when a NaN/Inf key was seen
    uint32_t sel_bin;              // bin chosen by the last selection pass
    uint32_t T_key;                // final threshold as |x| bit pattern
    uint32_t done_hist;            // CTAs finished with the histogram pass
    uint32_t done_refine;          // CTAs finished with the fp32 refine pass
    uint32_t done_clamp;           // CTAs finished with the clamp pass
    // bf16 band pass: keys in [band_lo, band_hi] are histogrammed, the ones
    // at or above band_lo counted (band_below holds that count, from which
    // the number below the band follows); band_missed is set when the order
    // statistic fell outside the band and an exact fallback ran
    unsigned long long band_below;
    uint32_t band_lo;
    uint32_t band_hi;
    uint32_t done_band;
    uint32_t band_missed;
};

// Staging of dA: every row owns `row_slots` entries (its first entries in
// column order, stored at row * row_slots + rank); entries past that go to an
// overflow list of (row, rank, col, val) with room for every clamped entry.
inline int64_t staging_row_slots(int64_t M, int64_t K, int64_t cap) {
    int64_t per = (cap + M - 1) / (M > 0 ? M : 1);
    int64_t r = 2 * per + 16;
    return r < K ? r : K;
}

// ---------------------------------------------------------------- workspace
constexpr size_t kAlign = 256;
constexpr int kHist1Bins = 1 << 15;   // 15-bit keys (bf16 |x|, fp32 |x| >> 16)
constexpr int kHist2Bins = 1 << 16;   // fp32 refine: low 16 bits of |x|

inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Grid barrier of the cooperative kernels (inside the status block, so
// qg_workspace_init zeroes it; the count is back to 0 after every barrier),
// and the fused activation kernel's flag: gen + 1 once CTA 0 has zeroed that
// call's counters.
struct GridSync {
    uint32_t count;
    uint32_t gen;
    uint32_t zflag;
};
constexpr size_t kGridSyncOffset = 16;   // bytes from the workspace base
static_assert(kGridSyncOffset + sizeof(GridSync) <= 2 * kAlign, "inside the zeroed header");

// Scratch of the compensated GEMM: two slots of 128 rows x 224 fp32 columns
// per CTA, for up to 160 CTAs (36.7 MB; it stays in L2).
constexpr size_t kCorrScratchBytes = (size_t)160 * 2 * 128 * 224 * 4;

// The layer with bf16 Y goes through its rows in chunks: the compensation of
// a chunk is written into an fp32 scratch of R rows x N (at most this many
// bytes, R a multiple of the GEMM's 256-row pair tile, at least 256 rows or
// all of M) and the GEMM reads it back while it writes that chunk of Y.
constexpr size_t kLinearScratchMaxBytes = (size_t)128 << 20;
inline int64_t linear_chunk_rows(int64_t M, int64_t N) {
    int64_t r = (int64_t)(kLinearScratchMaxBytes / ((size_t)N * 4)) / 256 * 256;
    if (r < 256) r = 256;
    return r < M ? r : M;
}

struct WsLayout {
    size_t gsync = 0;
    size_t rowpre = 0;
    size_t g_codes_a = 0, g_scales_a = 0, g_codes_b = 0, g_scales_b = 0;
    size_t status = 0, counters = 0, hist1 = 0, hist2 = 0, rowmax = 0, rowcnt = 0;
    size_t st_row = 0, st_rank = 0, st_col = 0, st_val = 0, colmax = 0;
    size_t act_codes = 0, act_scales = 0, csr_row_ptr = 0, csr_col = 0, csr_val = 0,
           csr_nnz = 0, thr = 0, corr_scratch = 0, linear_scratch = 0;
    size_t total = 0;
    int64_t cap = 0;
    int64_t row_slots = 0;
};

// Compute the layout for an op.  Offsets are relative to the workspace base.
inline WsLayout ws_layout(qg_op op, int64_t M, int64_t K, int64_t N, qg_dtype dtype,
                          double alpha) {
    WsLayout L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t at = off;
        off = align_up(off + (bytes ? bytes : 1));
        return at;
    };
    L.status = take(kGridSyncOffset + sizeof(GridSync));   // status word at +0, GridSync at +16
    L.gsync = L.status + kGridSyncOffset;
    L.counters = take(sizeof(Counters));
    bool act = (op == QG_OP_CLAMP_COMPENSATE || op == QG_OP_QUANTIZE_ACT ||
                op == QG_OP_FP4_LINEAR);
    if (act) {
        int64_t n = M * K;
        int64_t k = (int64_t)ceil(alpha * (double)n) - 1;
        if (k < 0) k = 0;
        if (k > n - 1) k = n - 1;
        L.cap = n - (k + 1);
        int64_t cap = L.cap > 0 ? L.cap : 1;
        L.hist1 = take(sizeof(uint32_t) * kHist1Bins);
        if (dtype == QG_F32) L.hist2 = take(sizeof(uint32_t) * kHist2Bins);
        // row maxima: one per (row, 1024-column step) for the cooperative
        // bf16 kernel (the other kernels use the first M words, one per row)
        const int64_t steps = (K / 8 + 127) / 128;
        L.rowmax = take(sizeof(uint32_t) * (size_t)M * (size_t)steps);
        L.rowcnt = take(sizeof(uint32_t) * (size_t)M);
        L.rowpre = take(sizeof(uint32_t) * (size_t)M);
        L.row_slots = staging_row_slots(M, K, L.cap);
        const size_t slots = (size_t)M * (size_t)L.row_slots + (size_t)cap;
        L.st_row = take(sizeof(int32_t) * (size_t)cap);     // overflow list only
        L.st_rank = take(sizeof(int32_t) * (size_t)cap);    // overflow list only
        L.st_col = take(sizeof(int32_t) * slots);
        L.st_val = take(sizeof(double) * slots);
    }
    // column maxima: N words (fp32 path); the cooperative bf16 kernel keeps
    // per-split partial maxima, up to 32 splits
    if (op == QG_OP_QUANTIZE_COLS) L.colmax = take(sizeof(uint32_t) * 32 * (size_t)N);
    // backward GEMMs (forward dims M, K, N): the two operands' codes + scales
    //   dgrad: a = dY rows (M x N/2, M), b = W rows (K x N/2, K)
    //   wgrad: a = A columns (K x M/2, K), b = dY columns (N x M/2, N), plus
    //          the column quantizer's partial maxima
    if (op == QG_OP_FP4_DGRAD) {
        L.g_codes_a = take((size_t)M * (size_t)(N / 2));
        L.g_scales_a = take(sizeof(float) * (size_t)M);
        L.g_codes_b = take((size_t)K * (size_t)(N / 2));
        L.g_scales_b = take(sizeof(float) * (size_t)K);
    }
    if (op == QG_OP_FP4_WGRAD) {
        L.g_codes_a = take((size_t)K * (size_t)(M / 2));
        L.g_scales_a = take(sizeof(float) * (size_t)K);
        L.g_codes_b = take((size_t)N * (size_t)(M / 2));
        L.g_scales_b = take(sizeof(float) * (size_t)N);
        L.colmax = take(sizeof(uint32_t) * 32 * (size_t)(K > N ? K : N));
    }
    if (op == QG_OP_FP4_LINEAR) {
        int64_t cap = L.cap > 0 ? L.cap : 1;
        L.act_codes = take((size_t)M * (size_t)(K / 2));
        L.act_scales = take(sizeof(float) * (size_t)M);
        L.csr_row_ptr = take(sizeof(int32_t) * (size_t)(M + 1));
        L.csr_col = take(sizeof(int32_t) * (size_t)cap);
        L.csr_val = take(sizeof(double) * (size_t)cap);
        L.csr_nnz = take(sizeof(int64_t));
        L.thr = take(sizeof(float));
    }
    // the compensated GEMM's scratch slots
    if (op == QG_OP_FP4_GEMM_COMPENSATED) L.corr_scratch = take(kCorrScratchBytes);
    // the layer's chunk of fp32 compensation rows (bf16 Y)
    if (op == QG_OP_FP4_LINEAR)
        L.linear_scratch = take((size_t)linear_chunk_rows(M, N) * (size_t)N * sizeof(float));
    L.total = off;
    return L;
}

// ------------------------------------------------------------- device helpers
#ifdef __CUDACC__

__device__ __forceinline__ void flag_status(uint32_t* status, uint32_t bits) {
    atomicOr(status, bits);
}

// Two fp32 values -> one byte of E2M1 codes by the hardware conversion
// (cvt.rn.satfinite.e2m1x2.f32: round to nearest even, saturate at 6; a
// negative input that rounds to zero keeps its sign, code 0x8, which a check
// over every non-NaN fp32 pattern confirmed).  lo lands in bits 3..0.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
    uint16_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}"
        : "=h"(r)
        : "f"(hi), "f"(lo));
    return (uint32_t)r & 0xFFu;
}

// Scale a bf16 pair by r and encode it: one byte, element 0 in the low nibble.
__device__ __forceinline__ uint32_t bf16x2_encode(uint32_t w, float r) {
    const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xFFFF0000u);
    float a, b;
    asm("{\n\t.reg .b64 p, q, t;\n\tmov.b64 p, {%2, %3};\n\tmov.b64 q, {%4, %4};\n\t"
        "mul.rn.f32x2 t, p, q;\n\tmov.b64 {%0, %1}, t;\n\t}"
        : "=f"(a), "=f"(b)
        : "f"(lo), "f"(hi), "f"(r));
    return e2m1x2(a, b);
}

// Eight values -> four packed bytes (element 0 in the low nibble of byte 0).
__device__ __forceinline__ uint32_t e2m1x8(const float (&x)[8]) {
    return e2m1x2(x[0], x[1]) | (e2m1x2(x[2], x[3]) << 8) | (e2m1x2(x[4], x[5]) << 16) |
           (e2m1x2(x[6], x[7]) << 24);
}

// Scale factors of one row/column from its absolute maximum:
// r = 6 / amax and s = amax / 6, IEEE correctly rounded; both 0 for a zero
// (or so tiny that 6 / amax overflows) maximum.
__device__ __forceinline__ void scale_factors(float amax, float& r, float& s) {
    float rr = __fdiv_rn(6.0f, amax);
    if (amax == 0.0f || isinf(rr)) {
        r = 0.0f;
        s = 0.0f;
    } else {
        r = rr;
        s = __fdiv_rn(amax, 6.0f);
    }
}

// Magnitude key of a value: the bit pattern without the sign.  For finite
// values the keys order like |x|.
__device__ __forceinline__ uint32_t key_of(float x) { return __float_as_uint(x) & 0x7FFFFFFFu; }
__device__ __forceinline__ uint32_t key_of_bf16_bits(uint32_t b) { return b & 0x7FFFu; }
__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

// Load 8 consecutive elements (16-byte aligned) as fp32.
template <qg_dtype DT>
__device__ __forceinline__ void load8(const void* base, int64_t idx, float (&x)[8]) {
    if constexpr (DT == QG_BF16) {
        uint4 v = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + idx));
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    } else {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
        float4 a = __ldg(p), b = __ldg(p + 1);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
}

// Magnitude key in the histogram's domain: bf16 -> 15-bit key, fp32 -> 31-bit.
template <qg_dtype DT>
__device__ __forceinline__ uint32_t mag_key(float x) {
    if constexpr (DT == QG_BF16) return (__float_as_uint(x) >> 16) & 0x7FFFu;
    else return __float_as_uint(x) & 0x7FFFFFFFu;
}

template <qg_dtype DT>
__device__ __forceinline__ float key_to_float(uint32_t key) {
    if constexpr (DT == QG_BF16) return __uint_as_float(key << 16);
    else return __uint_as_float(key);
}

// Keys at or above this are Inf/NaN.
template <qg_dtype DT>
__device__ __forceinline__ uint32_t nonfinite_key() {
    if constexpr (DT == QG_BF16) return 0x7F80u;
    else return 0x7F800000u;
}

// Per-16-bit-half unsigned maximum.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ int warp_inclusive_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        int t = __shfl_up_sync(0xFFFFFFFFu, v, d);
        if (lane >= d) v += t;
    }
    return v;
}

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, d));
    return v;
}

// ------------------------------------------------------- grid barrier
// For cooperative launches (every CTA resident).  A count and a generation
// word (GridSync, in the workspace status block, zero between barriers):
// grid_arrive returns true in the CTA that arrived last, which runs its
// serial work and calls grid_release; the other CTAs call grid_wait.  Waits
// are bounded: a CTA that gives up sets the timeout bit and must return.
constexpr long long kGridWaitLimit = 2000000000LL;   // SM clocks (~1-2 s)

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Arrive at a grid barrier.  Returns (in every thread) true in the CTA that
// arrived last, which then runs its serial work and calls grid_release; the
// others call grid_wait with gen0.  The arrival is an acq_rel atomic (this
// CTA's writes, ordered by bar.sync, are released; the last CTA acquires
// everyone's).
__device__ __forceinline__ bool grid_arrive(GridSync* g, uint32_t& gen0) {
    __shared__ int s_last;
    __shared__ uint32_t s_gen;
    __syncthreads();
    if (threadIdx.x == 0) {
        s_gen = ld_relaxed_u32(&g->gen);
        uint32_t old;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(&g->count) : "memory");
        s_last = (old == gridDim.x - 1) ? 1 : 0;
    }
    __syncthreads();
    gen0 = s_gen;
    return s_last != 0;
}
__device__ __forceinline__ void grid_release(GridSync* g) {
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(&g->count) : "memory");
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&g->gen) : "memory");
    }
}
__device__ __forceinline__ bool grid_wait(GridSync* g, uint32_t gen0, uint32_t* status) {
    __shared__ int s_ok;
    if (threadIdx.x == 0) {
        int ok = 1;
        const long long t0 = clock64();
        while (ld_acquire_u32(&g->gen) == gen0) {
            if (clock64() - t0 > kGridWaitLimit) {
                ok = 0;
                flag_status(status, kStatusTimeout);
                break;
            }
        }
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}


// Publish a flag value (thread 0, after every thread of the CTA is done with
// the writes it orders) and wait for it (thread 0 polls with a bound; every
// thread returns false when the wait gave up, after the timeout bit is set).
__device__ __forceinline__ void flag_publish(uint32_t* flag, uint32_t value) {
    __syncthreads();
    if (threadIdx.x == 0)
        asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(flag), "r"(value) : "memory");
}
__device__ __forceinline__ bool flag_wait(const uint32_t* flag, uint32_t want, uint32_t* status) {
    __shared__ int s_fok;
    if (threadIdx.x == 0) {
        int ok = 1;
        const long long t0 = clock64();
        while (ld_acquire_u32(flag) != want) {
            if (clock64() - t0 > kGridWaitLimit) {
                ok = 0;
                flag_status(status, kStatusTimeout);
                break;
            }
        }
        s_fok = ok;
    }
    __syncthreads();
    return s_fok != 0;
}

#endif  // __CUDACC__

// Pointers into a workspace for the threshold / clamp passes.
struct ActBuffers {
    uint32_t* status;
    GridSync* gsync;
    Counters* ctr;
    uint32_t* hist1;
    uint32_t* hist2;
    uint32_t* rowmax;
    uint32_t* rowcnt;
    uint32_t* rowpre;    // CTA-local prefix of the row counts (cooperative kernel)
    int32_t *st_row, *st_rank, *st_col;
    double* st_val;
    int64_t cap;
    int64_t row_slots;
};

// The layer's fp32 order switch: with at least this many clamped entries per
// row possible for every 4096 of K (n - ceil(alpha n) >= 10 M K / 4096), the
// GEMM writes Y first and the SpMM adds into it; below it, the SpMM writes Y
// and the GEMM adds its product into it.  Measured on the 7B block at
// M = 16384: on the K = 4096 layers GEMM first is 5-11 % faster at 20 entries
// per row and 2-6 % at 12, the two are within a few per cent at 8, and SpMM
// first is 5-11 % faster at 4; the K = 11008 layer favours SpMM first up to
// ~33 per row (the rule puts its switch at 27).  The crossover grows with K
// because the adding GEMM hides its reads of Y under more MMA work per tile.
constexpr int64_t kAddOrderEntriesPer4096K = 10;

inline bool linear_gemm_first(int64_t cap, int64_t M, int64_t K)
{
    return cap * 4096 >= kAddOrderEntriesPer4096K * M * K;
}

// QGEMM_NO_COOPERATIVE=1 in the environment (read when a device is first set
// up) makes the library treat the device as having no cooperative launch, so
// the bf16 activation and column quantizers take their multi-kernel
// sequences: the same results by other kernels, for testing those paths.
inline bool cooperative_disabled() {
    const char* v = getenv("QGEMM_NO_COOPERATIVE");
    return v != nullptr && v[0] == '1';
}

// Host-side argument checks shared by the C entry points.
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool dtype_ok(qg_dtype d) { return d == QG_F32 || d == QG_BF16; }
// Rows x K operand: K a multiple of 32 and at most 16384, both sizes positive.
inline qg_status check_mk(int64_t M, int64_t K) {
    if (M < 1 || K < 1) return QG_ERR_UNSUPPORTED_SHAPE;
    if (K % 32 != 0 || K > 16384) return QG_ERR_UNSUPPORTED_SHAPE;
    if (M > (int64_t)INT32_MAX - 1) return QG_ERR_UNSUPPORTED_SHAPE;
    return QG_OK;
}
inline qg_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QG_OK : QG_ERR_CUDA; }

// Launch sequences (kernel files) used by the C ABI layer.
void launch_zero_u32(uint32_t* p, int64_t n, cudaStream_t s);
void launch_e2m1_encode(const float* x, int64_t n, uint8_t* packed, cudaStream_t s);
void launch_quantize_rows(const void* A, qg_dtype dt, int64_t M, int64_t K, int64_t lda,
                          uint8_t* codes, float* scales, cudaStream_t s);
void launch_quantize_cols(const void* W, qg_dtype dt, int64_t K, int64_t N, int64_t ldw,
                          uint8_t* codesT, float* scales, uint32_t* colmax, cudaStream_t s);
void launch_spmm(const qg_csr* dA, int64_t M, const void* W, qg_dtype dt, int64_t N, int64_t ldw,
                 float* C, uint32_t* status, cudaStream_t s, bool add = false);
void launch_mx_quantize_rows(const void* A, qg_dtype dt, int64_t M, int64_t K, int64_t lda,
                             uint8_t* codes, uint8_t* sf, uint32_t* status, cudaStream_t s);
void launch_mx_quantize_cols(const void* W, qg_dtype dt, int64_t K, int64_t N, int64_t ldw,
                             uint8_t* codesT, uint8_t* sf, uint32_t* status, cudaStream_t s);
cudaError_t launch_fp4_gemm_mx(const uint8_t* codesA, const uint8_t* sfA, const uint8_t* codesWT,
                               const uint8_t* sfW, int64_t M, int64_t N, int64_t K, const float* C,
                               void* Y, qg_dtype y_dtype, float* raw_acc, uint32_t* status,
                               cudaStream_t s);
cudaError_t launch_fp4_gemm(const uint8_t* codesA, const float* sA, const uint8_t* codesWT,
                            const float* sW, int64_t M, int64_t N, int64_t K, const float* C,
                            void* Y, qg_dtype y_dtype, float* raw_acc, uint32_t* status,
                            cudaStream_t s, bool y_add = false);
cudaError_t launch_fp4_gemm_corr(const uint8_t* codesA, const float* sA, const uint8_t* codesWT,
                                 const float* sW, int64_t M, int64_t N, int64_t K,
                                 const qg_csr* dA, const void* W, qg_dtype w_dtype, int64_t ldw,
                                 float* scratch, void* Y, qg_dtype y_dtype, uint32_t* status,
                                 cudaStream_t s);
cudaError_t run_quantize_act(const void* A, qg_dtype dt, int64_t M, int64_t K, int64_t lda,
                             int64_t rank, const ActBuffers& b, uint8_t* codes, float* scales,
                             const qg_csr* dA, float* T_out, cudaStream_t s);
cudaError_t run_clamp_compensate(const void* A, qg_dtype dt, int64_t M, int64_t K, int64_t lda,
                                 int64_t rank, const ActBuffers& b, void* A_c, const qg_csr* dA,
                                 float* T_out, cudaStream_t s);
cudaError_t act_setup();
cudaError_t cols_setup();
bool launch_quantize_cols_fused(const void* W, int64_t K, int64_t N, int64_t ldw, uint8_t* codesT,
                                float* scales, uint32_t* colpart, GridSync* gsync,
                                uint32_t* status, cudaStream_t s);
cudaError_t gemm_setup();
cudaError_t spmm_setup();
// MMA-only loop on the tensor pipe (a CTA per SM, or 2-SM pairs); *flops gets
// the MMA flops of the launch.
cudaError_t launch_fp4_mma_loop(int64_t iters, bool pair, double* flops, float* acc_out,
                                uint32_t* status, cudaStream_t s);

// Number of SMs of the current device (cached per device id).
int num_sms();

// One-time per-device set-up of the library (kernel attributes, SM count),
// for the current device.
cudaError_t device_setup();

// Count kernel launches enqueued by this library (reported by qg_launch_count).
void count_launch(int n = 1);

}  // namespace qg
