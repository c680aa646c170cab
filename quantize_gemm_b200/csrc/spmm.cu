// spmm.cu -- the compensation product C = dA . W of the FP4 linear layer.
//
// Method: QbitAI write-up of "Optimizing LLM Training Using FP4 Quantization"
// (news.movedaos.com/post/4103), outlier clamping and compensation paragraph:
// the clamped-off part dA = A - A_clamped is sparse and is multiplied in
// higher precision than FP4; here fp32 products and sums with W read in its
// stored dtype (bf16 or fp32).
//
// Work: 2 * nnz * N flops, and every non-zero (i, k) needs the whole row k of
// W, so the kernel streams W rows from L2.  Layout of the work:
//   * a CTA owns a 256-column slice of C for a block of 32 rows; blocks are
//     numbered row-block-fastest, so the CTAs in flight share one W slice
//     (K x 512 bytes for bf16) and it stays resident in L2;
//   * a warp owns one row at a time, each lane 8 consecutive columns (one
//     16-byte load per W row), accumulators in registers;
//   * the row's (col, val) entries are fetched 32 at a time, one per lane,
//     and broadcast with shuffles; four W rows are loaded before their FMAs
//     so each lane keeps four independent loads in flight.
// Rows without non-zeros write zeros, so C is fully defined.  The sum for one
// output is a chain of fp32 FMAs in the CSR order of the row.
#include "qg_internal.cuh"

namespace qg {

constexpr int kSpmmThreads = 256;
constexpr int kSpmmWarps = kSpmmThreads / 32;
constexpr int kSpmmSlice = 256;       // columns per CTA (32 lanes x 8)
constexpr int kSpmmRowsPerCta = 32;

// Y += v element by element in the memory system (red.global.add: fire and
// forget, the L2 adds; fp32 round to nearest, with subnormal sums flushed to
// zero).  Used when the compensation is added into an output that already
// holds the scaled FP4 product.
__device__ __forceinline__ void red_add4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}
__device__ __forceinline__ void red_add1(float* p, float a) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(a) : "memory");
}

template <qg_dtype DT>
__device__ __forceinline__ void load_w8(const void* W, int64_t idx, bool vec, int n0, int N,
                                        float (&w)[8]) {
    if (vec) {
        load8<DT>(W, idx, w);
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (n0 + e < N) {
                if constexpr (DT == QG_BF16)
                    w[e] = __uint_as_float((uint32_t)static_cast<const uint16_t*>(W)[idx + e] << 16);
                else
                    w[e] = static_cast<const float*>(W)[idx + e];
            } else {
                w[e] = 0.0f;
            }
        }
    }
}

template <qg_dtype DT, bool ADD>
__global__ void __launch_bounds__(kSpmmThreads)
spmm_slice_kernel(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col,
                  const double* __restrict__ val, const void* __restrict__ W, int64_t ldw, int M,
                  int N, float* __restrict__ C) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int n0 = blockIdx.y * kSpmmSlice + lane * 8;
    const bool col_ok = n0 < N;
    const bool vec = col_ok && (n0 + 8 <= N) && (N % 8) == 0 && (ldw % 8) == 0;
    const int r_end = min(M, (int)(blockIdx.x + 1) * kSpmmRowsPerCta);
    for (int r = blockIdx.x * kSpmmRowsPerCta + warp; r < r_end; r += kSpmmWarps) {
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
        const int p0 = row_ptr[r], p1 = row_ptr[r + 1];
        for (int pb = p0; pb < p1; pb += 32) {
            int myk = 0;
            float myv = 0.0f;
            if (pb + lane < p1) {
                myk = col[pb + lane];
                myv = (float)val[pb + lane];
            }
            const int cnt = min(32, p1 - pb);
            int q = 0;
            for (; q + 4 <= cnt; q += 4) {
                int k[4];
                float v[4], w[4][8];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    k[u] = __shfl_sync(0xFFFFFFFFu, myk, q + u);
                    v[u] = __shfl_sync(0xFFFFFFFFu, myv, q + u);
                }
                if (col_ok) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) load_w8<DT>(W, (int64_t)k[u] * ldw + n0, vec, n0, N, w[u]);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] = __fmaf_rn(v[u], w[u][e], acc[e]);
                }
            }
            for (; q < cnt; ++q) {
                const int k = __shfl_sync(0xFFFFFFFFu, myk, q);
                const float v = __shfl_sync(0xFFFFFFFFu, myv, q);
                if (col_ok) {
                    float w[8];
                    load_w8<DT>(W, (int64_t)k * ldw + n0, vec, n0, N, w);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[e] = __fmaf_rn(v, w[e], acc[e]);
                }
            }
        }
        if (!col_ok) continue;
        if (ADD && row_ptr[r] == row_ptr[r + 1]) continue;   // nothing to add
        float* crow = C + (int64_t)r * N + n0;
        if (ADD) {
            if (vec) {
                red_add4(crow, acc[0], acc[1], acc[2], acc[3]);
                red_add4(crow + 4, acc[4], acc[5], acc[6], acc[7]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (n0 + e < N) red_add1(crow + e, acc[e]);
            }
        } else if (vec) {
            float4* d = reinterpret_cast<float4*>(crow);
            d[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            d[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (n0 + e < N) crow[e] = acc[e];
        }
    }
}

// --------------------------------------------------------------------------
// Fast path (bf16 W, N and ldw multiples of 8).  The kernel is bound by
// instruction issue and L2 bandwidth at large shapes and by the latency of the
// W-row reads at small ones, so the work per non-zero is made as wide and as
// lean as possible and each warp keeps several rows' segments in flight: a CTA owns a 1024-column slice (each lane 32 columns, in four
// 256-column quarters so every load and store is coalesced), W row segments
// go straight from L2 into a register ring kDepth entries deep (the ring
// position is a compile-time index: the entry loop is unrolled by kDepth),
// and each bf16 pair feeds one packed fp32x2 FMA (one rounding per
// product-sum, as fmaf) on accumulators kept as 64-bit register pairs.
// A warp owns RPW consecutive rows, whose CSR entries form one contiguous
// range consumed in order.
constexpr int kStreamWarps = 8;
// A warp owns RPW consecutive rows (4, 2 or 1): the launcher takes the
// largest RPW that still gives every SM eight CTAs' worth of work, so narrow
// or short problems get more, smaller CTAs.  (8 or 16 rows per warp for
// short rows -- alpha 0.999, ~4 entries per row -- measured no faster.)
constexpr int kStreamMaxRowsPerWarp = 4;
#ifndef QG_SPMM_PARTS
#define QG_SPMM_PARTS 4
#endif
#ifndef QG_SPMM_DEPTH
#define QG_SPMM_DEPTH 4
#endif
constexpr int kStreamParts = QG_SPMM_PARTS;       // 256-column quarters per slice
constexpr int kStreamSlice = 256 * kStreamParts;
constexpr int kDepth = QG_SPMM_DEPTH;             // entries in flight per warp
static_assert(32 % kDepth == 0, "entry batches of 32 hold whole ring turns");

// acc += vv * (lo(w), hi(w)) for a bf16 pair w; acc and vv hold fp32 pairs.
// The low half can be moved up by a shift (which the compiler may place on
// the FMA pipe) or by a byte permute (ALU pipe); ALU_LO picks the second, so
// a caller can spread the unpacking over both pipes.
template <bool ALU_LO>
__device__ __forceinline__ void fma_bf16x2(uint64_t& acc, uint64_t vv, uint32_t w) {
    if (ALU_LO) {
        asm("{\n\t.reg .b32 lo, hi;\n\t.reg .b64 x;\n\t"
            "prmt.b32 lo, %2, 0, 0x1044;\n\tand.b32 hi, %2, 0xFFFF0000;\n\t"
            "mov.b64 x, {lo, hi};\n\tfma.rn.f32x2 %0, x, %1, %0;\n\t}"
            : "+l"(acc)
            : "l"(vv), "r"(w));
    } else {
        asm("{\n\t.reg .b32 lo, hi;\n\t.reg .b64 x;\n\t"
            "shl.b32 lo, %2, 16;\n\tand.b32 hi, %2, 0xFFFF0000;\n\t"
            "mov.b64 x, {lo, hi};\n\tfma.rn.f32x2 %0, x, %1, %0;\n\t}"
            : "+l"(acc)
            : "l"(vv), "r"(w));
    }
}
#ifndef QG_SPMM_ALU_WORDS
#define QG_SPMM_ALU_WORDS 1     // words per 16-byte segment unpacked on the ALU (0..4)
#endif

// FULL: every quarter of the slice is inside N (all slices but the last when
// N is not a multiple of the slice width), so loads and stores need no checks.
template <int RPW, bool FULL, bool ADD>
__device__ __forceinline__ void spmm_stream_body(const int32_t* __restrict__ row_ptr,
                                                 const int32_t* __restrict__ col,
                                                 const double* __restrict__ val,
                                                 const uint16_t* __restrict__ W, int64_t ldw,
                                                 int M, int N, float* __restrict__ C) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int r_begin = (blockIdx.x * kStreamWarps + warp) * RPW;
    if (r_begin >= M) return;
    const int r_end = min(M, r_begin + RPW);
    const int nbase = blockIdx.y * kStreamSlice + lane * 8;   // quarter h: nbase + 256 h
    bool okh[kStreamParts];
#pragma unroll
    for (int h = 0; h < kStreamParts; ++h) okh[h] = FULL || nbase + 256 * h < N;
    const uint16_t* wl = W + nbase;
    // row_ptr[r_begin .. r_end] held by lanes 0 .. RPW
    const int rp = (lane <= r_end - r_begin) ? row_ptr[r_begin + lane] : 0;
    const int P0 = __shfl_sync(0xFFFFFFFFu, rp, 0);
    const int n = __shfl_sync(0xFFFFFFFFu, rp, r_end - r_begin) - P0;
    // per batch of 32 entries B .. B + 31: lane l holds the value of entry
    // B + l (vc) and the column of entry B + kDepth + l (ks), the one whose
    // W segment is fetched while entry B + l is consumed
    int kc = (lane < n) ? col[P0 + lane] : 0;
    float vc = (lane < n) ? (float)val[P0 + lane] : 0.0f;
    int ks;
    {
        const int kn = (32 + lane < n) ? col[P0 + 32 + lane] : 0;
        const int a = __shfl_sync(0xFFFFFFFFu, kc, (lane + kDepth) & 31);
        const int b = __shfl_sync(0xFFFFFFFFu, kn, (lane + kDepth) & 31);
        ks = (lane + kDepth < 32) ? a : b;
    }

    uint4 buf[kDepth][kStreamParts];
    auto fetch = [&](uint4 (&d)[kStreamParts], int k) {
        const uint4* src = reinterpret_cast<const uint4*>(wl + (int64_t)k * ldw);
#pragma unroll
        for (int h = 0; h < kStreamParts; ++h) {
            if (FULL) d[h] = __ldg(src + 32 * h);
            else d[h] = okh[h] ? __ldg(src + 32 * h) : make_uint4(0u, 0u, 0u, 0u);
        }
    };
#pragma unroll
    for (int u = 0; u < kDepth; ++u)
        if (u < n) fetch(buf[u], __shfl_sync(0xFFFFFFFFu, kc, u));

    uint64_t acc[4 * kStreamParts];
#pragma unroll
    for (int e = 0; e < 4 * kStreamParts; ++e) acc[e] = 0ull;
    int row = r_begin;
    int rend = __shfl_sync(0xFFFFFFFFu, rp, 1) - P0;   // entries of rows <= row end here
    auto store_row = [&](int r) {
        float* crow = C + (int64_t)r * N + nbase;
        // ADD: a row without entries adds nothing (its accumulators are 0)
        const bool live = !ADD || __shfl_sync(0xFFFFFFFFu, rp, r - r_begin) !=
                                      __shfl_sync(0xFFFFFFFFu, rp, r - r_begin + 1);
#pragma unroll
        for (int h = 0; h < kStreamParts; ++h) {
            if (okh[h] && live) {
                if constexpr (ADD) {
                    float* d = crow + 256 * h;
                    red_add4(d, __uint_as_float((uint32_t)acc[4 * h + 0]),
                             __uint_as_float((uint32_t)(acc[4 * h + 0] >> 32)),
                             __uint_as_float((uint32_t)acc[4 * h + 1]),
                             __uint_as_float((uint32_t)(acc[4 * h + 1] >> 32)));
                    red_add4(d + 4, __uint_as_float((uint32_t)acc[4 * h + 2]),
                             __uint_as_float((uint32_t)(acc[4 * h + 2] >> 32)),
                             __uint_as_float((uint32_t)acc[4 * h + 3]),
                             __uint_as_float((uint32_t)(acc[4 * h + 3] >> 32)));
                } else {
                    ulonglong2* d = reinterpret_cast<ulonglong2*>(crow + 256 * h);
                    d[0] = make_ulonglong2(acc[4 * h + 0], acc[4 * h + 1]);
                    d[1] = make_ulonglong2(acc[4 * h + 2], acc[4 * h + 3]);
                }
            }
        }
#pragma unroll
        for (int e = 0; e < 4 * kStreamParts; ++e) acc[e] = 0ull;
    };
    for (int q = 0; q < n; q += kDepth) {
#pragma unroll
        for (int u = 0; u < kDepth; ++u) {
            const int j = q + u;                 // entry index within the warp's range
            if (j >= n) break;
            while (j >= rend) {                  // rows that end before entry j
                store_row(row);
                ++row;
                rend = __shfl_sync(0xFFFFFFFFu, rp, row - r_begin + 1) - P0;
            }
            const int t = (q & 31) + u;          // position in the batch
            const float v = __shfl_sync(0xFFFFFFFFu, vc, t);
            const int kf = __shfl_sync(0xFFFFFFFFu, ks, t);
            uint64_t vv;
            asm("mov.b64 %0, {%1, %1};" : "=l"(vv) : "f"(v));
#pragma unroll
            for (int h = 0; h < kStreamParts; ++h) {
                fma_bf16x2<(0 < QG_SPMM_ALU_WORDS)>(acc[4 * h + 0], vv, buf[u][h].x);
                fma_bf16x2<(1 < QG_SPMM_ALU_WORDS)>(acc[4 * h + 1], vv, buf[u][h].y);
                fma_bf16x2<(2 < QG_SPMM_ALU_WORDS)>(acc[4 * h + 2], vv, buf[u][h].z);
                fma_bf16x2<(3 < QG_SPMM_ALU_WORDS)>(acc[4 * h + 3], vv, buf[u][h].w);
            }
            // refill this ring position with entry j + kDepth
            if (j + kDepth < n) fetch(buf[u], kf);
        }
        if ((q & 31) == 32 - kDepth) {           // batch done: load the next one
            const int B = q + kDepth;
            kc = (B + lane < n) ? col[P0 + B + lane] : 0;
            vc = (B + lane < n) ? (float)val[P0 + B + lane] : 0.0f;
            const int kn = (B + 32 + lane < n) ? col[P0 + B + 32 + lane] : 0;
            const int a = __shfl_sync(0xFFFFFFFFu, kc, (lane + kDepth) & 31);
            const int b = __shfl_sync(0xFFFFFFFFu, kn, (lane + kDepth) & 31);
            ks = (lane + kDepth < 32) ? a : b;
        }
    }
    while (row < r_end) {                // the last rows (and empty ones)
        store_row(row);
        ++row;
    }
}

template <int RPW, bool ADD>
__global__ void __launch_bounds__(kStreamWarps * 32, 2)
spmm_stream_kernel(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col,
                   const double* __restrict__ val, const uint16_t* __restrict__ W, int64_t ldw,
                   int M, int N, float* __restrict__ C) {
    if ((int)(blockIdx.y + 1) * kStreamSlice <= N)
        spmm_stream_body<RPW, true, ADD>(row_ptr, col, val, W, ldw, M, N, C);
    else
        spmm_stream_body<RPW, false, ADD>(row_ptr, col, val, W, ldw, M, N, C);
}

cudaError_t spmm_setup() { return cudaSuccess; }

template <bool ADD>
static void launch_spmm_as(const qg_csr* dA, int64_t M, const void* W, qg_dtype dt, int64_t N,
                           int64_t ldw, float* C, cudaStream_t s) {
    if (dt == QG_BF16 && (N % 8) == 0 && (ldw % 8) == 0) {
        const int64_t slices = (N + kStreamSlice - 1) / kStreamSlice;
        const int64_t want = 8 * (int64_t)num_sms();
        int rpw = kStreamMaxRowsPerWarp;
        while (rpw > 1 && ((M + kStreamWarps * rpw - 1) / (kStreamWarps * rpw)) * slices < want) rpw /= 2;
        dim3 grid((unsigned)((M + kStreamWarps * rpw - 1) / (kStreamWarps * rpw)), (unsigned)slices);
        const uint16_t* Wb = static_cast<const uint16_t*>(W);
        if (rpw == 4)
            spmm_stream_kernel<4, ADD><<<grid, kStreamWarps * 32, 0, s>>>(dA->row_ptr, dA->col, dA->val, Wb, ldw, (int)M, (int)N, C);
        else if (rpw == 2)
            spmm_stream_kernel<2, ADD><<<grid, kStreamWarps * 32, 0, s>>>(dA->row_ptr, dA->col, dA->val, Wb, ldw, (int)M, (int)N, C);
        else
            spmm_stream_kernel<1, ADD><<<grid, kStreamWarps * 32, 0, s>>>(dA->row_ptr, dA->col, dA->val, Wb, ldw, (int)M, (int)N, C);
        count_launch(1);
        return;
    }
    dim3 grid((unsigned)((M + kSpmmRowsPerCta - 1) / kSpmmRowsPerCta),
              (unsigned)((N + kSpmmSlice - 1) / kSpmmSlice));
    if (dt == QG_BF16)
        spmm_slice_kernel<QG_BF16, ADD><<<grid, kSpmmThreads, 0, s>>>(dA->row_ptr, dA->col, dA->val, W,
                                                                       ldw, (int)M, (int)N, C);
    else
        spmm_slice_kernel<QG_F32, ADD><<<grid, kSpmmThreads, 0, s>>>(dA->row_ptr, dA->col, dA->val, W,
                                                                      ldw, (int)M, (int)N, C);
    count_launch(1);
}

// C = dA . W (add == false: every element of C written) or C += dA . W
// (add == true: rows with entries only, added by the memory system).
void launch_spmm(const qg_csr* dA, int64_t M, const void* W, qg_dtype dt, int64_t N, int64_t ldw,
                 float* C, uint32_t* status, cudaStream_t s, bool add) {
    (void)status;   // no device-side waits that could time out
    if (add) launch_spmm_as<true>(dA, M, W, dt, N, ldw, C, s);
    else launch_spmm_as<false>(dA, M, W, dt, N, ldw, C, s);
}

}  // namespace qg
