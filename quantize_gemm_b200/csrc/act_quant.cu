// act_quant.cu -- outlier threshold, clamp, sparse compensation and the fused
// token-wise activation quantizer.
//
// Method: QbitAI write-up of "Optimizing LLM Training Using FP4 Quantization"
// (news.movedaos.com/post/4103), outlier clamping and compensation
// paragraph: find the largest |A| by a quantile search, clamp them to the
// threshold (A_clamped), keep dA = A - A_clamped as a sparse matrix; then the
// granularity + ScaleShift paragraphs for the row quantization of A_clamped.
//
// The threshold is the exact order statistic T = sorted(|A|)[k] over the whole
// tensor, found by a radix histogram of the magnitude bit patterns (integer
// keys order like |x| for finite values):
//   bf16: one pass, 2^15 bins = every possible magnitude;
//   fp32: a 2^15-bin pass on bits 30..16, then a 2^16-bin pass on bits 15..0
//         restricted to the selected bucket.
// The pass that builds the histogram also keeps each row's max |a|, so the
// quantize pass knows amax_i = min(rowmax_i, T) without another reduction.
//
// dA is emitted in canonical CSR order without sorting: one warp owns a row
// and walks it in column order, so each outlier knows its rank within the row;
// entries go to a staging list through warp-aggregated slot reservation, and a
// final scatter puts entry (row, rank) at row_ptr[row] + rank.
#include "qg_internal.cuh"

namespace qg {

constexpr int kHistThreads = 1024;
constexpr int kQuantThreads = 256;

// --------------------------------------------------------------------------
// Pass 1: shared-memory histogram of the 15-bit keys + per-row max key.
template <qg_dtype DT>
__global__ void __launch_bounds__(kHistThreads, 1)
hist_rowmax_kernel(const void* __restrict__ A, int64_t lda, int M, int K,
                   uint32_t* __restrict__ ghist, uint32_t* __restrict__ rowmax,
                   Counters* __restrict__ ctr) {
    extern __shared__ uint32_t sh_hist[];
    for (int i = threadIdx.x; i < kHist1Bins; i += blockDim.x) sh_hist[i] = 0u;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int wpc = blockDim.x >> 5;
    const int total_warps = gridDim.x * wpc;
    const int nchunks = K / 8;
    uint32_t bad = 0;
    for (int row = blockIdx.x * wpc + (threadIdx.x >> 5); row < M; row += total_warps) {
        const int64_t base = (int64_t)row * lda;
        uint32_t kmax = 0;
        for (int c0 = 0; c0 < nchunks; c0 += 128) {
            float x[4][8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + 32 * j + lane;
                if (c < nchunks) load8<DT>(A, base + (int64_t)c * 8, x[j]);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + 32 * j + lane;
                if (c < nchunks) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const uint32_t k = mag_key<DT>(x[j][e]);
                        kmax = max(kmax, k);
                        const uint32_t bin = (DT == QG_BF16) ? k : (k >> 16);
                        atomicAdd(&sh_hist[bin], 1u);
                    }
                }
            }
        }
        kmax = warp_max_u32(kmax);
        if (lane == 0) rowmax[row] = kmax;
        bad |= (kmax >= nonfinite_key<DT>()) ? 1u : 0u;
    }
    if (bad && lane == 0) atomicOr(&ctr->nonfinite, 1u);
    __syncthreads();
    for (int i = threadIdx.x; i < kHist1Bins; i += blockDim.x) {
        const uint32_t v = sh_hist[i];
        if (v) atomicAdd(&ghist[i], v);
    }
}

// fp32 only: histogram of the low 16 key bits of the entries whose high bits
// equal the bucket chosen by the first selection.
__global__ void __launch_bounds__(256)
refine_hist_kernel(const float* __restrict__ A, int64_t lda, int M, int K,
                   const Counters* __restrict__ ctr, uint32_t* __restrict__ ghist2) {
    const uint32_t hi = ctr->sel_bin;
    const int nchunks = K / 8;
    const int64_t total = (int64_t)M * nchunks;
    for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
         t += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = t / nchunks;
        const int c = (int)(t - row * nchunks);
        float x[8];
        load8<QG_F32>(A, row * lda + (int64_t)c * 8, x);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t k = key_of(x[e]);
            if ((k >> 16) == hi) atomicAdd(&ghist2[k & 0xFFFFu], 1u);
        }
    }
}

// --------------------------------------------------------------------------
// Selection: the bin holding the entry of rank `rank` (0-based) in a
// histogram.  One CTA; each thread owns a run of consecutive bins.
//   mode 0: bf16, bins are full keys           -> T
//   mode 1: fp32 level 1 (bits 30..16)         -> sel_bin, sel_below
//   mode 2: fp32 level 2 (bits 15..0) of rank - sel_below in bucket sel_bin -> T
template <int MODE>
__global__ void __launch_bounds__(1024)
select_kernel(const uint32_t* __restrict__ hist, int nbins, unsigned long long rank,
              Counters* __restrict__ ctr, uint32_t* __restrict__ status, float* __restrict__ T_out) {
    __shared__ unsigned long long warp_tot[32];
    __shared__ int found;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    if (MODE == 2) rank -= ctr->sel_below;
    if (t == 0) found = 0;
    const int per = nbins / 1024;
    const uint32_t* h = hist + (int64_t)t * per;
    unsigned long long mine = 0;
    for (int i = 0; i < per; ++i) mine += h[i];
    // block-wide inclusive scan of `mine`
    unsigned long long v = mine;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        unsigned long long u = __shfl_up_sync(0xFFFFFFFFu, v, d);
        if (lane >= d) v += u;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        unsigned long long w = warp_tot[lane];
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            unsigned long long u = __shfl_up_sync(0xFFFFFFFFu, w, d);
            if (lane >= d) w += u;
        }
        warp_tot[lane] = w;
    }
    __syncthreads();
    const unsigned long long incl = v + (warp > 0 ? warp_tot[warp - 1] : 0ull);
    const unsigned long long excl = incl - mine;
    if (excl <= rank && rank < incl) {
        unsigned long long cum = excl;
        int b = 0;
        for (; b < per; ++b) {
            if (rank < cum + h[b]) break;
            cum += h[b];
        }
        const uint32_t bin = (uint32_t)(t * per + b);
        found = 1;
        if (MODE == 1) {
            ctr->sel_bin = bin;
            ctr->sel_below = cum;
        } else {
            const uint32_t key = (MODE == 0) ? bin : ((ctr->sel_bin << 16) | bin);
            ctr->T_key = key;
            *T_out = (MODE == 0) ? __uint_as_float(key << 16) : __uint_as_float(key);
        }
    }
    __syncthreads();
    if (t == 0) {
        if (!found) {
            // the histogram does not hold rank+1 entries: inconsistent input
            flag_status(status, kStatusOverflow);
            ctr->T_key = 0x7FFFFFFFu;
            if (MODE == 1) ctr->sel_bin = 0x7FFFu;
        }
        if (MODE != 1 && ctr->nonfinite) flag_status(status, kStatusNonFinite);
    }
}

// --------------------------------------------------------------------------
// Pass 2 (fused): clamp, row scale, E2M1 encode and dA staging.  One warp per
// row; per iteration a lane holds 4 groups of 8 consecutive elements, the
// groups of the warp covering 1024 consecutive columns.
//   WRITE_CODES = true : quantize_act (codes + scales)
//   WRITE_CODES = false: clamp_compensate (A_clamped in the input dtype)
template <qg_dtype DT, bool WRITE_CODES>
__global__ void __launch_bounds__(kQuantThreads)
clamp_quant_kernel(const void* __restrict__ A, int64_t lda, int M, int K,
                   const uint32_t* __restrict__ rowmax, Counters* __restrict__ ctr,
                   uint8_t* __restrict__ codes, float* __restrict__ scales,
                   void* __restrict__ A_c,
                   int32_t* __restrict__ st_row, int32_t* __restrict__ st_rank,
                   int32_t* __restrict__ st_col, double* __restrict__ st_val, int64_t cap,
                   uint32_t* __restrict__ rowcnt, uint32_t* __restrict__ status) {
    const uint32_t Tk = ctr->T_key;
    const float T = key_to_float<DT>(Tk);
    const int lane = threadIdx.x & 31;
    const int wpc = blockDim.x >> 5;
    const int total_warps = gridDim.x * wpc;
    const int nchunks = K / 8;
    for (int row = blockIdx.x * wpc + (threadIdx.x >> 5); row < M; row += total_warps) {
        const int64_t base = (int64_t)row * lda;
        const uint32_t akey = min(rowmax[row], Tk);
        float r = 0.0f, s = 0.0f;
        if (WRITE_CODES) {
            scale_factors(key_to_float<DT>(akey), r, s);
            if (lane == 0) scales[row] = s;
        }
        int row_rank = 0;
        for (int c0 = 0; c0 < nchunks; c0 += 128) {
            float x[4][8];
            uint32_t om[4];
            int cnt[4], ex[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + 32 * j + lane;
                om[j] = 0;
                if (c < nchunks) {
                    load8<DT>(A, base + (int64_t)c * 8, x[j]);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        om[j] |= (mag_key<DT>(x[j][e]) > Tk ? 1u : 0u) << e;
                }
            }
            // ranks of this iteration's outliers in column order
            int iter_total = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                cnt[j] = __popc(om[j]);
                const int incl = warp_inclusive_scan(cnt[j]);
                ex[j] = iter_total + incl - cnt[j];
                iter_total += __shfl_sync(0xFFFFFFFFu, incl, 31);
            }
            if (iter_total > 0) {
                unsigned long long slot0 = 0;
                if (lane == 0) slot0 = atomicAdd(&ctr->nnz, (unsigned long long)iter_total);
                slot0 = __shfl_sync(0xFFFFFFFFu, slot0, 0);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (om[j] == 0) continue;
                    int idx = ex[j];
                    const int c = c0 + 32 * j + lane;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        if (!((om[j] >> e) & 1u)) continue;
                        const unsigned long long slot = slot0 + (unsigned long long)idx;
                        if (slot < (unsigned long long)cap) {
                            const float a = x[j][e];
                            st_row[slot] = row;
                            st_rank[slot] = row_rank + idx;
                            st_col[slot] = c * 8 + e;
                            st_val[slot] = (double)a - (double)copysignf(T, a);
                        } else {
                            flag_status(status, kStatusOverflow);
                        }
                        ++idx;
                    }
                }
            }
            row_rank += iter_total;
            // clamp, then encode (or store the clamped values)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + 32 * j + lane;
                if (c >= nchunks) continue;
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if ((om[j] >> e) & 1u) x[j][e] = copysignf(T, x[j][e]);
                if (WRITE_CODES) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = __fmul_rn(x[j][e], r);
                    reinterpret_cast<uint32_t*>(codes + (int64_t)row * (K / 2))[c] = e2m1x8(y);
                } else if (A_c == nullptr) {
                    continue;
                } else if (DT == QG_BF16) {
                    uint32_t w[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        w[i] = (__float_as_uint(x[j][2 * i]) >> 16) |
                               (__float_as_uint(x[j][2 * i + 1]) & 0xFFFF0000u);
                    reinterpret_cast<uint4*>(static_cast<uint16_t*>(A_c) + (int64_t)row * K)[c] =
                        make_uint4(w[0], w[1], w[2], w[3]);
                } else {
                    float4* d = reinterpret_cast<float4*>(static_cast<float*>(A_c) + (int64_t)row * K) + 2 * c;
                    d[0] = make_float4(x[j][0], x[j][1], x[j][2], x[j][3]);
                    d[1] = make_float4(x[j][4], x[j][5], x[j][6], x[j][7]);
                }
            }
        }
        if (lane == 0) rowcnt[row] = (uint32_t)row_rank;
    }
}

// --------------------------------------------------------------------------
// CSR finalize: row_ptr = exclusive scan of the row counts (one CTA), then
// scatter each staged entry to row_ptr[row] + rank.
__global__ void __launch_bounds__(1024)
csr_scan_kernel(const uint32_t* __restrict__ rowcnt, int M, int32_t* __restrict__ row_ptr,
                int64_t* __restrict__ nnz_out, const Counters* __restrict__ ctr, int64_t cap,
                uint32_t* __restrict__ status) {
    __shared__ unsigned long long warp_tot[32];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int per = (M + 1023) / 1024;
    const int r0 = min(M, t * per), r1 = min(M, r0 + per);
    unsigned long long mine = 0;
    for (int i = r0; i < r1; ++i) mine += rowcnt[i];
    unsigned long long v = mine;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        unsigned long long u = __shfl_up_sync(0xFFFFFFFFu, v, d);
        if (lane >= d) v += u;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        unsigned long long w = warp_tot[lane];
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            unsigned long long u = __shfl_up_sync(0xFFFFFFFFu, w, d);
            if (lane >= d) w += u;
        }
        warp_tot[lane] = w;
    }
    __syncthreads();
    unsigned long long run = v + (warp > 0 ? warp_tot[warp - 1] : 0ull) - mine;
    for (int i = r0; i < r1; ++i) {
        row_ptr[i] = (int32_t)run;
        run += rowcnt[i];
    }
    if (t == 1023) {
        const unsigned long long total = warp_tot[31];
        row_ptr[M] = (int32_t)total;
        *nnz_out = (int64_t)total;
        if (total != ctr->nnz || total > (unsigned long long)cap) flag_status(status, kStatusOverflow);
    }
}

__global__ void __launch_bounds__(256)
csr_scatter_kernel(const Counters* __restrict__ ctr, int64_t cap,
                   const int32_t* __restrict__ st_row, const int32_t* __restrict__ st_rank,
                   const int32_t* __restrict__ st_col, const double* __restrict__ st_val,
                   const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col,
                   double* __restrict__ val) {
    const unsigned long long n = min(ctr->nnz, (unsigned long long)cap);
    for (unsigned long long e = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; e < n;
         e += (unsigned long long)gridDim.x * blockDim.x) {
        const int64_t dst = (int64_t)row_ptr[st_row[e]] + st_rank[e];
        col[dst] = st_col[e];
        val[dst] = st_val[e];
    }
}

// --------------------------------------------------------------------------
// Host-side sequences.
static cudaError_t threshold_passes(const void* A, qg_dtype dt, int64_t M, int64_t K,
                                    int64_t lda, int64_t rank, const ActBuffers& b, float* T_out,
                                    cudaStream_t s) {
    // counters and histograms are contiguous in the workspace
    uint32_t* zbeg = reinterpret_cast<uint32_t*>(b.ctr);
    uint32_t* zend = (dt == QG_F32 ? b.hist2 + kHist2Bins : b.hist1 + kHist1Bins);
    launch_zero_u32(zbeg, zend - zbeg, s);
    const int nsm = num_sms();
    const int grid1 = (int)std::min<int64_t>(nsm, (M + 31) / 32);
    const size_t shmem = sizeof(uint32_t) * kHist1Bins;
    if (dt == QG_BF16) {
        hist_rowmax_kernel<QG_BF16><<<grid1, kHistThreads, shmem, s>>>(A, lda, (int)M, (int)K,
                                                                      b.hist1, b.rowmax, b.ctr);
        select_kernel<0><<<1, 1024, 0, s>>>(b.hist1, kHist1Bins, (unsigned long long)rank, b.ctr,
                                            b.status, T_out);
        count_launch(2);
    } else {
        hist_rowmax_kernel<QG_F32><<<grid1, kHistThreads, shmem, s>>>(A, lda, (int)M, (int)K,
                                                                     b.hist1, b.rowmax, b.ctr);
        select_kernel<1><<<1, 1024, 0, s>>>(b.hist1, kHist1Bins, (unsigned long long)rank, b.ctr,
                                            b.status, T_out);
        const int64_t work = M * (K / 8);
        const int g2 = (int)std::max<int64_t>(1, std::min<int64_t>((work + 255) / 256, nsm * 8));
        refine_hist_kernel<<<g2, 256, 0, s>>>(static_cast<const float*>(A), lda, (int)M, (int)K,
                                              b.ctr, b.hist2);
        select_kernel<2><<<1, 1024, 0, s>>>(b.hist2, kHist2Bins, (unsigned long long)rank, b.ctr,
                                            b.status, T_out);
        count_launch(4);
    }
    return cudaGetLastError();
}

static void finalize_csr(int64_t M, const ActBuffers& b, const qg_csr* dA, cudaStream_t s) {
    csr_scan_kernel<<<1, 1024, 0, s>>>(b.rowcnt, (int)M, dA->row_ptr, dA->nnz_out, b.ctr, b.cap,
                                       b.status);
    const int grid = std::max(1, num_sms() * 4);
    csr_scatter_kernel<<<grid, 256, 0, s>>>(b.ctr, b.cap, b.st_row, b.st_rank, b.st_col, b.st_val,
                                            dA->row_ptr, dA->col, dA->val);
    count_launch(2);
}

template <qg_dtype DT, bool CODES>
static void launch_clamp(const void* A, int64_t M, int64_t K, int64_t lda, const ActBuffers& b,
                         uint8_t* codes, float* scales, void* A_c, cudaStream_t s) {
    const int wpc = kQuantThreads / 32;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((M + wpc - 1) / wpc, (int64_t)num_sms() * 8));
    clamp_quant_kernel<DT, CODES><<<grid, kQuantThreads, 0, s>>>(
        A, lda, (int)M, (int)K, b.rowmax, b.ctr, codes, scales, A_c, b.st_row, b.st_rank, b.st_col,
        b.st_val, b.cap, b.rowcnt, b.status);
    count_launch(1);
}

cudaError_t act_setup() {
    cudaError_t e = cudaFuncSetAttribute(hist_rowmax_kernel<QG_BF16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(sizeof(uint32_t) * kHist1Bins));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(hist_rowmax_kernel<QG_F32>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(sizeof(uint32_t) * kHist1Bins));
}

cudaError_t run_quantize_act(const void* A, qg_dtype dt, int64_t M, int64_t K, int64_t lda,
                             int64_t rank, const ActBuffers& b, uint8_t* codes, float* scales,
                             const qg_csr* dA, float* T_out, cudaStream_t s) {
    cudaError_t e = threshold_passes(A, dt, M, K, lda, rank, b, T_out, s);
    if (e != cudaSuccess) return e;
    if (dt == QG_BF16) launch_clamp<QG_BF16, true>(A, M, K, lda, b, codes, scales, nullptr, s);
    else launch_clamp<QG_F32, true>(A, M, K, lda, b, codes, scales, nullptr, s);
    finalize_csr(M, b, dA, s);
    return cudaGetLastError();
}

cudaError_t run_clamp_compensate(const void* A, qg_dtype dt, int64_t M, int64_t K, int64_t lda,
                                 int64_t rank, const ActBuffers& b, void* A_c, const qg_csr* dA,
                                 float* T_out, cudaStream_t s) {
    cudaError_t e = threshold_passes(A, dt, M, K, lda, rank, b, T_out, s);
    if (e != cudaSuccess) return e;
    if (dt == QG_BF16) launch_clamp<QG_BF16, false>(A, M, K, lda, b, nullptr, nullptr, A_c, s);
    else launch_clamp<QG_F32, false>(A, M, K, lda, b, nullptr, nullptr, A_c, s);
    finalize_csr(M, b, dA, s);
    return cudaGetLastError();
}

}  // namespace qg
