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
// quantize pass knows amax_i = min(rowmax_i, T) without another reduction, and
// its last CTA to finish selects the bin (no separate launch).
//
// dA is emitted in canonical CSR order without sorting and without global
// atomics in the common case: one warp owns a row and walks it in column
// order, so each outlier knows its rank within the row; rank < row_slots goes
// to the row's own staging region, later ones to an overflow list.  The last
// CTA of the clamp pass scans the row counts into row_ptr; a scatter kernel
// then moves entry (row, rank) to row_ptr[row] + rank.
#include "qg_internal.cuh"

namespace qg {

constexpr int kHistThreads = 1024;
constexpr int kQuantThreads = 256;

// --------------------------------------------------------------------------
// Selection of the bin that holds the entry of rank `rank` (0-based) in a
// histogram of 1024 * PER bins, by one CTA of 1024 threads.  Reads go around
// L1 (the bins were just written by atomics).
struct SelectResult {
    uint32_t bin;
    unsigned long long below;   // entries in bins < bin
    int found;
};

template <int PER>
__device__ SelectResult block_select(const uint32_t* __restrict__ hist, unsigned long long rank) {
    // 1024 threads; warp w owns bins [w * 32 * PER, (w + 1) * 32 * PER); lane l
    // holds bins w * 32 * PER + 32 i + l, i < PER, in registers (one round of
    // coalesced loads), so the walk inside the chosen segment reloads nothing.
    __shared__ unsigned long long s_warp[32];
    __shared__ SelectResult s_res;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int seg = 32 * PER;
    const uint32_t* h = hist + (int64_t)warp * seg;
    uint32_t v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) v[i] = __ldcg(h + 32 * i + lane);
    unsigned long long mine = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) mine += v[i];
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) mine += __shfl_xor_sync(0xFFFFFFFFu, mine, d);
    if (lane == 0) s_warp[warp] = mine;
    if (t == 0) s_res.found = 0;
    __syncthreads();
    unsigned long long before = 0, incl = 0;
    for (int w = 0; w < 32; ++w) {
        const unsigned long long c = s_warp[w];
        if (w < warp) before += c;
        if (w <= warp) incl += c;
    }
    if (before <= rank && rank < incl) {
        // this warp's segment holds the rank: walk it 32 bins at a time
        unsigned long long cum = before;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const unsigned long long c = v[i];
            unsigned long long ci = c;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                unsigned long long u = __shfl_up_sync(0xFFFFFFFFu, ci, d);
                if (lane >= d) ci += u;
            }
            const unsigned long long ce = cum + ci - c;
            const unsigned hit = __ballot_sync(0xFFFFFFFFu, ce <= rank && rank < cum + ci);
            if (hit) {
                const int lb = __ffs(hit) - 1;
                if (lane == lb) {
                    s_res.bin = (uint32_t)(warp * seg + 32 * i + lb);
                    s_res.below = ce;
                    s_res.found = 1;
                }
                break;
            }
            cum += __shfl_sync(0xFFFFFFFFu, ci, 31);
        }
    }
    __syncthreads();
    return s_res;
}

// Store the selection.  MODE 0: bf16 threshold; 1: fp32 bucket; 2: fp32 threshold.
template <int MODE>
__device__ void finish_select(const SelectResult& r, Counters* ctr, uint32_t* status,
                              float* T_out) {
    if (threadIdx.x != 0) return;
    if (!r.found) {
        // the histogram does not hold rank + 1 entries: inconsistent input
        flag_status(status, kStatusOverflow);
        ctr->T_key = 0x7FFFFFFFu;
        if (MODE == 1) ctr->sel_bin = 0x7FFFu;
    } else if (MODE == 1) {
        ctr->sel_bin = r.bin;
        ctr->sel_below = r.below;
    } else {
        const uint32_t key = (MODE == 0) ? r.bin : ((ctr->sel_bin << 16) | r.bin);
        ctr->T_key = key;
        *T_out = (MODE == 0) ? __uint_as_float(key << 16) : __uint_as_float(key);
    }
    if (MODE != 1 && ctr->nonfinite) flag_status(status, kStatusNonFinite);
}

// True in the CTA that finished last (after all CTAs' global writes).
__device__ __forceinline__ bool last_block_done(uint32_t* counter) {
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(counter, 1u) == gridDim.x - 1);
    __syncthreads();
    if (s_last) __threadfence();
    return s_last != 0;
}

// --------------------------------------------------------------------------
// Pass 1: shared-memory histogram of the 15-bit keys + per-row max key; the
// last CTA selects the threshold bin (bf16) or the bucket (fp32).
template <qg_dtype DT>
__global__ void __launch_bounds__(kHistThreads, 1)
hist_rowmax_kernel(const void* __restrict__ A, int64_t lda, int M, int K,
                   uint32_t* __restrict__ ghist, uint32_t* __restrict__ rowmax,
                   Counters* __restrict__ ctr, unsigned long long rank,
                   uint32_t* __restrict__ status, float* __restrict__ T_out) {
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
    if (last_block_done(&ctr->done_hist)) {
        const SelectResult r = block_select<kHist1Bins / 1024>(ghist, rank);
        if (DT == QG_BF16) finish_select<0>(r, ctr, status, T_out);
        else finish_select<1>(r, ctr, status, T_out);
    }
}

// fp32 only: histogram of the low 16 key bits of the entries whose high bits
// equal the selected bucket; the last CTA selects the threshold.
__global__ void __launch_bounds__(kHistThreads)
refine_hist_kernel(const float* __restrict__ A, int64_t lda, int M, int K,
                   Counters* __restrict__ ctr, uint32_t* __restrict__ ghist2,
                   unsigned long long rank, uint32_t* __restrict__ status,
                   float* __restrict__ T_out) {
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
    if (last_block_done(&ctr->done_refine)) {
        const SelectResult r = block_select<kHist2Bins / 1024>(ghist2, rank - ctr->sel_below);
        finish_select<2>(r, ctr, status, T_out);
    }
}

// --------------------------------------------------------------------------
// Pass 2 (fused): clamp, row scale, E2M1 encode and dA staging.  One warp per
// row; per iteration a lane holds 4 groups of 8 consecutive elements, the
// groups of the warp covering 1024 consecutive columns.
//   WRITE_CODES = true : quantize_act (codes + scales)
//   WRITE_CODES = false: clamp_compensate (A_clamped in the input dtype)
// The last CTA to finish turns the row counts into row_ptr.
template <qg_dtype DT, bool WRITE_CODES>
__global__ void __launch_bounds__(kQuantThreads)
clamp_quant_kernel(const void* __restrict__ A, int64_t lda, int M, int K,
                   const uint32_t* __restrict__ rowmax, Counters* __restrict__ ctr,
                   uint8_t* __restrict__ codes, float* __restrict__ scales,
                   void* __restrict__ A_c, ActBuffers b, int32_t* __restrict__ row_ptr,
                   int64_t* __restrict__ nnz_out) {
    const uint32_t Tk = ctr->T_key;
    const float T = key_to_float<DT>(Tk);
    const int lane = threadIdx.x & 31;
    const int wpc = blockDim.x >> 5;
    const int total_warps = gridDim.x * wpc;
    const int nchunks = K / 8;
    const int row_slots = (int)b.row_slots;
    for (int row = blockIdx.x * wpc + (threadIdx.x >> 5); row < M; row += total_warps) {
        const int64_t base = (int64_t)row * lda;
        const uint32_t rmax = rowmax[row];
        const uint32_t akey = min(rmax, Tk);
        const bool any_out = rmax > Tk;
        float r = 0.0f, s = 0.0f;
        if (WRITE_CODES) {
            scale_factors(key_to_float<DT>(akey), r, s);
            if (lane == 0) scales[row] = s;
        }
        int32_t* rcol = b.st_col + (int64_t)row * row_slots;
        double* rval = b.st_val + (int64_t)row * row_slots;
        int row_rank = 0;
        for (int c0 = 0; c0 < nchunks; c0 += 128) {
            float x[4][8];
            uint32_t om[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + 32 * j + lane;
                om[j] = 0;
                if (c < nchunks) {
                    load8<DT>(A, base + (int64_t)c * 8, x[j]);
                    if (any_out) {
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            om[j] |= (mag_key<DT>(x[j][e]) > Tk ? 1u : 0u) << e;
                    }
                }
            }
            if (any_out) {
                // ranks of this iteration's outliers in column order
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int cnt = __popc(om[j]);
                    const int incl = warp_inclusive_scan(cnt);
                    int idx = row_rank + incl - cnt;
                    row_rank += __shfl_sync(0xFFFFFFFFu, incl, 31);
                    if (om[j] == 0) continue;
                    const int c = c0 + 32 * j + lane;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        if (!((om[j] >> e) & 1u)) continue;
                        const float a = x[j][e];
                        const double d = (double)a - (double)copysignf(T, a);
                        if (idx < row_slots) {
                            rcol[idx] = c * 8 + e;
                            rval[idx] = d;
                        } else {
                            const unsigned long long o = atomicAdd(&ctr->nnz, 1ull);
                            if (o < (unsigned long long)b.cap) {
                                const int64_t slot = (int64_t)M * row_slots + (int64_t)o;
                                b.st_row[o] = row;
                                b.st_rank[o] = idx;
                                b.st_col[slot] = c * 8 + e;
                                b.st_val[slot] = d;
                            } else {
                                flag_status(b.status, kStatusOverflow);
                            }
                        }
                        ++idx;
                    }
                }
            }
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
        if (lane == 0) b.rowcnt[row] = (uint32_t)row_rank;
    }

    // last CTA: row_ptr = exclusive scan of the row counts.  Thread t owns a
    // contiguous run of rows; its counts are read with independent loads (no
    // load waits on another), then written back as running sums.
    if (last_block_done(&ctr->done_clamp)) {
        __shared__ unsigned long long s_warp[kQuantThreads / 32];
        const int t = threadIdx.x, w = t >> 5;
        const int per = (M + kQuantThreads - 1) / kQuantThreads;
        const int r0 = min(M, t * per), r1 = min(M, r0 + per);
        unsigned long long mine = 0;
#pragma unroll 8
        for (int i = r0; i < r1; ++i) mine += __ldcg(b.rowcnt + i);
        unsigned long long v = mine;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            unsigned long long u = __shfl_up_sync(0xFFFFFFFFu, v, d);
            if (lane >= d) v += u;
        }
        if (lane == 31) s_warp[w] = v;
        __syncthreads();
        unsigned long long before = 0, total = 0;
        for (int i = 0; i < kQuantThreads / 32; ++i) {
            if (i < w) before += s_warp[i];
            total += s_warp[i];
        }
        unsigned long long run = before + v - mine;
#pragma unroll 8
        for (int i = r0; i < r1; ++i) {
            const uint32_t c = __ldcg(b.rowcnt + i);
            row_ptr[i] = (int32_t)run;
            run += c;
        }
        if (t == 0) {
            row_ptr[M] = (int32_t)total;
            *nnz_out = (int64_t)total;
            if (total > (unsigned long long)b.cap) flag_status(b.status, kStatusOverflow);
        }
    }
}

// Move staged entries to their CSR positions: a warp per row for the row
// regions, then a thread per overflow entry.
__global__ void __launch_bounds__(256)
csr_scatter_kernel(const Counters* __restrict__ ctr, ActBuffers b, int M,
                   const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col,
                   double* __restrict__ val) {
    const int lane = threadIdx.x & 31;
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nw = (gridDim.x * blockDim.x) >> 5;
    const int row_slots = (int)b.row_slots;
    for (int r = gw; r < M; r += nw) {
        const int n = min((int)b.rowcnt[r], row_slots);
        const int64_t dst = row_ptr[r];
        const int64_t src = (int64_t)r * row_slots;
        for (int j = lane; j < n; j += 32) {
            col[dst + j] = b.st_col[src + j];
            val[dst + j] = b.st_val[src + j];
        }
    }
    const unsigned long long n_over = min(ctr->nnz, (unsigned long long)b.cap);
    const int64_t base = (int64_t)M * row_slots;
    for (unsigned long long e = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x;
         e < n_over; e += (unsigned long long)gridDim.x * blockDim.x) {
        const int64_t dst = (int64_t)row_ptr[b.st_row[e]] + b.st_rank[e];
        col[dst] = b.st_col[base + e];
        val[dst] = b.st_val[base + e];
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
        hist_rowmax_kernel<QG_BF16><<<grid1, kHistThreads, shmem, s>>>(
            A, lda, (int)M, (int)K, b.hist1, b.rowmax, b.ctr, (unsigned long long)rank, b.status,
            T_out);
        count_launch(1);
    } else {
        hist_rowmax_kernel<QG_F32><<<grid1, kHistThreads, shmem, s>>>(
            A, lda, (int)M, (int)K, b.hist1, b.rowmax, b.ctr, (unsigned long long)rank, b.status,
            T_out);
        const int64_t work = M * (K / 8);
        const int g2 = (int)std::max<int64_t>(1, std::min<int64_t>((work + kHistThreads - 1) / kHistThreads, nsm * 2));
        refine_hist_kernel<<<g2, kHistThreads, 0, s>>>(static_cast<const float*>(A), lda, (int)M,
                                                       (int)K, b.ctr, b.hist2,
                                                       (unsigned long long)rank, b.status, T_out);
        count_launch(2);
    }
    return cudaGetLastError();
}

template <qg_dtype DT, bool CODES>
static void launch_clamp(const void* A, int64_t M, int64_t K, int64_t lda, const ActBuffers& b,
                         uint8_t* codes, float* scales, void* A_c, const qg_csr* dA,
                         cudaStream_t s) {
    const int wpc = kQuantThreads / 32;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((M + wpc - 1) / wpc, (int64_t)num_sms() * 8));
    clamp_quant_kernel<DT, CODES><<<grid, kQuantThreads, 0, s>>>(
        A, lda, (int)M, (int)K, b.rowmax, b.ctr, codes, scales, A_c, b, dA->row_ptr, dA->nnz_out);
    const int g2 = (int)std::max<int64_t>(1, std::min<int64_t>((M * 32 + 255) / 256, (int64_t)num_sms() * 8));
    csr_scatter_kernel<<<g2, 256, 0, s>>>(b.ctr, b, (int)M, dA->row_ptr, dA->col, dA->val);
    count_launch(2);
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
    if (dt == QG_BF16) launch_clamp<QG_BF16, true>(A, M, K, lda, b, codes, scales, nullptr, dA, s);
    else launch_clamp<QG_F32, true>(A, M, K, lda, b, codes, scales, nullptr, dA, s);
    return cudaGetLastError();
}

cudaError_t run_clamp_compensate(const void* A, qg_dtype dt, int64_t M, int64_t K, int64_t lda,
                                 int64_t rank, const ActBuffers& b, void* A_c, const qg_csr* dA,
                                 float* T_out, cudaStream_t s) {
    cudaError_t e = threshold_passes(A, dt, M, K, lda, rank, b, T_out, s);
    if (e != cudaSuccess) return e;
    if (dt == QG_BF16) launch_clamp<QG_BF16, false>(A, M, K, lda, b, nullptr, nullptr, A_c, dA, s);
    else launch_clamp<QG_F32, false>(A, M, K, lda, b, nullptr, nullptr, A_c, dA, s);
    return cudaGetLastError();
}

}  // namespace qg
