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
// tensor; integer keys (the magnitude bit patterns) order like |x| for finite
// values.
//   bf16: a sample of A puts a band of at most 4096 keys around the sample
//         quantile; one pass counts the keys below the band and histograms
//         the keys inside it (SWAR on packed bf16 pairs), and the order
//         statistic is selected from the band -- or, when it is not inside
//         it, by an exact two-level count over all of A (same result).
//   fp32: a 2^15-bin pass on bits 30..16, then a 2^16-bin pass on bits 15..0
//         restricted to the selected bucket.
// The pass that finds T also keeps each row's max |a|, so the quantize pass
// knows amax_i = min(rowmax_i, T) without another reduction.
//
// dA is emitted in canonical CSR order without sorting: one warp owns a row
// and walks it in column order, so each outlier knows its rank within the
// row; rank < row_slots goes to the row's own staging region, later ones to
// an overflow list.  The row counts are scanned into row_ptr and a scatter
// moves entry (row, rank) to row_ptr[row] + rank.
//
// bf16 quantize_act runs as one cooperative kernel (act_fused_bf16_kernel,
// phases separated by bounded grid barriers); fp32 input, clamp_compensate
// and devices without cooperative launch use the multi-kernel sequence.
#include "qg_internal.cuh"

namespace qg {

constexpr int kHistThreads = 1024;
constexpr int kQuantThreads = 256;

// --------------------------------------------------------------------------
// Selection of the bin that holds the entry of rank `rank` (0-based) in a
// histogram of NT * PER bins, by one CTA of NT threads.  Reads go around L1
// (the bins were just written by atomics, maybe by other SMs).
struct SelectResult {
    uint32_t bin;
    unsigned long long below;   // entries in bins < bin
    int found;
};

template <int PER, bool SMEM = false, int NT = 1024>
__device__ SelectResult block_select(const uint32_t* __restrict__ hist, unsigned long long rank) {
    // NT threads; warp w owns bins [w * 32 * PER, (w + 1) * 32 * PER); lane l
    // holds bins w * 32 * PER + 32 i + l, i < PER, in registers (one round of
    // coalesced loads), so the walk inside the chosen segment reloads nothing.
    constexpr int NW = NT / 32;
    __shared__ unsigned long long s_warp[NW];
    __shared__ SelectResult s_res;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int seg = 32 * PER;
    const uint32_t* h = hist + (int64_t)warp * seg;
    uint32_t v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) v[i] = SMEM ? h[32 * i + lane] : __ldcg(h + 32 * i + lane);
    unsigned long long mine = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) mine += v[i];
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) mine += __shfl_xor_sync(0xFFFFFFFFu, mine, d);
    if (lane == 0) s_warp[warp] = mine;
    if (t == 0) s_res.found = 0;
    __syncthreads();
    unsigned long long before = 0, incl = 0;
    for (int w = 0; w < NW; ++w) {
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
        const uint32_t key = (MODE == 0) ? r.bin : ((__ldcg(&ctr->sel_bin) << 16) | r.bin);
        ctr->T_key = key;
        *T_out = (MODE == 0) ? __uint_as_float(key << 16) : __uint_as_float(key);
    }
    if (MODE != 1 && __ldcg(&ctr->nonfinite)) flag_status(status, kStatusNonFinite);
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

// --------------------------------------------------------------------------
// bf16 threshold by a band histogram.  A full 2^15-bin histogram costs one
// shared-memory atomic per element; here only the elements whose key falls in
// a narrow band around the order statistic take one, the rest are counted
// with SWAR arithmetic on the packed bf16 pairs.  The band comes from a
// sample of A; the result does not depend on it: when the order
// statistic is not inside the band, an exact two-level count over all of A
// takes its place (slow, but exact).
//
// SWAR compare of the two 15-bit keys of m = w & 0x7FFF7FFF with a constant
// c in [0, 0x7FFF]: key + (0x8000 - c) sets bit 15 of its half iff key >= c,
// and key + (0x7FFF - c) iff key > c; no sum leaves its 16-bit half.
constexpr int kBandBins = 4096;            // band width in keys
constexpr int kBandThreads = 1024;
constexpr int kSampleBins = 4096;          // sample histogram of key >> 3
constexpr int64_t kSampleTarget = 8192;    // sampled elements
constexpr int kSampleRows = 64;            // from this many rows

__device__ __forceinline__ uint32_t swar_ge(uint32_t m, uint32_t c) {
    return (m + (0x8000u - c) * 0x10001u) & 0x80008000u;
}
__device__ __forceinline__ uint32_t swar_gt(uint32_t m, uint32_t c) {
    return (m + (0x7FFFu - c) * 0x10001u) & 0x80008000u;
}

// Bins of a 4096-bin shared histogram holding the entries of ranks r[0..2]
// (each r < total), by NT threads: thread t owns 4096 / NT consecutive bins;
// one block scan.
template <int NT>
__device__ void block_select3(const uint32_t* sh, const unsigned long long (&r)[3],
                              uint32_t* s_out /* 3 entries, shared */) {
    constexpr int B = kSampleBins / NT;
    __shared__ uint32_t s_w[NT / 32];
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    uint32_t b[B];
#pragma unroll
    for (int i = 0; i < B / 4; ++i) {
        const uint4 v = reinterpret_cast<const uint4*>(sh)[t * (B / 4) + i];
        b[4 * i] = v.x;
        b[4 * i + 1] = v.y;
        b[4 * i + 2] = v.z;
        b[4 * i + 3] = v.w;
    }
    uint32_t mine = 0;
#pragma unroll
    for (int i = 0; i < B; ++i) mine += b[i];
    const uint32_t incl = (uint32_t)warp_inclusive_scan((int)mine);
    if (lane == 31) s_w[w] = incl;
    __syncthreads();
    uint32_t before = 0;
    for (int i = 0; i < w; ++i) before += s_w[i];
    uint32_t c = before + incl - mine;   // entries in bins < B t
#pragma unroll
    for (int q = 0; q < B; ++q) {
#pragma unroll
        for (int k = 0; k < 3; ++k)
            if (c <= r[k] && r[k] < (unsigned long long)c + b[q]) s_out[k] = B * t + q;
        c += b[q];
    }
    __syncthreads();
}

// One CTA of NT threads: histogram the keys >> 3 of a sample (windows of 64
// rows spread evenly over A) in sh, and put the band around the sample
// quantile with a margin of six standard deviations of a sample quantile's
// rank plus 32.  A margin that runs past the sample's largest (smallest) key
// opens the band upwards (downwards), up to its 4096-key width, so an extreme
// quantile is not missed for want of sampled keys above it.  Writes nothing
// but sh: every CTA that runs it on the same A gets the same band.
template <int NT>
__device__ void cta_band_local(const uint16_t* __restrict__ A, int64_t lda, int M, int K,
                               unsigned long long rank, uint32_t* sh, uint32_t& lo_out,
                               uint32_t& hi_out) {
    __shared__ uint32_t s_sel[3];
    __shared__ uint32_t s_band[2];
    const int t = threadIdx.x;
    // R rows evenly spaced over M (row ri * M / R); from each a window of cpr
    // 16-byte chunks whose start moves from row to row
    const int nch = K / 8;
    const int R = M < kSampleRows ? M : kSampleRows;
    const int per_row = (int)((kSampleTarget / 8 + R - 1) / R);
    const int cpr = nch < per_row ? nch : per_row;
    const int total = R * cpr;
    const int mq = M / R, mr = M % R;
    constexpr int U = (int)((kSampleTarget / 8 + NT - 1) / NT);   // loads per thread per round
    for (int i = t; i < kSampleBins; i += NT) sh[i] = 0u;
    if (t < 3) s_sel[t] = 0u;
    __syncthreads();
    for (int q0 = t; q0 < total; q0 += U * NT) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int q = q0 + u * NT;
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (q < total) {
                const int ri = q / cpr;
                const int off = (ri * 977) % (nch - cpr + 1);
                const int c = off + (q - ri * cpr);
                const int64_t row = (int64_t)ri * mq + (ri * mr) / R;
                v[u] = __ldg(reinterpret_cast<const uint4*>(A + row * lda) + c);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (q0 + u * NT >= total) continue;
            const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                atomicAdd(&sh[(w[i] & 0x7FFFu) >> 3], 1u);
                atomicAdd(&sh[(w[i] >> 19) & 0xFFFu], 1u);
            }
        }
    }
    __syncthreads();
    const double n = (double)M * (double)K;
    const double ns = (double)total * 8.0;
    const double p = ((double)rank + 0.5) / n;
    const double center = p * ns;
    const double margin = 6.0 * sqrt(ns * p * (1.0 - p)) + 32.0;
    const double top = ns - 1.0;
    const unsigned long long r[3] = {
        (unsigned long long)fmin(fmax(floor(center - margin), 0.0), top),
        (unsigned long long)fmin(fmax(ceil(center + margin), 0.0), top),
        (unsigned long long)fmin(fmax(center, 0.0), top)};
    block_select3<NT>(sh, r, s_sel);
    if (t == 0) {
        uint32_t lo = s_sel[0] << 3, hi = (s_sel[1] << 3) + 7u;
        const uint32_t mid = s_sel[2] << 3;
        if (center + margin >= top) hi = 0x7FFFu;
        if (center - margin <= 0.0) lo = 0u;
        if (hi - lo + 1 > (uint32_t)kBandBins) {
            lo = max(lo, mid > (uint32_t)(kBandBins / 2) ? mid - kBandBins / 2 : 0u);
            hi = min(hi, lo + kBandBins - 1);
        }
        s_band[0] = lo;
        s_band[1] = hi;
    }
    __syncthreads();
    lo_out = s_band[0];
    hi_out = s_band[1];
    __syncthreads();   // sh and s_band may be reused
}

// The same band, with the counters and band bins zeroed and the band stored
// in the counters (the one-CTA kernel of the multi-kernel sequence).
template <int NT>
__device__ void cta_sample_band(const uint16_t* __restrict__ A, int64_t lda, int M, int K,
                                Counters* __restrict__ ctr, uint32_t* __restrict__ band_bins,
                                unsigned long long rank, uint32_t* sh) {
    uint32_t* cz = reinterpret_cast<uint32_t*>(ctr);
    for (int i = threadIdx.x; i < (int)(sizeof(Counters) / 4); i += NT) cz[i] = 0u;
    for (int i = threadIdx.x; i < kBandBins; i += NT) band_bins[i] = 0u;
    uint32_t lo, hi;
    cta_band_local<NT>(A, lda, M, K, rank, sh, lo, hi);
    if (threadIdx.x == 0) {
        ctr->band_lo = lo;
        ctr->band_hi = hi;
    }
}

__global__ void __launch_bounds__(kBandThreads, 1)
band_prep_kernel(const uint16_t* __restrict__ A, int64_t lda, int M, int K,
                 Counters* __restrict__ ctr, uint32_t* __restrict__ band_bins,
                 unsigned long long rank) {
    __shared__ __align__(16) uint32_t sh[kSampleBins];
    cta_sample_band<kBandThreads>(A, lda, M, K, ctr, band_bins, rank, sh);
}

// Exact selection of the key of rank `rank` over all of A by one CTA of NT
// threads (the band missed): a count of the 4096 buckets key >> 3, then of
// the 8 keys of the chosen bucket.  sh holds kBandBins counters.
template <int NT>
__device__ SelectResult cta_exact_select(const uint16_t* __restrict__ A, int64_t lda, int M, int K,
                                         uint32_t* sh, unsigned long long rank) {
    const int nch = K / 8;
    const int64_t total = (int64_t)M * nch;
    SelectResult r1;
    uint32_t bucket = 0;
    for (int level = 0; level < 2; ++level) {
        for (int i = threadIdx.x; i < kBandBins; i += NT) sh[i] = 0u;
        __syncthreads();
        for (int64_t q = threadIdx.x; q < total; q += NT) {
            const int64_t row = q / nch;
            const int c = (int)(q - row * nch);
            const uint4 v = __ldcg(reinterpret_cast<const uint4*>(A + row * lda) + c);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t key = (i & 1) ? ((w[i >> 1] >> 16) & 0x7FFFu) : (w[i >> 1] & 0x7FFFu);
                if (level == 0) atomicAdd(&sh[key >> 3], 1u);
                else if ((key >> 3) == bucket) atomicAdd(&sh[key & 7u], 1u);
            }
        }
        __syncthreads();
        if (level == 0) {
            r1 = block_select<kBandBins / NT, true, NT>(sh, rank);
            __syncthreads();
            if (!r1.found) return r1;
            bucket = r1.bin;
        } else {
            SelectResult r2 = block_select<kBandBins / NT, true, NT>(sh, rank - r1.below);
            r2.bin = bucket * 8 + r2.bin;
            r2.below += r1.below;
            return r2;
        }
    }
    return r1;
}

// The band pass over the rows of warp gwarp, gwarp + nwarps, ...: per-row max
// key into rowmax, count of keys >= lo into n_ge, keys in [lo, hi] into the
// shared histogram sh (at key - lo), non-finite keys into bad.
__device__ __forceinline__ void band_rows(const uint16_t* __restrict__ A, int64_t lda, int M, int K,
                                          uint32_t lo, uint32_t hi, uint32_t* sh,
                                          uint32_t* __restrict__ rowmax, int gwarp, int nwarps,
                                          unsigned long long& n_ge, uint32_t& bad) {
    const int lane = threadIdx.x & 31;
    const int nchunks = K / 8;
    const int steps_per_row = (nchunks + 127) / 128;
    int row = gwarp, step = 0;
    uint4 nxt[4];
    auto load_step = [&](int r, int st, uint4 (&dst)[4]) {
        const uint16_t* base = A + (int64_t)r * lda;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = st * 128 + 32 * j + lane;
            dst[j] = (c < nchunks) ? __ldg(reinterpret_cast<const uint4*>(base) + c)
                                   : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    if (row < M) load_step(row, 0, nxt);
    uint32_t mx = 0, cnt = 0, mx1 = 0, cnt1 = 0;
    while (row < M) {
        uint4 cur[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) cur[j] = nxt[j];
        int nrow = row, nstep = step + 1;
        if (nstep == steps_per_row) nrow = row + nwarps, nstep = 0;
        if (nrow < M) load_step(nrow, nstep, nxt);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (step * 128 + 32 * j + lane >= nchunks) continue;   // past K
            const uint32_t w[4] = {cur[j].x, cur[j].y, cur[j].z, cur[j].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t m = w[i] & 0x7FFF7FFFu;
                // two accumulator chains each (shorter dependency chains)
                if (i & 1) mx1 = max_u16x2(mx1, m);
                else mx = max_u16x2(mx, m);
                const uint32_t ge = swar_ge(m, lo);
                if (i & 1) cnt1 += ge >> 15;
                else cnt += ge >> 15;
                const uint32_t in = ge & ~swar_gt(m, hi);
                if (in) {
                    if (in & 0x8000u) atomicAdd(&sh[(m & 0xFFFFu) - lo], 1u);
                    if (in >> 16) atomicAdd(&sh[(m >> 16) - lo], 1u);
                }
            }
        }
        if (nstep == 0) {
            // row done: its max key and its count of keys >= lo
            mx = max_u16x2(mx, mx1);
            cnt += cnt1;
            const uint32_t km = warp_max_u32(max(mx & 0xFFFFu, mx >> 16));
            if (lane == 0) rowmax[row] = km;
            bad |= (km >= nonfinite_key<QG_BF16>()) ? 1u : 0u;
            n_ge += (cnt & 0xFFFFu) + (cnt >> 16);
            mx = mx1 = 0;
            cnt = cnt1 = 0;
        }
        row = nrow;
        step = nstep;
    }
}

// The band pass over (row, 1024-column step) units u = gwarp, gwarp + nwarps,
// ... (u = row * steps + step): the unit's max key into rowmax[u], count of
// keys >= lo into n_ge, keys in [lo, hi] into sh (at key - lo), non-finite
// keys into bad.  Finer than whole rows, so the warps finish together.
__device__ __forceinline__ void band_units(const uint16_t* __restrict__ A, int64_t lda, int M, int K,
                                           uint32_t lo, uint32_t hi, uint32_t* sh,
                                           uint32_t* __restrict__ rowmax, int gwarp, int nwarps,
                                           unsigned long long& n_ge, uint32_t& bad) {
    const int lane = threadIdx.x & 31;
    const int nchunks = K / 8;
    const int steps = (nchunks + 127) / 128;
    // unit u = row * steps + step, walked u = gwarp, gwarp + nwarps, ...; the
    // (row, step) pair is advanced by (dq, dr) = (nwarps / steps, nwarps %
    // steps) per unit instead of dividing u (a 64-bit division per unit)
    const int dq = nwarps / steps, dr = nwarps % steps;
    int r = gwarp / steps, st = gwarp % steps;
    auto advance = [&](int& rr, int& ss) {
        rr += dq;
        ss += dr;
        if (ss >= steps) {
            ss -= steps;
            ++rr;
        }
    };
    auto load_unit = [&](int rr, int ss, uint4 (&dst)[4]) {
        const uint16_t* base = A + (int64_t)rr * lda;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = ss * 128 + 32 * j + lane;
            dst[j] = (c < nchunks) ? __ldg(reinterpret_cast<const uint4*>(base) + c)
                                   : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    uint4 nxt[4];
    if (r < M) load_unit(r, st, nxt);
    while (r < M) {
        uint4 cur[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) cur[j] = nxt[j];
        int nr = r, ns = st;
        advance(nr, ns);
        if (nr < M) load_unit(nr, ns, nxt);
        uint32_t mx = 0, mx1 = 0, cnt = 0, cnt1 = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (st * 128 + 32 * j + lane >= nchunks) continue;   // past K
            const uint32_t w[4] = {cur[j].x, cur[j].y, cur[j].z, cur[j].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t m = w[i] & 0x7FFF7FFFu;
                if (i & 1) mx1 = max_u16x2(mx1, m);
                else mx = max_u16x2(mx, m);
                const uint32_t ge = swar_ge(m, lo);
                if (i & 1) cnt1 += ge >> 15;
                else cnt += ge >> 15;
                const uint32_t in = ge & ~swar_gt(m, hi);
                if (in) {
                    if (in & 0x8000u) atomicAdd(&sh[(m & 0xFFFFu) - lo], 1u);
                    if (in >> 16) atomicAdd(&sh[(m >> 16) - lo], 1u);
                }
            }
        }
        mx = max_u16x2(mx, mx1);
        cnt += cnt1;
        const uint32_t km = warp_max_u32(max(mx & 0xFFFFu, mx >> 16));
        if (lane == 0) rowmax[(int64_t)r * steps + st] = km;
        bad |= (km >= nonfinite_key<QG_BF16>()) ? 1u : 0u;
        n_ge += (cnt & 0xFFFFu) + (cnt >> 16);
        r = nr;
        st = ns;
    }
}

// A CTA's share of the band pass into the global counters and bins.
template <int NT>
__device__ void band_flush(const uint32_t* sh, uint32_t* __restrict__ band_bins,
                           unsigned long long n_ge, uint32_t bad, Counters* __restrict__ ctr) {
    __shared__ unsigned long long s_ge[NT / 32];
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) n_ge += __shfl_xor_sync(0xFFFFFFFFu, n_ge, d);
    if (lane == 0) s_ge[threadIdx.x >> 5] = n_ge;
    if (bad && lane == 0) atomicOr(&ctr->nonfinite, 1u);
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long tot = 0;
        for (int i = 0; i < NT / 32; ++i) tot += s_ge[i];
        if (tot) atomicAdd(&ctr->band_below, tot);
    }
    for (int i = threadIdx.x; i < kBandBins; i += NT) {
        const uint32_t v = sh[i];
        if (v) atomicAdd(&band_bins[i], v);
    }
}

// Selection over NB global bins (written by other SMs: read around L1) by NT
// threads in one pass: thread t sums its NB / NT consecutive bins, one block
// scan locates the thread that holds the rank, which walks its own bins.
template <int NT, int NB>
__device__ SelectResult block_select_seq(const uint32_t* __restrict__ hist, unsigned long long rank) {
    constexpr int B = NB / NT;
    static_assert(B % 4 == 0, "whole 16-byte groups per thread");
    __shared__ unsigned long long s_w[NT / 32];
    __shared__ SelectResult s_res;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    uint32_t v[B];
#pragma unroll
    for (int i = 0; i < B / 4; ++i) {
        const uint4 q = __ldcg(reinterpret_cast<const uint4*>(hist) + t * (B / 4) + i);
        v[4 * i] = q.x;
        v[4 * i + 1] = q.y;
        v[4 * i + 2] = q.z;
        v[4 * i + 3] = q.w;
    }
    unsigned long long mine = 0;
#pragma unroll
    for (int i = 0; i < B; ++i) mine += v[i];
    unsigned long long incl = mine;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const unsigned long long u = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += u;
    }
    if (lane == 31) s_w[w] = incl;
    if (t == 0) s_res.found = 0;
    __syncthreads();
    unsigned long long c = incl - mine;
    for (int i = 0; i < w; ++i) c += s_w[i];
    if (c <= rank && rank < c + mine) {
#pragma unroll
        for (int i = 0; i < B; ++i) {
            if (c <= rank && rank < c + v[i]) {
                s_res.bin = (uint32_t)(B * t + i);
                s_res.below = c;
                s_res.found = 1;
            }
            c += v[i];
        }
    }
    __syncthreads();
    return s_res;
}

// After every CTA's flush: the threshold from the band, or from the exact
// fallback when the band does not hold the order statistic (one CTA).
template <int NT>
__device__ void band_select(const uint16_t* __restrict__ A, int64_t lda, int M, int K,
                            const uint32_t* band_bins, Counters* __restrict__ ctr,
                            unsigned long long rank, uint32_t* __restrict__ status,
                            float* __restrict__ T_out, uint32_t* sh) {
    const uint32_t lo = __ldcg(&ctr->band_lo);
    // band_below holds the count of keys >= lo
    const unsigned long long n = (unsigned long long)M * (unsigned long long)K;
    const unsigned long long nbelow = n - __ldcg(&ctr->band_below);
    SelectResult r;
    r.found = 0;
    if (rank >= nbelow) {
        r = block_select_seq<NT, kBandBins>(band_bins, rank - nbelow);
        r.bin += lo;
        r.below += nbelow;
    }
    __syncthreads();
    if (!r.found) {
        if (threadIdx.x == 0) ctr->band_missed = 1u;
        r = cta_exact_select<NT>(A, lda, M, K, sh, rank);
    }
    finish_select<0>(r, ctr, status, T_out);
}

// Full pass over A (grid-stride rows); the last CTA selects the threshold.
__global__ void __launch_bounds__(kBandThreads, 1)
band_hist_rowmax_kernel(const uint16_t* __restrict__ A, int64_t lda, int M, int K,
                        uint32_t* __restrict__ band_bins, uint32_t* __restrict__ rowmax,
                        Counters* __restrict__ ctr, unsigned long long rank,
                        uint32_t* __restrict__ status, float* __restrict__ T_out) {
    __shared__ uint32_t sh[kBandBins];
    for (int i = threadIdx.x; i < kBandBins; i += blockDim.x) sh[i] = 0u;
    __syncthreads();
    const uint32_t lo = __ldcg(&ctr->band_lo), hi = __ldcg(&ctr->band_hi);
    const int wpc = kBandThreads / 32;
    unsigned long long n_ge = 0;
    uint32_t bad = 0;
    band_rows(A, lda, M, K, lo, hi, sh, rowmax, blockIdx.x * wpc + (threadIdx.x >> 5),
              gridDim.x * wpc, n_ge, bad);
    band_flush<kBandThreads>(sh, band_bins, n_ge, bad, ctr);
    if (last_block_done(&ctr->done_band))
        band_select<kBandThreads>(A, lda, M, K, band_bins, ctr, rank, status, T_out, sh);
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

// --------------------------------------------------------------------------
// The same pass for bf16 A with codes out, written for instruction count: the
// bf16 pairs stay packed until they are scaled.  Per 32-bit word (two bf16):
// the outlier test is a SWAR compare of the two magnitudes with T (one add,
// one and), the scale one packed fp32x2 multiply (IEEE round to nearest, as
// __fmul_rn), the encode one cvt; the clamp itself costs nothing, because the
// saturating conversion already maps an outlier to the code of +-T (see the
// encode below).  The next step's loads are issued before this step's work.
// Warps walk rows grid-stride; a step covers 1024 columns of one row.
constexpr int kQ3Threads = 256;
constexpr int kStepListCap = 512;   // outliers per 1024-column step held in a warp's list
#ifndef QG_CLAMP_MIN_BLOCKS
#define QG_CLAMP_MIN_BLOCKS 3
#endif
constexpr int kQ3MinBlocks = QG_CLAMP_MIN_BLOCKS;   // resident CTAs per SM (register cap)


// The clamp / quantize pass over rows first, first + stride, ... (< row_end)
// of this warp; M is the matrix height (the overflow slots follow M row
// regions).  olist: this warp's kStepListCap-entry list in shared memory, in
// which a step's outliers are placed at their ranks before the warp writes
// their entries together.
__device__ __forceinline__ void clamp_rows_bf16(const uint16_t* __restrict__ A, int64_t lda, int M,
                                                int K, uint32_t T_key,
                                                const uint32_t* __restrict__ rowmax,
                                                Counters* __restrict__ ctr,
                                                uint8_t* __restrict__ codes,
                                                float* __restrict__ scales, const ActBuffers& b,
                                                int first, int stride, int row_end,
                                                int nparts, uint16_t* olist) {
    // (an unselected threshold reads as the largest finite-or-not key)
    const uint32_t Tk = min(T_key, 0x7FFFu);
    const uint32_t cT = (0x7FFFu - Tk) * 0x10001u;   // SWAR: key > T sets bit 15
    const float T = __uint_as_float(Tk << 16);
    const int lane = threadIdx.x & 31;
    const int nchunks = K / 8;                       // 16-byte chunks per row
    const int steps_per_row = (nchunks + 127) / 128;
    const int row_slots = (int)b.row_slots;

    int row = first, step = 0;
    uint4 nxt[4];
    auto load_step = [&](int r, int st, uint4 (&dst)[4]) {
        const uint16_t* base = A + (int64_t)r * lda;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = st * 128 + 32 * j + lane;
            dst[j] = (c < nchunks) ? __ldg(reinterpret_cast<const uint4*>(base) + c)
                                   : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    if (row < row_end) load_step(row, 0, nxt);

    float r = 0.0f;
    int row_rank = 0;
    while (row < row_end) {
        if (step == 0) {
            uint32_t rmax = 0;   // the row's max key: over its nparts partial maxima
            for (int q = 0; q < nparts; ++q) rmax = max(rmax, __ldcg(rowmax + (int64_t)row * nparts + q));
            float s;
            scale_factors(__uint_as_float(min(rmax, Tk) << 16), r, s);
            if (lane == 0) scales[row] = s;
            row_rank = 0;
        }
        uint32_t w[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            w[j][0] = nxt[j].x;
            w[j][1] = nxt[j].y;
            w[j][2] = nxt[j].z;
            w[j][3] = nxt[j].w;
        }
        int nrow = row, nstep = step + 1;
        if (nstep == steps_per_row) nrow = row + stride, nstep = 0;
        if (nrow < row_end) load_step(nrow, nstep, nxt);

        // outlier test: the 16x2 max of |w| over the step, then bit 15 / 31
        // of (max + cT); zero-filled columns past K never exceed T
        uint32_t mx0 = 0, mx1 = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (i & 1) mx1 = max_u16x2(mx1, w[j][i] & 0x7FFF7FFFu);
                else mx0 = max_u16x2(mx0, w[j][i] & 0x7FFF7FFFu);
            }
        }
        const uint32_t any = (max_u16x2(mx0, mx1) + cT) & 0x80008000u;
        if (__any_sync(0xFFFFFFFFu, any != 0)) {
            // this lane's outliers: element e of chunk j at bit 8 j + e.  The
            // flags sit in bit 7 of bytes 1 and 3 of (|w| + cT); a byte
            // permute gathers four of them into one word, and a multiply
            // packs the four bit-7s into a nibble
            uint32_t ob = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t g[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) g[i] = (w[j][i] & 0x7FFF7FFFu) + cT;
                const uint32_t p01 = (__byte_perm(g[0], g[1], 0x7531) >> 7) & 0x01010101u;
                const uint32_t p23 = (__byte_perm(g[2], g[3], 0x7531) >> 7) & 0x01010101u;
                const uint32_t nib01 = (p01 * 0x01020408u) >> 24;
                const uint32_t nib23 = (p23 * 0x01020408u) >> 24;
                ob |= (nib01 | (nib23 << 4)) << (8 * j);
            }
            // ranks in column order: chunks j-major, then lanes, then
            // elements; the four per-lane counts are scanned as two pairs of
            // 16-bit fields
            const uint32_t c01 = __popc(ob & 0xFFu) | (__popc(ob & 0xFF00u) << 16);
            const uint32_t c23 = __popc(ob & 0xFF0000u) | (__popc(ob & 0xFF000000u) << 16);
            const uint32_t i01 = (uint32_t)warp_inclusive_scan((int)c01);
            const uint32_t i23 = (uint32_t)warp_inclusive_scan((int)c23);
            const uint32_t t01 = __shfl_sync(0xFFFFFFFFu, i01, 31);
            const uint32_t t23 = __shfl_sync(0xFFFFFFFFu, i23, 31);
            const uint32_t e01 = i01 - c01, e23 = i23 - c23;
            // first rank within the step of this lane's outliers in chunk j
            const int b0 = (int)(e01 & 0xFFFF);
            const int b1 = (int)(t01 & 0xFFFF) + (int)(e01 >> 16);
            const int b2 = (int)(t01 & 0xFFFF) + (int)(t01 >> 16) + (int)(e23 & 0xFFFF);
            const int b3 = (int)(t01 & 0xFFFF) + (int)(t01 >> 16) + (int)(t23 & 0xFFFF) + (int)(e23 >> 16);
            const int n_step = b3 - (int)(e23 >> 16) + (int)(t23 >> 16);
            const uint16_t* arow = A + (int64_t)row * lda;
            // entry of rank row_rank + q (step column c): dA value and staging
            auto emit = [&](int q, int c) {
                const int col = step * 1024 + c;
                const int idx = row_rank + q;
                const float a = __uint_as_float((uint32_t)__ldg(arow + col) << 16);
                const double d = (double)a - (double)copysignf(T, a);
                if (idx < row_slots) {
                    b.st_col[(int64_t)row * row_slots + idx] = col;
                    b.st_val[(int64_t)row * row_slots + idx] = d;
                } else {
                    const unsigned long long o = atomicAdd(&ctr->nnz, 1ull);
                    if (o < (unsigned long long)b.cap) {
                        const int64_t slot = (int64_t)M * row_slots + (int64_t)o;
                        b.st_row[o] = row;
                        b.st_rank[o] = idx;
                        b.st_col[slot] = col;
                        b.st_val[slot] = d;
                    } else {
                        flag_status(b.status, kStatusOverflow);
                    }
                }
            };
            if (n_step <= kStepListCap) {
                // each lane drops its outliers' step columns into the warp's
                // list at their ranks (dense: 0 .. n_step - 1), then the
                // warp emits the step's entries together, a lane each
                for (uint32_t mm = ob; mm != 0; mm &= mm - 1) {
                    const int bit = __ffs(mm) - 1;
                    const int j = bit >> 3;
                    const int q = (j == 0 ? b0 : j == 1 ? b1 : j == 2 ? b2 : b3) +
                                  __popc(ob & ((1u << bit) - 1u) & (0xFFu << (8 * j)));
                    olist[q] = (uint16_t)((32 * j + lane) * 8 + (bit & 7));
                }
                __syncwarp();
                for (int q = lane; q < n_step; q += 32) emit(q, olist[q]);
                __syncwarp();   // the list is rewritten by the next step
            } else {
                for (uint32_t mm = ob; mm != 0; mm &= mm - 1) {
                    const int bit = __ffs(mm) - 1;
                    const int j = bit >> 3;
                    const int q = (j == 0 ? b0 : j == 1 ? b1 : j == 2 ? b2 : b3) +
                                  __popc(ob & ((1u << bit) - 1u) & (0xFFu << (8 * j)));
                    emit(q, (32 * j + lane) * 8 + (bit & 7));
                }
            }
            row_rank += n_step;
        }
        // codes of the clamped row: an outlier x (|x| > T, so amax = T) has
        // |x r| >= |T r|, and T r is 6 within an ulp, so the saturating
        // conversion of x r gives +-6 -- the code of sign(x) T r; hence the
        // row is encoded without writing the clamp back into registers
        uint32_t* out = reinterpret_cast<uint32_t*>(codes + (int64_t)row * (K / 2));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = step * 128 + 32 * j + lane;
            if (c < nchunks) {
                const uint32_t q01 = __byte_perm(bf16x2_encode(w[j][0], r), bf16x2_encode(w[j][1], r), 0x0040);
                const uint32_t q23 = __byte_perm(bf16x2_encode(w[j][2], r), bf16x2_encode(w[j][3], r), 0x0040);
                out[c] = __byte_perm(q01, q23, 0x5410);
            }
        }
        if (nstep == 0 && lane == 0) b.rowcnt[row] = (uint32_t)row_rank;
        row = nrow;
        step = nstep;
    }
}

// row_ptr = exclusive scan of the row counts, by one CTA of NT threads.
template <int NT>
__device__ void cta_scan_rowcnt(const ActBuffers& b, int M, int32_t* __restrict__ row_ptr,
                                int64_t* __restrict__ nnz_out) {
    __shared__ unsigned long long s_warp[NT / 32];
    const int t = threadIdx.x, wi = t >> 5, lane = t & 31;
    const int per = (M + NT - 1) / NT;
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
    if (lane == 31) s_warp[wi] = v;
    __syncthreads();
    unsigned long long before = 0, total = 0;
    for (int i = 0; i < NT / 32; ++i) {
        if (i < wi) before += s_warp[i];
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

__global__ void __launch_bounds__(kQ3Threads, kQ3MinBlocks)
clamp_quant_bf16_kernel(const uint16_t* __restrict__ A, int64_t lda, int M, int K,
                        const uint32_t* __restrict__ rowmax, Counters* __restrict__ ctr,
                        uint8_t* __restrict__ codes, float* __restrict__ scales, ActBuffers b,
                        int32_t* __restrict__ row_ptr, int64_t* __restrict__ nnz_out) {
    const int wpc = kQ3Threads / 32;
    __shared__ uint16_t s_list[kQ3Threads / 32][kStepListCap];
    clamp_rows_bf16(A, lda, M, K, __ldcg(&ctr->T_key), rowmax, ctr, codes, scales, b,
                    blockIdx.x * wpc + (threadIdx.x >> 5), gridDim.x * wpc, M, 1,
                    s_list[threadIdx.x >> 5]);
    if (last_block_done(&ctr->done_clamp)) cta_scan_rowcnt<kQ3Threads>(b, M, row_ptr, nnz_out);
}

// Move staged entries to their CSR positions: warp gwarp, gwarp + nwarps, ...
// per row for the row regions, then thread gtid, gtid + nthreads, ... per
// overflow entry.  Staged data is read around L1 (other SMs wrote it).
__device__ __forceinline__ void scatter_entries(const Counters* __restrict__ ctr,
                                                const ActBuffers& b, int M,
                                                const int32_t* __restrict__ row_ptr,
                                                int32_t* __restrict__ col,
                                                double* __restrict__ val, int gwarp, int nwarps,
                                                int64_t gtid, int64_t nthreads) {
    const int lane = threadIdx.x & 31;
    const int row_slots = (int)b.row_slots;
    for (int r = gwarp; r < M; r += nwarps) {
        const int n = min((int)__ldcg(b.rowcnt + r), row_slots);
        const int64_t dst = __ldcg(row_ptr + r);
        const int64_t src = (int64_t)r * row_slots;
        for (int j = lane; j < n; j += 32) {
            col[dst + j] = __ldcg(b.st_col + src + j);
            val[dst + j] = __ldcg(b.st_val + src + j);
        }
    }
    const unsigned long long n_over = min(__ldcg(&ctr->nnz), (unsigned long long)b.cap);
    const int64_t base = (int64_t)M * row_slots;
    for (unsigned long long e = (unsigned long long)gtid; e < n_over; e += (unsigned long long)nthreads) {
        const int64_t dst = (int64_t)__ldcg(row_ptr + __ldcg(b.st_row + e)) + __ldcg(b.st_rank + e);
        col[dst] = __ldcg(b.st_col + base + e);
        val[dst] = __ldcg(b.st_val + base + e);
    }
}

__global__ void __launch_bounds__(256)
csr_scatter_kernel(const Counters* __restrict__ ctr, ActBuffers b, int M,
                   const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col,
                   double* __restrict__ val) {
    scatter_entries(ctr, b, M, row_ptr, col, val, (blockIdx.x * blockDim.x + threadIdx.x) >> 5,
                    (gridDim.x * blockDim.x) >> 5, blockIdx.x * (int64_t)blockDim.x + threadIdx.x,
                    (int64_t)gridDim.x * blockDim.x);
}

// Exclusive scan of n counts (in[0..n), written by any CTA: read around L1)
// into out[0..n) by one CTA of NT threads; the total goes to *total.
template <int NT>
__device__ void cta_local_scan(const uint32_t* in, int n, uint32_t* out, uint32_t* total) {
    __shared__ uint32_t s_w[NT / 32];
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int per = (n + NT - 1) / NT;
    const int a = min(n, t * per), e = min(n, a + per);
    uint32_t mine = 0;
    for (int i = a; i < e; ++i) mine += __ldcg(in + i);
    const uint32_t incl = (uint32_t)warp_inclusive_scan((int)mine);
    if (lane == 31) s_w[w] = incl;
    __syncthreads();
    uint32_t run = incl - mine, all = 0;
    for (int i = 0; i < NT / 32; ++i) {
        if (i < w) run += s_w[i];
        all += s_w[i];
    }
    for (int i = a; i < e; ++i) {
        const uint32_t c = __ldcg(in + i);
        out[i] = run;
        run += c;
    }
    if (t == 0) *total = all;
}

// The last CTA: exclusive scan of the per-CTA totals in place (offsets), the
// grand total into row_ptr[M] and nnz_out, and the capacity check.
template <int NT>
__device__ void cta_scan_offsets(uint32_t* cta_tot, int ncta, const ActBuffers& b, int M,
                                 int32_t* __restrict__ row_ptr, int64_t* __restrict__ nnz_out) {
    __shared__ unsigned long long s_w[NT / 32];
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int per = (ncta + NT - 1) / NT;
    const int a = min(ncta, t * per), e = min(ncta, a + per);
    unsigned long long mine = 0;
    for (int i = a; i < e; ++i) mine += __ldcg(cta_tot + i);
    unsigned long long incl = mine;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const unsigned long long u = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += u;
    }
    if (lane == 31) s_w[w] = incl;
    __syncthreads();
    unsigned long long run = incl - mine, all = 0;
    for (int i = 0; i < NT / 32; ++i) {
        if (i < w) run += s_w[i];
        all += s_w[i];
    }
    for (int i = a; i < e; ++i) {
        const uint32_t c = __ldcg(cta_tot + i);
        cta_tot[i] = (uint32_t)run;
        run += c;
    }
    if (t == 0) {
        row_ptr[M] = (int32_t)all;
        *nnz_out = (int64_t)all;
        if (all > (unsigned long long)b.cap) flag_status(b.status, kStatusOverflow);
    }
}

// --------------------------------------------------------------------------
// Phase 5 of the fused kernel: the staged entries of rows [r0, r1) to their
// CSR positions rowpre[r] + off.  A warp takes kScatterRows rows at a time and
// issues the loads of all of them before any store (staged data was written
// by other SMs: read around L1).
constexpr int kScatterRows = 4;
template <int NT>
__device__ __forceinline__ void scatter_rows(const ActBuffers& b, int r0, int r1, uint32_t off,
                                             int32_t* __restrict__ col, double* __restrict__ val) {
    constexpr int RB = kScatterRows;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int row_slots = (int)b.row_slots;
    for (int rb = r0 + warp * RB; rb < r1; rb += (NT / 32) * RB) {
        int cnt = 0;
        long long dst = 0;
        if (lane < RB && rb + lane < r1) {
            cnt = min((int)__ldcg(b.rowcnt + rb + lane), row_slots);
            dst = (long long)__ldcg(b.rowpre + rb + lane) + off;
        }
        int c4[RB];
        long long d4[RB];
        int maxn = 0;
#pragma unroll
        for (int q = 0; q < RB; ++q) {
            c4[q] = __shfl_sync(0xFFFFFFFFu, cnt, q);
            d4[q] = __shfl_sync(0xFFFFFFFFu, dst, q);
            maxn = max(maxn, c4[q]);
        }
        for (int j = lane; j < maxn; j += 32) {
            int cv[RB];
            double vv[RB];
#pragma unroll
            for (int q = 0; q < RB; ++q) {
                cv[q] = 0;
                vv[q] = 0.0;
                if (j < c4[q]) {
                    const int64_t src = (int64_t)(rb + q) * row_slots + j;
                    cv[q] = __ldcg(b.st_col + src);
                    vv[q] = __ldcg(b.st_val + src);
                }
            }
#pragma unroll
            for (int q = 0; q < RB; ++q) {
                if (j < c4[q]) {
                    col[d4[q] + j] = cv[q];
                    val[d4[q] + j] = vv[q];
                }
            }
        }
    }
}

// The whole bf16 quantize_act in one cooperative launch (all CTAs resident):
//   phase 0  every CTA puts the band around the quantile of the same sample
//            of A (so no barrier follows); CTA 0 also zeroes the counters
//   phase 1  band pass: row maxima, band histogram, count below the band
//   phase 2  the last CTA to finish phase 1 selects T, then releases the rest
//   phase 3  clamp / quantize / dA staging
//   phase 4  the last CTA to finish phase 3 scans the row counts into row_ptr
//   phase 5  CSR scatter (a warp moves four rows' entries at a time)
// The grid barriers are a count and a generation word in the workspace
// (count returns to 0 after every barrier).  Every wait is bounded: a CTA
// that gives up sets the timeout bit and returns (the workspace barrier words
// are then reset by qg_sync_status / qg_workspace_init).
// 16 warps per CTA, two CTAs per SM (64 registers): fewer, larger CTAs make
// the grid barriers, the band flush and the CTA-offset scan cheaper than
// 256-thread CTAs at the same warp count per SM.
constexpr int kFusedThreads = 512;
constexpr int kFusedMinBlocks = 2;
constexpr int kCtaTotOffset = 8192;   // per-CTA totals in hist1 (after the band bins)
constexpr int kFusedMaxGrid = 8192;

__global__ void __launch_bounds__(kFusedThreads, kFusedMinBlocks)
act_fused_bf16_kernel(const uint16_t* __restrict__ A, int64_t lda, int M, int K,
                      unsigned long long rank, ActBuffers b, uint8_t* __restrict__ codes,
                      float* __restrict__ scales, int32_t* __restrict__ row_ptr,
                      int32_t* __restrict__ col, double* __restrict__ val,
                      int64_t* __restrict__ nnz_out, float* __restrict__ T_out) {
    __shared__ __align__(16) uint32_t sh[kBandBins];   // sample bins, band bins, fallback counts
    constexpr int wpc = kFusedThreads / 32;
    const int gwarp = blockIdx.x * wpc + (threadIdx.x >> 5), nwarps = gridDim.x * wpc;
    GridSync* g = b.gsync;
    uint32_t gen0;
    uint32_t lo, hi;

    // phase 0: every CTA puts the band around the quantile of the same sample
    // of A, so no barrier follows.  CTA 0 also zeroes the counters and band
    // bins and then publishes zflag = gen + 1 (the generation word cannot
    // move before every CTA has arrived at the first barrier, so all CTAs
    // read the same gen here); each CTA checks it before adding into them.
    __shared__ uint32_t s_gen;
    if (threadIdx.x == 0) s_gen = ld_relaxed_u32(&g->gen);
    if (blockIdx.x == 0) {
        uint32_t* cz = reinterpret_cast<uint32_t*>(b.ctr);
        for (int i = threadIdx.x; i < (int)(sizeof(Counters) / 4); i += kFusedThreads) cz[i] = 0u;
        for (int i = threadIdx.x; i < kBandBins; i += kFusedThreads) b.hist1[i] = 0u;
    }
    cta_band_local<kFusedThreads>(A, lda, M, K, rank, sh, lo, hi);
    const uint32_t zwant = s_gen + 1u;
    if (blockIdx.x == 0) {
        if (threadIdx.x == 0) {
            b.ctr->band_lo = lo;
            b.ctr->band_hi = hi;
        }
        __threadfence();
        flag_publish(&g->zflag, zwant);
    }

    // phase 1
    for (int i = threadIdx.x; i < kBandBins; i += kFusedThreads) sh[i] = 0u;
    __syncthreads();
    {
        unsigned long long n_ge = 0;
        uint32_t bad = 0;
        band_units(A, lda, M, K, lo, hi, sh, b.rowmax, gwarp, nwarps, n_ge, bad);
        // the counters and bins that CTA 0 zeroed (published before its band pass)
        if (!flag_wait(&g->zflag, zwant, b.status)) return;
        band_flush<kFusedThreads>(sh, b.hist1, n_ge, bad, b.ctr);
    }
    // phase 2
    if (grid_arrive(g, gen0)) {
        band_select<kFusedThreads>(A, lda, M, K, b.hist1, b.ctr, rank, b.status, T_out, sh);
        grid_release(g);
    } else if (!grid_wait(g, gen0, b.status)) {
        return;
    }

    // phase 3: CTA c clamps rows [r0, r1), a warp per row, then scans its
    // rows' counts locally into rowpre
    const int rpc = (M + (int)gridDim.x - 1) / (int)gridDim.x;
    const int r0 = min(M, (int)blockIdx.x * rpc), r1 = min(M, r0 + rpc);
    // (the band histogram's shared memory holds the warps' outlier lists now)
    static_assert(kBandBins * 2 >= (kFusedThreads / 32) * kStepListCap, "lists fit in sh");
    clamp_rows_bf16(A, lda, M, K, __ldcg(&b.ctr->T_key), b.rowmax, b.ctr, codes, scales, b,
                    r0 + (int)(threadIdx.x >> 5), wpc, r1, (K / 8 + 127) / 128,
                    reinterpret_cast<uint16_t*>(sh) + (threadIdx.x >> 5) * kStepListCap);
    uint32_t* cta_off = b.hist1 + kCtaTotOffset;   // per-CTA totals, then offsets
    __syncthreads();
    cta_local_scan<kFusedThreads>(b.rowcnt + r0, r1 - r0, b.rowpre + r0, cta_off + blockIdx.x);
    // phase 4: the last CTA turns the CTA totals into offsets
    if (grid_arrive(g, gen0)) {
        cta_scan_offsets<kFusedThreads>(cta_off, (int)gridDim.x, b, M, row_ptr, nnz_out);
        grid_release(g);
    } else if (!grid_wait(g, gen0, b.status)) {
        return;
    }

    // phase 5: row_ptr and the row regions of this CTA's rows, then a slice of
    // the overflow list
    const uint32_t off = __ldcg(cta_off + blockIdx.x);
    for (int r = r0 + (int)threadIdx.x; r < r1; r += kFusedThreads)
        row_ptr[r] = (int32_t)(__ldcg(b.rowpre + r) + off);
    scatter_rows<kFusedThreads>(b, r0, r1, off, col, val);
    {
        const int row_slots = (int)b.row_slots;
        const unsigned long long n_over = min(__ldcg(&b.ctr->nnz), (unsigned long long)b.cap);
        const int64_t base = (int64_t)M * row_slots;
        for (unsigned long long e = blockIdx.x * (unsigned long long)kFusedThreads + threadIdx.x;
             e < n_over; e += (unsigned long long)gridDim.x * kFusedThreads) {
            const int rr = __ldcg(b.st_row + e);
            const int64_t dst = (int64_t)__ldcg(b.rowpre + rr) + __ldcg(cta_off + rr / rpc) +
                                __ldcg(b.st_rank + e);
            col[dst] = __ldcg(b.st_col + base + e);
            val[dst] = __ldcg(b.st_val + base + e);
        }
    }
}

// --------------------------------------------------------------------------
// Host-side sequences.
static cudaError_t threshold_passes(const void* A, qg_dtype dt, int64_t M, int64_t K,
                                    int64_t lda, int64_t rank, const ActBuffers& b, float* T_out,
                                    cudaStream_t s) {
    const int nsm = num_sms();
    const int grid1 = (int)std::min<int64_t>(nsm, (M + 31) / 32);
    const size_t shmem = sizeof(uint32_t) * kHist1Bins;
    if (dt == QG_BF16) {
        // the band bins live at the start of hist1; the prep kernel zeroes
        // them and the counters
        const uint16_t* Ab = static_cast<const uint16_t*>(A);
        band_prep_kernel<<<1, kBandThreads, 0, s>>>(Ab, lda, (int)M, (int)K, b.ctr, b.hist1,
                                                        (unsigned long long)rank);
        band_hist_rowmax_kernel<<<grid1, kBandThreads, 0, s>>>(Ab, lda, (int)M, (int)K, b.hist1,
                                                               b.rowmax, b.ctr,
                                                               (unsigned long long)rank, b.status,
                                                               T_out);
        count_launch(2);
    } else {
        // counters and histograms are contiguous in the workspace
        uint32_t* zbeg = reinterpret_cast<uint32_t*>(b.ctr);
        launch_zero_u32(zbeg, (b.hist2 + kHist2Bins) - zbeg, s);
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
    if (DT == QG_BF16 && CODES) {
        const int g = (int)std::max<int64_t>(1, std::min<int64_t>((M + wpc - 1) / wpc, (int64_t)num_sms() * kQ3MinBlocks));
        clamp_quant_bf16_kernel<<<g, kQ3Threads, 0, s>>>(static_cast<const uint16_t*>(A), lda, (int)M,
                                                         (int)K, b.rowmax, b.ctr, codes, scales, b,
                                                         dA->row_ptr, dA->nnz_out);
    } else {
        const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((M + wpc - 1) / wpc, (int64_t)num_sms() * 8));
        clamp_quant_kernel<DT, CODES><<<grid, kQuantThreads, 0, s>>>(
            A, lda, (int)M, (int)K, b.rowmax, b.ctr, codes, scales, A_c, b, dA->row_ptr, dA->nnz_out);
    }
    const int g2 = (int)std::max<int64_t>(1, std::min<int64_t>((M * 32 + 255) / 256, (int64_t)num_sms() * 8));
    csr_scatter_kernel<<<g2, 256, 0, s>>>(b.ctr, b, (int)M, dA->row_ptr, dA->col, dA->val);
    count_launch(2);
}

// Resident CTAs per SM of the cooperative kernel, per device (0: not usable).
static int g_fused_blocks[64];

cudaError_t act_setup() {
    int dev = 0, coop = 0, nb = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
    if (e != cudaSuccess) return e;
    if (cooperative_disabled()) coop = 0;
    if (coop) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, act_fused_bf16_kernel, kFusedThreads, 0);
        if (e != cudaSuccess) return e;
    }
    if (dev >= 0 && dev < 64) g_fused_blocks[dev] = coop ? nb : 0;
    e = cudaFuncSetAttribute(hist_rowmax_kernel<QG_BF16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(sizeof(uint32_t) * kHist1Bins));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(hist_rowmax_kernel<QG_F32>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(sizeof(uint32_t) * kHist1Bins));
}

// The bf16 path as one cooperative launch; false when it cannot be used here.
static bool launch_act_fused(const void* A, int64_t M, int64_t K, int64_t lda, int64_t rank,
                             const ActBuffers& b, uint8_t* codes, float* scales, const qg_csr* dA,
                             float* T_out, cudaStream_t s) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    const int nb = g_fused_blocks[dev];
    if (nb < 1) return false;
    const int64_t want = (M + kFusedThreads / 32 - 1) / (kFusedThreads / 32);   // a warp per row
    const int grid = (int)std::max<int64_t>(
        1, std::min<int64_t>({want, (int64_t)nb * num_sms(), (int64_t)kFusedMaxGrid}));
    const uint16_t* Ab = static_cast<const uint16_t*>(A);
    int Mi = (int)M, Ki = (int)K;
    unsigned long long rk = (unsigned long long)rank;
    ActBuffers bb = b;
    int32_t* row_ptr = dA->row_ptr;
    int32_t* col = dA->col;
    double* val = dA->val;
    int64_t* nnz_out = dA->nnz_out;
    void* args[] = {(void*)&Ab, (void*)&lda, (void*)&Mi, (void*)&Ki, (void*)&rk, (void*)&bb,
                    (void*)&codes, (void*)&scales, (void*)&row_ptr, (void*)&col, (void*)&val,
                    (void*)&nnz_out, (void*)&T_out};
    const cudaError_t e = cudaLaunchCooperativeKernel((const void*)act_fused_bf16_kernel,
                                                      dim3((unsigned)grid), dim3(kFusedThreads),
                                                      args, 0, s);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();   // not sticky: fall back to the multi-kernel sequence
        return false;
    }
    count_launch(1);
    return true;
}

cudaError_t run_quantize_act(const void* A, qg_dtype dt, int64_t M, int64_t K, int64_t lda,
                             int64_t rank, const ActBuffers& b, uint8_t* codes, float* scales,
                             const qg_csr* dA, float* T_out, cudaStream_t s) {
    if (dt == QG_BF16 && launch_act_fused(A, M, K, lda, rank, b, codes, scales, dA, T_out, s))
        return cudaSuccess;
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
