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

template <qg_dtype DT>
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
        float* crow = C + (int64_t)r * N + n0;
        if (vec) {
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
// Fast path (bf16 W, N and ldw multiples of 8): the W row segments a warp needs
// are fetched ahead with bulk async copies into a per-warp ring of 32 slots
// (512 bytes each, one mbarrier per slot), so each warp keeps up to 16 KB of
// W in flight without spending registers on it.  A warp owns 4 consecutive
// rows: their CSR entries form one contiguous range, consumed in order; slot
// j % 32 holds entry j and is refilled with entry j + 32 once every lane has
// read it.  All waits are bounded; on a timeout the warp flags the status
// word, waits (bounded) for its copies still in flight and stops.
constexpr int kAsyncWarps = 4;
constexpr int kAsyncRowsPerWarp = 4;
constexpr int kAsyncDepth = 32;
constexpr int kAsyncSeg = kSpmmSlice * 2;   // bytes of one bf16 row segment
constexpr long long kSpmmWaitLimit = 2000000000LL;
constexpr size_t kAsyncSmem =
    (size_t)kAsyncWarps * kAsyncDepth * kAsyncSeg + (size_t)kAsyncWarps * kAsyncDepth * 8;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ bool slot_ready(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool slot_wait(uint64_t* bar, uint32_t parity) {
    if (slot_ready(bar, parity)) return true;
    const long long t0 = clock64();
    while (!slot_ready(bar, parity))
        if (clock64() - t0 > kSpmmWaitLimit) return false;
    return true;
}
__device__ __forceinline__ void slot_fetch(uint64_t* bar, void* dst, const void* src,
                                           uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__global__ void __launch_bounds__(kAsyncWarps * 32)
spmm_async_kernel(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col,
                  const double* __restrict__ val, const uint16_t* __restrict__ W, int64_t ldw,
                  int M, int N, float* __restrict__ C, uint32_t* __restrict__ status) {
    extern __shared__ __align__(128) uint8_t sm[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    uint8_t* ring = sm + (size_t)warp * kAsyncDepth * kAsyncSeg;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + (size_t)kAsyncWarps * kAsyncDepth * kAsyncSeg) +
                     warp * kAsyncDepth;
    const int r_begin = (blockIdx.x * kAsyncWarps + warp) * kAsyncRowsPerWarp;
    if (r_begin >= M) return;
    const int r_end = min(M, r_begin + kAsyncRowsPerWarp);
    if (lane == 0) {
        for (int i = 0; i < kAsyncDepth; ++i)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&bars[i])));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    const int n0 = blockIdx.y * kSpmmSlice;
    const int ncols = min(kSpmmSlice, N - n0);
    const uint32_t seg_bytes = (uint32_t)ncols * 2u;
    const uint16_t* wslice = W + n0;
    // row_ptr[r_begin .. r_end] held by lanes 0..4
    const int rp = (lane <= r_end - r_begin) ? row_ptr[r_begin + lane] : 0;
    const int P0 = __shfl_sync(0xFFFFFFFFu, rp, 0);
    const int P1 = __shfl_sync(0xFFFFFFFFu, rp, r_end - r_begin);
    // prologue: entries P0 .. P0 + 31 into slots 0 .. 31
    {
        const int kn = (P0 + lane < P1) ? col[P0 + lane] : 0;
        for (int t = 0; t < kAsyncDepth; ++t) {
            const int k = __shfl_sync(0xFFFFFFFFu, kn, t);
            if (lane == 0 && P0 + t < P1)
                slot_fetch(&bars[t], ring + t * kAsyncSeg, wslice + (int64_t)k * ldw, seg_bytes);
        }
    }
    const bool lane_ok = lane * 8 < ncols;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
    int row = r_begin;
    int rend = __shfl_sync(0xFFFFFFFFu, rp, 1);
    int consumed = P0;            // entries consumed so far (absolute index)
    bool ok = true;
    auto store_row = [&](int r) {
        if (lane_ok) {
            float4* d = reinterpret_cast<float4*>(C + (int64_t)r * N + n0 + lane * 8);
            d[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            d[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
    };
    for (int B = P0; ok && B < P1; B += kAsyncDepth) {
        const int cnt = min(kAsyncDepth, P1 - B);
        const float vc = (B + lane < P1) ? (float)val[B + lane] : 0.0f;
        const int kn = (B + kAsyncDepth + lane < P1) ? col[B + kAsyncDepth + lane] : 0;
        const uint32_t par = (uint32_t)(((B - P0) / kAsyncDepth) & 1);
        for (int t = 0; t < cnt; ++t) {
            const int j = B + t;
            while (j >= rend) {          // rows that end before entry j
                store_row(row);
                ++row;
                rend = __shfl_sync(0xFFFFFFFFu, rp, row - r_begin + 1);
            }
            const bool got = __all_sync(0xFFFFFFFFu, slot_wait(&bars[t], par));
            if (!got) {
                if (lane == 0) atomicOr(status, kStatusTimeout);
                ok = false;
                break;
            }
            const uint4 w = *reinterpret_cast<const uint4*>(ring + t * kAsyncSeg + lane * 16);
            const float v = __shfl_sync(0xFFFFFFFFu, vc, t);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] = __fmaf_rn(v, __uint_as_float(ww[i] << 16), acc[2 * i]);
                acc[2 * i + 1] = __fmaf_rn(v, __uint_as_float(ww[i] & 0xFFFF0000u), acc[2 * i + 1]);
            }
            consumed = j + 1;
            __syncwarp();                // every lane has read slot t
            const int k = __shfl_sync(0xFFFFFFFFu, kn, t);
            if (lane == 0 && j + kAsyncDepth < P1)
                slot_fetch(&bars[t], ring + t * kAsyncSeg, wslice + (int64_t)k * ldw, seg_bytes);
        }
    }
    if (!ok) {
        // copies issued and not consumed: entries consumed .. min(P1, consumed + 31)
        if (lane == 0) {
            const int last = min(P1, consumed + kAsyncDepth);
            for (int j = consumed; j < last; ++j) {
                const int rel = j - P0;
                const long long t0 = clock64();
                while (!slot_ready(&bars[rel % kAsyncDepth], (uint32_t)((rel / kAsyncDepth) & 1)))
                    if (clock64() - t0 > kSpmmWaitLimit) break;
            }
        }
        __syncwarp();
        return;
    }
    while (row < r_end) {                // the last rows (and empty ones)
        store_row(row);
        ++row;
    }
}

cudaError_t spmm_setup() {
    return cudaFuncSetAttribute(spmm_async_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kAsyncSmem);
}

void launch_spmm(const qg_csr* dA, int64_t M, const void* W, qg_dtype dt, int64_t N, int64_t ldw,
                 float* C, uint32_t* status, cudaStream_t s) {
    if (dt == QG_BF16 && (N % 8) == 0 && (ldw % 8) == 0) {
        const int rows_per_cta = kAsyncWarps * kAsyncRowsPerWarp;
        dim3 grid((unsigned)((M + rows_per_cta - 1) / rows_per_cta),
                  (unsigned)((N + kSpmmSlice - 1) / kSpmmSlice));
        spmm_async_kernel<<<grid, kAsyncWarps * 32, kAsyncSmem, s>>>(
            dA->row_ptr, dA->col, dA->val, static_cast<const uint16_t*>(W), ldw, (int)M, (int)N, C,
            status);
        count_launch(1);
        return;
    }
    dim3 grid((unsigned)((M + kSpmmRowsPerCta - 1) / kSpmmRowsPerCta),
              (unsigned)((N + kSpmmSlice - 1) / kSpmmSlice));
    if (dt == QG_BF16)
        spmm_slice_kernel<QG_BF16><<<grid, kSpmmThreads, 0, s>>>(dA->row_ptr, dA->col, dA->val, W,
                                                                  ldw, (int)M, (int)N, C);
    else
        spmm_slice_kernel<QG_F32><<<grid, kSpmmThreads, 0, s>>>(dA->row_ptr, dA->col, dA->val, W,
                                                                 ldw, (int)M, (int)N, C);
    count_launch(1);
}

}  // namespace qg
