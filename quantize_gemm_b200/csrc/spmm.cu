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

void launch_spmm(const qg_csr* dA, int64_t M, const void* W, qg_dtype dt, int64_t N, int64_t ldw,
                 float* C, cudaStream_t s) {
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
