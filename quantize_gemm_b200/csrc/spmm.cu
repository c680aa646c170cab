// spmm.cu -- the compensation product C = dA . W of the FP4 linear layer.
//
// Method: QbitAI write-up of "Optimizing LLM Training Using FP4 Quantization"
// (news.movedaos.com/post/4103), outlier clamping and compensation paragraph:
// the clamped-off part dA = A - A_clamped is sparse and is multiplied in
// higher precision than FP4; here fp32 products and sums with W read in its
// stored dtype (bf16 or fp32).
//
// One CTA per row of dA: the row's (col, val) list is shared by all threads,
// each thread owns groups of 8 consecutive output columns, keeps them in
// registers across the row's non-zeros and writes them once (zeros for
// empty rows, so C is fully defined).
#include "qg_internal.cuh"

namespace qg {

constexpr int kSpmmThreads = 256;
constexpr int kSpmmGroups = 4;   // 8-column groups held per thread per pass

template <qg_dtype DT>
__global__ void __launch_bounds__(kSpmmThreads)
spmm_rows_kernel(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col,
                 const double* __restrict__ val, const void* __restrict__ W, int64_t ldw, int N,
                 float* __restrict__ C) {
    const int64_t row = blockIdx.x;
    const int p0 = row_ptr[row], p1 = row_ptr[row + 1];
    const int ngroups = (N + 7) / 8;
    const bool vec_ok = (N % 8) == 0 && (ldw % 8) == 0;
    float* crow = C + row * N;
    for (int g0 = 0; g0 < ngroups; g0 += kSpmmThreads * kSpmmGroups) {
        float acc[kSpmmGroups][8];
#pragma unroll
        for (int i = 0; i < kSpmmGroups; ++i)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[i][e] = 0.0f;
        for (int p = p0; p < p1; ++p) {
            const int64_t k = col[p];
            const float v = (float)val[p];
#pragma unroll
            for (int i = 0; i < kSpmmGroups; ++i) {
                const int g = g0 + threadIdx.x + i * kSpmmThreads;
                if (g >= ngroups) continue;
                float w[8];
                if (vec_ok) {
                    load8<DT>(W, k * ldw + (int64_t)g * 8, w);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int n = g * 8 + e;
                        if (n < N) {
                            if constexpr (DT == QG_BF16)
                                w[e] = __uint_as_float((uint32_t)static_cast<const uint16_t*>(W)[k * ldw + n] << 16);
                            else
                                w[e] = static_cast<const float*>(W)[k * ldw + n];
                        } else {
                            w[e] = 0.0f;
                        }
                    }
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[i][e] = __fmaf_rn(v, w[e], acc[i][e]);
            }
        }
#pragma unroll
        for (int i = 0; i < kSpmmGroups; ++i) {
            const int g = g0 + threadIdx.x + i * kSpmmThreads;
            if (g >= ngroups) continue;
            if (vec_ok) {
                float4* d = reinterpret_cast<float4*>(crow + (int64_t)g * 8);
                d[0] = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
                d[1] = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
            } else {
                for (int e = 0; e < 8; ++e)
                    if (g * 8 + e < N) crow[g * 8 + e] = acc[i][e];
            }
        }
    }
}

void launch_spmm(const qg_csr* dA, int64_t M, const void* W, qg_dtype dt, int64_t N, int64_t ldw,
                 float* C, cudaStream_t s) {
    if (dt == QG_BF16)
        spmm_rows_kernel<QG_BF16><<<(unsigned)M, kSpmmThreads, 0, s>>>(dA->row_ptr, dA->col, dA->val,
                                                                        W, ldw, (int)N, C);
    else
        spmm_rows_kernel<QG_F32><<<(unsigned)M, kSpmmThreads, 0, s>>>(dA->row_ptr, dA->col, dA->val,
                                                                       W, ldw, (int)N, C);
    count_launch(1);
}

}  // namespace qg
