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
// Fast path (bf16 W, N and ldw multiples of 8).  The kernel is bound by
// instruction issue, so the work per non-zero is made as wide as possible:
// a CTA owns a 1024-column slice (each lane 32 columns, in four 256-column
// quarters so every load and store is coalesced), the bf16 pairs feed packed
// fp32x2 FMAs (one rounding per product-sum, as fmaf), and W row segments are
// prefetched with per-lane 16-byte cp.async copies into a per-lane ring of
// kDepth slots in shared memory.  Every lane copies exactly the bytes it will
// read, so no synchronisation between lanes is needed: after committing the
// copy of entry j + kDepth - 1, waiting until at most kDepth - 1 groups are
// pending makes entry j's bytes visible to the lane that copied them.
// A warp owns 4 consecutive rows, whose CSR entries form one contiguous
// range consumed in order.
constexpr int kStreamWarps = 8;
constexpr int kStreamRowsPerWarp = 4;
constexpr int kStreamParts = 4;                   // 256-column quarters per slice
constexpr int kStreamSlice = 256 * kStreamParts;
constexpr int kDepth = 4;
constexpr int kSlotBytes = kStreamParts * 512;    // 32 lanes x 16 bytes per quarter
constexpr size_t kAsyncSmem = (size_t)kStreamWarps * kDepth * kSlotBytes;

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// acc0 += v * lo(w), acc1 += v * hi(w) for a bf16 pair w, as one packed FMA.
__device__ __forceinline__ void fma_bf16x2(float& a0, float& a1, float v, uint32_t w) {
    asm("{\n\t.reg .b32 lo, hi;\n\t.reg .b64 x, acc, vv;\n\t"
        "shl.b32 lo, %3, 16;\n\tand.b32 hi, %3, 0xFFFF0000;\n\t"
        "mov.b64 x, {lo, hi};\n\tmov.b64 acc, {%0, %1};\n\tmov.b64 vv, {%2, %2};\n\t"
        "fma.rn.f32x2 acc, x, vv, acc;\n\tmov.b64 {%0, %1}, acc;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "f"(v), "r"(w));
}

__global__ void __launch_bounds__(kStreamWarps * 32)
spmm_stream_kernel(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col,
                   const double* __restrict__ val, const uint16_t* __restrict__ W, int64_t ldw,
                   int M, int N, float* __restrict__ C) {
    extern __shared__ __align__(128) uint8_t sm[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    // slot s of this lane: quarter h at ring + s * kSlotBytes + h * 512 (16 bytes)
    uint8_t* ring = sm + (size_t)warp * kDepth * kSlotBytes + lane * 16;
    const int r_begin = (blockIdx.x * kStreamWarps + warp) * kStreamRowsPerWarp;
    if (r_begin >= M) return;
    const int r_end = min(M, r_begin + kStreamRowsPerWarp);
    const int nbase = blockIdx.y * kStreamSlice + lane * 8;   // quarter h: nbase + 256 h
    bool okh[kStreamParts];
#pragma unroll
    for (int h = 0; h < kStreamParts; ++h) okh[h] = nbase + 256 * h < N;
    const uint16_t* wl = W + nbase;
    // row_ptr[r_begin .. r_end] held by lanes 0..4
    const int rp = (lane <= r_end - r_begin) ? row_ptr[r_begin + lane] : 0;
    const int P0 = __shfl_sync(0xFFFFFFFFu, rp, 0);
    const int P1 = __shfl_sync(0xFFFFFFFFu, rp, r_end - r_begin);
    // batches of 32 entries: current (kc, vc) and the next one's columns (kn)
    int kc = (P0 + lane < P1) ? col[P0 + lane] : 0;
    float vc = (P0 + lane < P1) ? (float)val[P0 + lane] : 0.0f;
    int kn = (P0 + 32 + lane < P1) ? col[P0 + 32 + lane] : 0;
    auto fetch = [&](int slot, int k) {
        uint8_t* d = ring + slot * kSlotBytes;
        const uint16_t* src = wl + (int64_t)k * ldw;
#pragma unroll
        for (int h = 0; h < kStreamParts; ++h)
            if (okh[h]) cp_async16(d + h * 512, src + 256 * h);
    };
#pragma unroll
    for (int t = 0; t < kDepth - 1; ++t) {
        const int k = __shfl_sync(0xFFFFFFFFu, kc, t);
        if (P0 + t < P1) fetch(t, k);
        cp_async_commit();
    }
    float acc[8 * kStreamParts];
#pragma unroll
    for (int e = 0; e < 8 * kStreamParts; ++e) acc[e] = 0.0f;
    int row = r_begin;
    int rend = __shfl_sync(0xFFFFFFFFu, rp, 1);
    auto store_row = [&](int r) {
        float* crow = C + (int64_t)r * N + nbase;
#pragma unroll
        for (int h = 0; h < kStreamParts; ++h) {
            if (okh[h]) {
                float4* d = reinterpret_cast<float4*>(crow + 256 * h);
                d[0] = make_float4(acc[8 * h + 0], acc[8 * h + 1], acc[8 * h + 2], acc[8 * h + 3]);
                d[1] = make_float4(acc[8 * h + 4], acc[8 * h + 5], acc[8 * h + 6], acc[8 * h + 7]);
            }
        }
#pragma unroll
        for (int e = 0; e < 8 * kStreamParts; ++e) acc[e] = 0.0f;
    };
    for (int B = P0; B < P1; B += 32) {
        const int cnt = min(32, P1 - B);
        for (int t = 0; t < cnt; ++t) {
            const int j = B + t;
            // look-ahead copy of entry j + kDepth - 1
            const int li = t + kDepth - 1;
            const int ka = __shfl_sync(0xFFFFFFFFu, kc, li & 31);
            const int kb = __shfl_sync(0xFFFFFFFFu, kn, li & 31);
            if (j + kDepth - 1 < P1) fetch((j + kDepth - 1 - P0) % kDepth, li < 32 ? ka : kb);
            cp_async_commit();
            while (j >= rend) {          // rows that end before entry j
                store_row(row);
                ++row;
                rend = __shfl_sync(0xFFFFFFFFu, rp, row - r_begin + 1);
            }
            cp_async_wait<kDepth - 1>();
            const uint8_t* src = ring + ((j - P0) % kDepth) * kSlotBytes;
            const float v = __shfl_sync(0xFFFFFFFFu, vc, t);
#pragma unroll
            for (int h = 0; h < kStreamParts; ++h) {
                const uint4 a = *reinterpret_cast<const uint4*>(src + h * 512);
                fma_bf16x2(acc[8 * h + 0], acc[8 * h + 1], v, a.x);
                fma_bf16x2(acc[8 * h + 2], acc[8 * h + 3], v, a.y);
                fma_bf16x2(acc[8 * h + 4], acc[8 * h + 5], v, a.z);
                fma_bf16x2(acc[8 * h + 6], acc[8 * h + 7], v, a.w);
            }
        }
        // advance the batches
        kc = kn;
        vc = (B + 32 + lane < P1) ? (float)val[B + 32 + lane] : 0.0f;
        kn = (B + 64 + lane < P1) ? col[B + 64 + lane] : 0;
    }
    cp_async_wait<0>();
    while (row < r_end) {                // the last rows (and empty ones)
        store_row(row);
        ++row;
    }
}

cudaError_t spmm_setup() {
    return cudaFuncSetAttribute(spmm_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kAsyncSmem);
}

void launch_spmm(const qg_csr* dA, int64_t M, const void* W, qg_dtype dt, int64_t N, int64_t ldw,
                 float* C, uint32_t* status, cudaStream_t s) {
    (void)status;   // no device-side waits that could time out
    if (dt == QG_BF16 && (N % 8) == 0 && (ldw % 8) == 0) {
        const int rows_per_cta = kStreamWarps * kStreamRowsPerWarp;
        dim3 grid((unsigned)((M + rows_per_cta - 1) / rows_per_cta),
                  (unsigned)((N + kStreamSlice - 1) / kStreamSlice));
        spmm_stream_kernel<<<grid, kStreamWarps * 32, kAsyncSmem, s>>>(
            dA->row_ptr, dA->col, dA->val, static_cast<const uint16_t*>(W), ldw, (int)M, (int)N, C);
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
