// mx.cu -- MXFP4 block quantization: E2M1 codes with one E8M0 scale per 32
// consecutive elements along the contraction dimension.
//
// Method: the micro-scaling section of the lecture page "FP4量化训练的硬件挑战：
// NVIDIA Blackwell架构上的微缩放格式（Micro-scaling）实现" (zyxy.net/?p=24232):
// group the tensor, scale each group by its largest magnitude, divide and round
// to FP4; and the micro-scaling paragraph of the low-precision training survey
// (10100.com/article/123065115): the block scale is an E8M0 power of two.
// Block scale 2^e with e the smallest exponent such that 6 * 2^e >= amax of the
// block (the block max lands in the E2M1 range without clipping), e clamped to
// [-127, 126]; codes E2M1(fp32(x * 2^-e)) by the hardware conversion.
//
// Codes are row-major (M x K/2, two codes per byte, even k in the low nibble),
// as for the per-row quantizer.  The scales are written in the layout the
// block-scaled GEMM reads ("atoms"): rows in blocks of 128, K in groups of
// 128 (4 blocks); one 512-byte atom per (row block, k group), atoms ordered
// k group fastest, 2 * ceil(K / 256) groups per row block (the last one may
// be padding); inside an atom the scale of row r (0..127 in the block) and
// block j (0..3 in the group) is byte (r % 32) * 16 + (r / 32) * 4 + j.
// Rows past M and blocks past K / 32 hold 127 (2^0).
#include "qg_internal.cuh"

namespace qg {

constexpr int kMxThreads = 256;

// e from the fp32 bit pattern of a finite, non-negative amax: with
// amax = m * 2^E, m in [1, 2), 6 * 2^e >= amax first holds at e = E - 2 when
// m <= 1.5 and at e = E - 1 otherwise; zero and subnormal maxima give -127.
__device__ __forceinline__ int mx_exponent_bits(uint32_t abits) {
    const int ex = (int)(abits >> 23);
    if (ex == 0) return -127;
    const int e = ex - 129 + ((abits & 0x7FFFFFu) > 0x400000u ? 1 : 0);
    return e < -127 ? -127 : (e > 126 ? 126 : e);
}

__device__ __forceinline__ int64_t mx_atom_byte(int64_t r, int64_t kb, int64_t groups) {
    return ((r >> 7) * groups + (kb >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (kb & 3);
}

// A warp per unit (row r, 256 columns c): lane l holds the 8 elements of
// block 8 c + l / 4 starting at column 256 c + 8 l; the four lanes of a block
// reduce its max by shuffles.  Rows up to the padded row count, so every
// scale byte of the atoms is written.
template <qg_dtype DT>
__global__ void __launch_bounds__(kMxThreads)
mx_quantize_rows_kernel(const void* __restrict__ A, int64_t lda, int M, int K, int Mp,
                        uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                        uint32_t* __restrict__ status) {
    const int lane = threadIdx.x & 31;
    const int chunks = (K + 255) / 256;
    const int64_t groups = 2 * (int64_t)chunks;
    const int64_t units = (int64_t)Mp * chunks;
    const int64_t nwarps = (int64_t)gridDim.x * (kMxThreads / 32);
    for (int64_t u = (int64_t)blockIdx.x * (kMxThreads / 32) + (threadIdx.x >> 5); u < units;
         u += nwarps) {
        const int r = (int)(u / chunks);
        const int c = (int)(u - (int64_t)r * chunks);
        const int col = 256 * c + 8 * lane;
        const bool live = r < M && col < K;
        float x[8];
        uint32_t amax = 0;   // fp32 bit pattern of the max magnitude
        if (DT == QG_BF16) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (live) v = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(A) + (int64_t)r * lda + col));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                m = max_u16x2(m, w[i] & 0x7FFF7FFFu);
                x[2 * i] = __uint_as_float(w[i] << 16);
                x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            }
            amax = max(m & 0xFFFFu, m >> 16) << 16;
        } else {
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
            if (live) {
                const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(A) + (int64_t)r * lda + col);
                a = __ldg(src);
                b = __ldg(src + 1);
            }
            x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
            x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = max(amax, __float_as_uint(x[i]) & 0x7FFFFFFFu);
        }
        amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
        if (live && amax >= 0x7F800000u && (lane & 3) == 0) flag_status(status, kStatusNonFinite);
        const int e = mx_exponent_bits(amax);
        const float inv = __uint_as_float((uint32_t)(127 - e) << 23);
        if (live) {
            float y[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = __fmul_rn(x[i], inv);
            *reinterpret_cast<uint32_t*>(codes + (int64_t)r * (K / 2) + col / 2) = e2m1x8(y);
        }
        if ((lane & 3) == 0) {
            const int64_t kb = 8 * (int64_t)c + (lane >> 2);
            sf[mx_atom_byte(r, kb, groups)] = (uint8_t)(live ? e + 127 : 127);
        }
    }
}

// Columns of W (K x N, blocks along K): a CTA stages a 32 (k) x 256 (n) tile
// in shared memory (one k block), thread j encodes column j's block into 16
// code bytes of row j of codesT and one scale byte.  The grid covers the
// padded column count in steps of 256 and the padded k blocks.
template <qg_dtype DT>
__global__ void __launch_bounds__(kMxThreads)
mx_quantize_cols_kernel(const void* __restrict__ W, int64_t ldw, int K, int N, int Np,
                        uint8_t* __restrict__ codesT, uint8_t* __restrict__ sf,
                        uint32_t* __restrict__ status) {
    __shared__ float tile[32][257];
    const int n0 = blockIdx.x * 256;
    const int kb = blockIdx.y;               // k block (32 rows of W)
    const int k0 = 32 * kb;
    const int chunks = (K + 255) / 256;
    const int64_t groups = 2 * (int64_t)chunks;
    const bool kin = k0 < K;
    // coalesced loads: warp w reads rows w, w + 8, ...; lane covers 8 columns
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int rr = warp; rr < 32; rr += kMxThreads / 32) {
        const int k = k0 + rr;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int n = n0 + lane + 32 * e;
            float v = 0.0f;
            if (kin && n < N) {
                if (DT == QG_BF16)
                    v = __uint_as_float((uint32_t)__ldg(static_cast<const uint16_t*>(W) + (int64_t)k * ldw + n) << 16);
                else
                    v = __ldg(static_cast<const float*>(W) + (int64_t)k * ldw + n);
            }
            tile[rr][lane + 32 * e] = v;
        }
    }
    __syncthreads();
    const int j = threadIdx.x;
    const int n = n0 + j;
    if (n >= Np) return;
    const bool live = kin && n < N;
    uint32_t amax = 0;
#pragma unroll
    for (int t = 0; t < 32; ++t) amax = max(amax, __float_as_uint(tile[t][j]) & 0x7FFFFFFFu);
    if (live && amax >= 0x7F800000u) flag_status(status, kStatusNonFinite);
    const int e = mx_exponent_bits(amax);
    if (live) {
        const float inv = __uint_as_float((uint32_t)(127 - e) << 23);
        uint32_t out[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float y[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = __fmul_rn(tile[8 * q + i][j], inv);
            out[q] = e2m1x8(y);
        }
        *reinterpret_cast<uint4*>(codesT + (int64_t)n * (K / 2) + k0 / 2) =
            make_uint4(out[0], out[1], out[2], out[3]);
    }
    sf[mx_atom_byte(n, kb, groups)] = (uint8_t)(live ? e + 127 : 127);
}

void launch_mx_quantize_rows(const void* A, qg_dtype dt, int64_t M, int64_t K, int64_t lda,
                             uint8_t* codes, uint8_t* sf, uint32_t* status, cudaStream_t s) {
    const int64_t Mp = (M + 127) / 128 * 128;
    const int64_t units = Mp * ((K + 255) / 256);
    const int grid = (int)std::max<int64_t>(
        1, std::min<int64_t>((units + kMxThreads / 32 - 1) / (kMxThreads / 32), (int64_t)num_sms() * 8));
    if (dt == QG_BF16)
        mx_quantize_rows_kernel<QG_BF16><<<grid, kMxThreads, 0, s>>>(A, lda, (int)M, (int)K, (int)Mp,
                                                                    codes, sf, status);
    else
        mx_quantize_rows_kernel<QG_F32><<<grid, kMxThreads, 0, s>>>(A, lda, (int)M, (int)K, (int)Mp,
                                                                   codes, sf, status);
    count_launch(1);
}

void launch_mx_quantize_cols(const void* W, qg_dtype dt, int64_t K, int64_t N, int64_t ldw,
                             uint8_t* codesT, uint8_t* sf, uint32_t* status, cudaStream_t s) {
    const int64_t Np = (N + 127) / 128 * 128;
    dim3 grid((unsigned)((Np + 255) / 256), (unsigned)(8 * ((K + 255) / 256)));
    if (dt == QG_BF16)
        mx_quantize_cols_kernel<QG_BF16><<<grid, kMxThreads, 0, s>>>(W, ldw, (int)K, (int)N, (int)Np,
                                                                    codesT, sf, status);
    else
        mx_quantize_cols_kernel<QG_F32><<<grid, kMxThreads, 0, s>>>(W, ldw, (int)K, (int)N, (int)Np,
                                                                   codesT, sf, status);
    count_launch(1);
}

}  // namespace qg
