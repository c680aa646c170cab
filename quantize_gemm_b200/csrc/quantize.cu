// quantize.cu -- token-wise (row) and channel-wise (column) E2M1 quantizers
// and the elementwise encoder.
//
// Method: QbitAI write-up of "Optimizing LLM Training Using FP4 Quantization"
// (news.movedaos.com/post/4103): granularity paragraph (rows of A,
// columns of W) and ScaleShift paragraph (scale by 6 / amax, round to the
// nearest E2M1 value; ties to the even code).
//
// Streaming passes with 16-byte loads: the bf16 row quantizer holds a row in
// registers (a warp per row); the bf16 column quantizer is one cooperative
// kernel (partial column maxima, a grid barrier, then 32 x 256 tiles).
#include "qg_internal.cuh"

namespace qg {

// --------------------------------------------------------------------------
// Elementwise encoder: packed[i] = e2m1(x[2i]) | e2m1(x[2i+1]) << 4.
__global__ void e2m1_encode_kernel(const float* __restrict__ x, int64_t n,
                                   uint8_t* __restrict__ packed) {
    const int64_t nchunk = n / 8;
    for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < nchunk;
         c += (int64_t)gridDim.x * blockDim.x) {
        float v[8];
        load8<QG_F32>(x, c * 8, v);
        reinterpret_cast<uint32_t*>(packed)[c] = e2m1x8(v);
    }
    // tail (n even, n % 8 != 0)
    if (blockIdx.x == 0) {
        for (int64_t i = nchunk * 8 + 2 * threadIdx.x; i < n; i += 2 * blockDim.x)
            packed[i / 2] = (uint8_t)e2m1x2(x[i], x[i + 1]);
    }
}

void launch_e2m1_encode(const float* x, int64_t n, uint8_t* packed, cudaStream_t s) {
    int64_t nchunk = n / 8;
    int blocks = (int)std::min<int64_t>((nchunk + 255) / 256, (int64_t)num_sms() * 16);
    if (blocks < 1) blocks = 1;
    e2m1_encode_kernel<<<blocks, 256, 0, s>>>(x, n, packed);
    count_launch(1);
}

// --------------------------------------------------------------------------
// Token-wise quantization without clamp.  One CTA per row; the row stays in
// registers between the max reduction and the encode, so A is read once.
constexpr int kRowThreads = 256;

template <qg_dtype DT, int CPT>
__global__ void __launch_bounds__(kRowThreads)
quantize_rows_kernel(const void* __restrict__ A, int64_t lda, int K,
                     uint8_t* __restrict__ codes, float* __restrict__ scales) {
    const int64_t row = blockIdx.x;
    const int nchunks = K / 8;
    float x[CPT][8];
    uint32_t kmax = 0;
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = threadIdx.x + kRowThreads * i;
        if (c < nchunks) {
            load8<DT>(A, row * lda + (int64_t)c * 8, x[i]);
#pragma unroll
            for (int e = 0; e < 8; ++e) kmax = max(kmax, key_of(x[i][e]));
        }
    }
    __shared__ uint32_t red[kRowThreads / 32];
    kmax = warp_max_u32(kmax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = kmax;
    __syncthreads();
    uint32_t m = 0;
#pragma unroll
    for (int w = 0; w < kRowThreads / 32; ++w) m = max(m, red[w]);
    float r, s;
    scale_factors(__uint_as_float(m), r, s);
    if (threadIdx.x == 0) scales[row] = s;
    uint32_t* out = reinterpret_cast<uint32_t*>(codes + row * (int64_t)(K / 2));
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = threadIdx.x + kRowThreads * i;
        if (c < nchunks) {
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = __fmul_rn(x[i][e], r);
            out[c] = e2m1x8(y);
        }
    }
}

// bf16, K <= 16384: G warps per row (G = 1, 2, 4), each holding its segment
// of SPR steps of 1024 columns in registers (each lane four 16-byte chunks per
// step); the row's max by a 16x2 max, a warp reduction and, for G > 1, a
// shared-memory exchange between the row's warps; then one packed fp32x2
// multiply and one conversion per bf16 pair.  Row groups walk the rows
// grid-stride; the loop bound is uniform over the CTA, so every thread
// reaches each barrier.
constexpr int kRowWarpThreads = 256;

template <int SPR, int G>
__global__ void __launch_bounds__(kRowWarpThreads, SPR >= 4 ? 2 : 3)
quantize_rows_bf16_kernel(const uint16_t* __restrict__ A, int64_t lda, int M, int K,
                          uint8_t* __restrict__ codes, float* __restrict__ scales) {
    constexpr int wpc = kRowWarpThreads / 32;
    constexpr int rpc = wpc / G;                 // rows per CTA per turn
    __shared__ uint32_t part[2][wpc];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = warp % G, slot = warp / G;
    const int nchunks = K / 8;
    const int c0 = sub * SPR * 128 + lane;       // this lane's first chunk
    int turn = 0;
    for (int row0 = blockIdx.x * rpc; row0 < M; row0 += gridDim.x * rpc, turn ^= 1) {
        const int row = row0 + slot;
        const bool active = row < M;
        const uint4* src = reinterpret_cast<const uint4*>(A + (int64_t)(active ? row : 0) * lda);
        uint4 v[SPR][4];
#pragma unroll
        for (int st = 0; st < SPR; ++st)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + st * 128 + 32 * j;
                v[st][j] = (active && c < nchunks) ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
            }
        uint32_t m0 = 0, m1 = 0;
#pragma unroll
        for (int st = 0; st < SPR; ++st)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                m0 = max_u16x2(m0, max_u16x2(v[st][j].x & 0x7FFF7FFFu, v[st][j].y & 0x7FFF7FFFu));
                m1 = max_u16x2(m1, max_u16x2(v[st][j].z & 0x7FFF7FFFu, v[st][j].w & 0x7FFF7FFFu));
            }
        const uint32_t mm = max_u16x2(m0, m1);
        uint32_t key = warp_max_u32(max(mm & 0xFFFFu, mm >> 16));
        if constexpr (G > 1) {
            if (lane == 0) part[turn][warp] = key;
            __syncthreads();
#pragma unroll
            for (int g = 0; g < G; ++g) key = max(key, part[turn][slot * G + g]);
        }
        if (!active) continue;
        float r, sc;
        scale_factors(__uint_as_float(key << 16), r, sc);
        if (sub == 0 && lane == 0) scales[row] = sc;
        uint32_t* out = reinterpret_cast<uint32_t*>(codes + (int64_t)row * (K / 2));
#pragma unroll
        for (int st = 0; st < SPR; ++st)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + st * 128 + 32 * j;
                if (c < nchunks) {
                    const uint32_t q01 = __byte_perm(bf16x2_encode(v[st][j].x, r), bf16x2_encode(v[st][j].y, r), 0x0040);
                    const uint32_t q23 = __byte_perm(bf16x2_encode(v[st][j].z, r), bf16x2_encode(v[st][j].w, r), 0x0040);
                    out[c] = __byte_perm(q01, q23, 0x5410);
                }
            }
    }
}

template <int SPR, int G>
static void launch_rows_bf16(const uint16_t* A, int64_t M, int64_t K, int64_t lda, uint8_t* codes,
                             float* scales, cudaStream_t s) {
    constexpr int rpc = kRowWarpThreads / 32 / G;
    const int grid = (int)std::max<int64_t>(
        1, std::min<int64_t>((M + rpc - 1) / rpc, (int64_t)num_sms() * (SPR >= 4 ? 2 : 3)));
    quantize_rows_bf16_kernel<SPR, G><<<grid, kRowWarpThreads, 0, s>>>(A, lda, (int)M, (int)K, codes,
                                                                      scales);
}

template <qg_dtype DT>
static void launch_rows_dt(const void* A, int64_t M, int64_t K, int64_t lda, uint8_t* codes,
                           float* scales, cudaStream_t s) {
    const int64_t nchunks = K / 8;
    const int cpt = (int)((nchunks + kRowThreads - 1) / kRowThreads);
    dim3 grid((unsigned)M);
    if (cpt <= 1) quantize_rows_kernel<DT, 1><<<grid, kRowThreads, 0, s>>>(A, lda, (int)K, codes, scales);
    else if (cpt <= 2) quantize_rows_kernel<DT, 2><<<grid, kRowThreads, 0, s>>>(A, lda, (int)K, codes, scales);
    else if (cpt <= 4) quantize_rows_kernel<DT, 4><<<grid, kRowThreads, 0, s>>>(A, lda, (int)K, codes, scales);
    else quantize_rows_kernel<DT, 8><<<grid, kRowThreads, 0, s>>>(A, lda, (int)K, codes, scales);
    count_launch(1);
}

void launch_quantize_rows(const void* A, qg_dtype dt, int64_t M, int64_t K, int64_t lda,
                          uint8_t* codes, float* scales, cudaStream_t s) {
    if (dt == QG_BF16 && K <= 16384) {
        // steps of 1024 columns; G warps per row, SPR steps per warp
        const int steps = (int)((K / 8 + 127) / 128);
        const uint16_t* Ab = static_cast<const uint16_t*>(A);
        if (steps <= 1) launch_rows_bf16<1, 1>(Ab, M, K, lda, codes, scales, s);
        else if (steps == 2) launch_rows_bf16<2, 1>(Ab, M, K, lda, codes, scales, s);
        else if (steps == 3) launch_rows_bf16<3, 1>(Ab, M, K, lda, codes, scales, s);
        else if (steps == 4) launch_rows_bf16<4, 1>(Ab, M, K, lda, codes, scales, s);
        else if (steps <= 6) launch_rows_bf16<3, 2>(Ab, M, K, lda, codes, scales, s);
        else if (steps <= 8) launch_rows_bf16<4, 2>(Ab, M, K, lda, codes, scales, s);
        else if (steps <= 12) launch_rows_bf16<3, 4>(Ab, M, K, lda, codes, scales, s);
        else launch_rows_bf16<4, 4>(Ab, M, K, lda, codes, scales, s);
        count_launch(1);
        return;
    }
    if (dt == QG_BF16) launch_rows_dt<QG_BF16>(A, M, K, lda, codes, scales, s);
    else launch_rows_dt<QG_F32>(A, M, K, lda, codes, scales, s);
}

// --------------------------------------------------------------------------
// Channel-wise quantization of W (K x N row-major) into codesT (N x K/2).
// Pass 1: column maxima (split over K, combined with atomicMax on the keys).
// Pass 2: a 32 (k) x 256 (n) tile goes through shared memory and each thread
//         encodes one column's 32 values into 16 output bytes.
template <qg_dtype DT>
__device__ __forceinline__ float load1(const void* base, int64_t idx) {
    if constexpr (DT == QG_BF16)
        return __uint_as_float((uint32_t)static_cast<const uint16_t*>(base)[idx] << 16);
    else
        return static_cast<const float*>(base)[idx];
}

// Pass 1: a CTA owns 256 columns (8 per lane) and a range of rows; its 8 warps
// split the rows, reduce in shared memory, and issue one atomicMax per column.
template <qg_dtype DT>
__global__ void __launch_bounds__(256)
colmax_kernel(const void* __restrict__ W, int64_t ldw, int K, int N, int rows_per_split,
              uint32_t* __restrict__ colmax) {
    __shared__ uint32_t red[8][256];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n0 = blockIdx.x * 256 + lane * 8;
    const int k0 = blockIdx.y * rows_per_split;
    const int k1 = min(K, k0 + rows_per_split);
    uint32_t m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (n0 < N) {
        const bool vec = (n0 + 8 <= N) && ((ldw & 7) == 0 || DT == QG_F32) && ((ldw & 3) == 0);
        int k = k0 + warp;
        for (; vec && k + 8 < k1; k += 16) {     // two rows in flight per lane
            float x[8], y[8];
            load8<DT>(W, (int64_t)k * ldw + n0, x);
            load8<DT>(W, (int64_t)(k + 8) * ldw + n0, y);
#pragma unroll
            for (int e = 0; e < 8; ++e) m[e] = max(m[e], max(key_of(x[e]), key_of(y[e])));
        }
        for (; k < k1; k += 8) {
            float x[8];
            if (vec) {
                load8<DT>(W, (int64_t)k * ldw + n0, x);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = (n0 + e < N) ? load1<DT>(W, (int64_t)k * ldw + n0 + e) : 0.0f;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) m[e] = max(m[e], key_of(x[e]));
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[warp][lane * 8 + e] = m[e];
    __syncthreads();
    const int c = threadIdx.x;          // one column per thread
    uint32_t v = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) v = max(v, red[w][c]);
    const int n = blockIdx.x * 256 + c;
    if (n < N && v != 0) atomicMax(&colmax[n], v);
}

constexpr int kColTileK = 32;
constexpr int kColTileN = 256;

template <qg_dtype DT>
__global__ void __launch_bounds__(256)
quantize_cols_kernel(const void* __restrict__ W, int64_t ldw, int K, int N,
                     const uint32_t* __restrict__ colmax, uint8_t* __restrict__ codesT,
                     float* __restrict__ scales) {
    __shared__ float tile[kColTileK][kColTileN];
    const int n_base = blockIdx.x * kColTileN;
    const int k_base = blockIdx.y * kColTileK;
    const int t = threadIdx.x;
    // load: warp w covers rows w, w + 8, ...; lane covers 8 consecutive columns
    const int lane = t & 31, warp = t >> 5;
    const int nc = n_base + lane * 8;
    const bool vec = (nc + 8 <= N) && ((ldw & 7) == 0 || DT == QG_F32) && ((ldw & 3) == 0);
    for (int kr = warp; kr < kColTileK; kr += 8) {
        const int k = k_base + kr;
        float x[8];
        if (vec) {
            load8<DT>(W, (int64_t)k * ldw + nc, x);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = (nc + e < N) ? load1<DT>(W, (int64_t)k * ldw + nc + e) : 0.0f;
        }
        float4* dst = reinterpret_cast<float4*>(&tile[kr][lane * 8]);
        dst[0] = make_float4(x[0], x[1], x[2], x[3]);
        dst[1] = make_float4(x[4], x[5], x[6], x[7]);
    }
    __syncthreads();
    const int n = n_base + t;
    if (n >= N) return;
    float r, s;
    scale_factors(__uint_as_float(colmax[n]), r, s);
    if (blockIdx.y == 0) scales[n] = s;
    uint32_t packed[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float y[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = __fmul_rn(tile[q * 8 + e][t], r);
        packed[q] = e2m1x8(y);
    }
    uint4* dst = reinterpret_cast<uint4*>(codesT + (int64_t)n * (K / 2) + k_base / 2);
    *dst = make_uint4(packed[0], packed[1], packed[2], packed[3]);
}

// --------------------------------------------------------------------------
// bf16 W in one cooperative launch (all CTAs resident):
//   phase 1  unit (split s, 256-column block): the max key of each column over
//            the split's rows -> colpart[s][n] (no atomics, nothing to zero)
//   barrier
//   phase 2  tiles of 32 rows x 64 columns, one warp each and a warp's tiles
//            consecutive in (column group, row tile) order: the column scales
//            from the partial maxima (once per column group), the tile
//            through the warp's own shared memory (W is read a second time,
//            partly from L2; only __syncwarp, so warps never wait for one
//            another), each lane encodes two adjacent columns (32 values
//            each into 16 output bytes); the next tile's loads are in flight
//            while the current one is encoded.
constexpr int kColsFusedThreads = 256;
constexpr int kColsMaxSplits = 32;
constexpr int kColsWarpTileN = 64;      // columns of a phase-2 warp tile

__global__ void __launch_bounds__(kColsFusedThreads)
quantize_cols_fused_bf16_kernel(const uint16_t* __restrict__ W, int64_t ldw, int K, int N,
                                int splits, int rows_per_split, uint32_t* __restrict__ colpart,
                                uint8_t* __restrict__ codesT, float* __restrict__ scales,
                                GridSync* __restrict__ gsync, uint32_t* __restrict__ status) {
    __shared__ uint32_t red[8][256];
    __shared__ __align__(16) uint16_t wtile[kColsFusedThreads / 32][kColTileK][kColsWarpTileN];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int cblocks = (N + 255) / 256;
    const bool ld_vec = (ldw & 7) == 0;

    // phase 1
    for (int u = blockIdx.x; u < cblocks * splits; u += gridDim.x) {
        const int cb = u % cblocks, sp = u / cblocks;
        const int n0 = cb * 256 + lane * 8;
        const int k0 = sp * rows_per_split, k1 = min(K, k0 + rows_per_split);
        uint32_t m[4] = {0u, 0u, 0u, 0u};   // 16x2 maxima of the lane's 8 columns
        if (n0 < N) {
            if (ld_vec && n0 + 8 <= N) {
                int k = k0 + warp;
                for (; k + 24 < k1; k += 32) {      // four rows in flight per lane
                    uint4 a[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        a[u] = __ldg(reinterpret_cast<const uint4*>(W + (int64_t)(k + 8 * u) * ldw + n0));
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        m[0] = max_u16x2(m[0], a[u].x & 0x7FFF7FFFu);
                        m[1] = max_u16x2(m[1], a[u].y & 0x7FFF7FFFu);
                        m[2] = max_u16x2(m[2], a[u].z & 0x7FFF7FFFu);
                        m[3] = max_u16x2(m[3], a[u].w & 0x7FFF7FFFu);
                    }
                }
                for (; k < k1; k += 8) {
                    const uint4 a = __ldg(reinterpret_cast<const uint4*>(W + (int64_t)k * ldw + n0));
                    m[0] = max_u16x2(m[0], a.x & 0x7FFF7FFFu);
                    m[1] = max_u16x2(m[1], a.y & 0x7FFF7FFFu);
                    m[2] = max_u16x2(m[2], a.z & 0x7FFF7FFFu);
                    m[3] = max_u16x2(m[3], a.w & 0x7FFF7FFFu);
                }
            } else {
                for (int k = k0 + warp; k < k1; k += 8) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        if (n0 + e >= N) continue;
                        const uint32_t key = W[(int64_t)k * ldw + n0 + e] & 0x7FFFu;
                        const uint32_t sh = (e & 1) ? 16 : 0;
                        m[e >> 1] = max_u16x2(m[e >> 1], key << sh);
                    }
                }
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) red[warp][lane * 8 + e] = (e & 1) ? (m[e >> 1] >> 16) : (m[e >> 1] & 0xFFFFu);
        __syncthreads();
        uint32_t v = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) v = max(v, red[w][t]);
        const int n = cb * 256 + t;
        if (n < N) colpart[(int64_t)sp * N + n] = v;
        __syncthreads();   // red is reused by the next unit
    }

    uint32_t gen0;
    if (grid_arrive(gsync, gen0)) grid_release(gsync);
    else if (!grid_wait(gsync, gen0, status)) return;

    // phase 2
    const int ktiles = K / kColTileK;
    const int cgroups = (N + kColsWarpTileN - 1) / kColsWarpTileN;
    const int total = cgroups * ktiles;                 // units (column group, row tile)
    const int gw = blockIdx.x * (kColsFusedThreads / 32) + warp;
    const int nw = gridDim.x * (kColsFusedThreads / 32);
    const int per = (total + nw - 1) / nw;
    const int u0 = min(total, gw * per), u1 = min(total, u0 + per);
    uint16_t (*tl)[kColsWarpTileN] = wtile[warp];
    // this lane's part of a unit: rows lane / 8 + 4 i (i < 8), columns
    // 8 (lane % 8) .. + 7 of the group
    auto load_unit = [&](int u, uint4 (&v)[8]) {
        const int cg = u / ktiles, kt = u - cg * ktiles;
        const int nc = cg * kColsWarpTileN + (lane & 7) * 8;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int k = kt * kColTileK + (lane >> 3) + 4 * i;
            v[i] = make_uint4(0u, 0u, 0u, 0u);
            if (ld_vec && nc + 8 <= N) {
                v[i] = __ldg(reinterpret_cast<const uint4*>(W + (int64_t)k * ldw + nc));
            } else if (nc < N) {
                uint16_t h[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) h[e] = (nc + e < N) ? W[(int64_t)k * ldw + nc + e] : (uint16_t)0;
                v[i] = make_uint4(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16),
                                  h[4] | ((uint32_t)h[5] << 16), h[6] | ((uint32_t)h[7] << 16));
            }
        }
    };
    uint4 nxt[8];
    if (u0 < u1) load_unit(u0, nxt);
    int cur_cg = -1;
    float r0 = 0.0f, r1 = 0.0f;
    for (int u = u0; u < u1; ++u) {
        const int cg = u / ktiles, kt = u - cg * ktiles;
        __syncwarp();   // the previous unit's reads of the tile are done
#pragma unroll
        for (int i = 0; i < 8; ++i)
            *reinterpret_cast<uint4*>(&tl[(lane >> 3) + 4 * i][(lane & 7) * 8]) = nxt[i];
        __syncwarp();
        if (u + 1 < u1) load_unit(u + 1, nxt);   // in flight while this unit is encoded
        const int n0 = cg * kColsWarpTileN + 2 * lane;   // this lane's columns n0, n0 + 1
        if (cg != cur_cg) {
            uint32_t key0 = 0, key1 = 0;
            for (int sp = 0; sp < splits; ++sp) {
                if (n0 < N) key0 = max(key0, __ldcg(colpart + (int64_t)sp * N + n0));
                if (n0 + 1 < N) key1 = max(key1, __ldcg(colpart + (int64_t)sp * N + n0 + 1));
            }
            float sc0, sc1;
            scale_factors(__uint_as_float(key0 << 16), r0, sc0);
            scale_factors(__uint_as_float(key1 << 16), r1, sc1);
            if (kt == 0) {
                if (n0 < N) scales[n0] = sc0;
                if (n0 + 1 < N) scales[n0 + 1] = sc1;
            }
            cur_cg = cg;
        }
        // column n0 is the low bf16 of each 32-bit word of the lane's pair, n0 + 1 the high one
        const uint32_t* tw = reinterpret_cast<const uint32_t*>(&tl[0][0]) + lane;
        uint32_t p0[4], p1[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float y0[8], y1[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint32_t w = tw[(q * 8 + e) * (kColsWarpTileN / 2)];
                y0[e] = __fmul_rn(__uint_as_float(w << 16), r0);
                y1[e] = __fmul_rn(__uint_as_float(w & 0xFFFF0000u), r1);
            }
            p0[q] = e2m1x8(y0);
            p1[q] = e2m1x8(y1);
        }
        if (n0 < N)
            *reinterpret_cast<uint4*>(codesT + (int64_t)n0 * (K / 2) + kt * (kColTileK / 2)) =
                make_uint4(p0[0], p0[1], p0[2], p0[3]);
        if (n0 + 1 < N)
            *reinterpret_cast<uint4*>(codesT + (int64_t)(n0 + 1) * (K / 2) + kt * (kColTileK / 2)) =
                make_uint4(p1[0], p1[1], p1[2], p1[3]);
    }
}

// Resident CTAs per SM of the cooperative column kernel, per device.
static int g_cols_blocks[64];

cudaError_t cols_setup() {
    int dev = 0, coop = 0, nb = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
    if (e != cudaSuccess) return e;
    if (cooperative_disabled()) coop = 0;
    if (coop) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, quantize_cols_fused_bf16_kernel,
                                                          kColsFusedThreads, 0);
        if (e != cudaSuccess) return e;
    }
    if (dev >= 0 && dev < 64) g_cols_blocks[dev] = coop ? nb : 0;
    return cudaSuccess;
}

size_t cols_fused_scratch_words(int64_t N) { return (size_t)kColsMaxSplits * (size_t)N; }

bool launch_quantize_cols_fused(const void* W, int64_t K, int64_t N, int64_t ldw, uint8_t* codesT,
                                float* scales, uint32_t* colpart, GridSync* gsync,
                                uint32_t* status, cudaStream_t s) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    const int nb = g_cols_blocks[dev];
    if (nb < 1) return false;
    const int cblocks = (int)((N + 255) / 256);
    const int ktiles = (int)(K / kColTileK);
    const int grid = (int)std::max<int64_t>(
        1, std::min<int64_t>((int64_t)nb * num_sms(), (int64_t)cblocks * ktiles));
    // splits: at most one unit per CTA, at least 32 rows per split
    int splits = (int)std::max<int64_t>(1, grid / cblocks);
    splits = (int)std::min<int64_t>({(int64_t)splits, (int64_t)kColsMaxSplits, std::max<int64_t>(1, K / 32)});
    const int rows_per = (int)((K + splits - 1) / splits);
    splits = (int)((K + rows_per - 1) / rows_per);
    const uint16_t* Wb = static_cast<const uint16_t*>(W);
    int Ki = (int)K, Ni = (int)N;
    void* args[] = {(void*)&Wb, (void*)&ldw, (void*)&Ki, (void*)&Ni, (void*)&splits, (void*)&rows_per,
                    (void*)&colpart, (void*)&codesT, (void*)&scales, (void*)&gsync, (void*)&status};
    const cudaError_t e = cudaLaunchCooperativeKernel((const void*)quantize_cols_fused_bf16_kernel,
                                                      dim3((unsigned)grid), dim3(kColsFusedThreads),
                                                      args, 0, s);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    count_launch(1);
    return true;
}

__global__ void zero_u32_kernel(uint32_t* __restrict__ p, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        p[i] = 0u;
}

void launch_zero_u32(uint32_t* p, int64_t n, cudaStream_t s) {
    int blocks = (int)std::min<int64_t>((n + 255) / 256, (int64_t)num_sms() * 4);
    if (blocks < 1) blocks = 1;
    zero_u32_kernel<<<blocks, 256, 0, s>>>(p, n);
    count_launch(1);
}

void launch_quantize_cols(const void* W, qg_dtype dt, int64_t K, int64_t N, int64_t ldw,
                          uint8_t* codesT, float* scales, uint32_t* colmax, cudaStream_t s) {
    launch_zero_u32(colmax, N, s);
    // enough CTAs for two waves, but at least 64 rows per CTA
    const int col_blocks = (int)((N + 255) / 256);
    int splits = (int)std::max<int64_t>(1, (2 * num_sms() + col_blocks - 1) / col_blocks);
    splits = (int)std::min<int64_t>(splits, std::max<int64_t>(1, K / 64));
    const int rows_per = (int)((K + splits - 1) / splits);
    splits = (int)((K + rows_per - 1) / rows_per);
    dim3 g1(col_blocks, splits);
    dim3 g2((unsigned)((N + kColTileN - 1) / kColTileN), (unsigned)(K / kColTileK));
    if (dt == QG_BF16) {
        colmax_kernel<QG_BF16><<<g1, 256, 0, s>>>(W, ldw, (int)K, (int)N, rows_per, colmax);
        quantize_cols_kernel<QG_BF16><<<g2, 256, 0, s>>>(W, ldw, (int)K, (int)N, colmax, codesT, scales);
    } else {
        colmax_kernel<QG_F32><<<g1, 256, 0, s>>>(W, ldw, (int)K, (int)N, rows_per, colmax);
        quantize_cols_kernel<QG_F32><<<g2, 256, 0, s>>>(W, ldw, (int)K, (int)N, colmax, codesT, scales);
    }
    count_launch(2);
}

}  // namespace qg
