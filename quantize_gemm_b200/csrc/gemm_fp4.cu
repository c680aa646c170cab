// gemm_fp4.cu -- FP4 (E2M1) GEMM on the sm_100a tensor cores (tcgen05) with
// the dequantization epilogue of the FP4 linear layer.
//
//   acc_ij = sum_k e2m1(A_ik) * e2m1(W_jk)         (fp32 accumulator in TMEM)
//   Y_ij   = acc_ij * sA_i * sW_j (+ C_ij)           (epilogue)
//
// Method: QbitAI write-up of "Optimizing LLM Training Using FP4 Quantization"
// (news.movedaos.com/post/4103): the FP4 GEMM kernel paragraph, and the
// granularity paragraph -- row scales of A and column scales of W factor out
// of the k-sum, so dequantization is a rank-1 scaling in the epilogue.  The
// page's kernel emulated FP4 on FP8 tensor cores through FP16 shared memory;
// here the operands stay packed 4-bit end to end and run on the native block-
// scaled FP4 MMA (tcgen05.mma kind::mxf4) with every block scale set to
// UE8M0 1.0, which makes each MMA the plain E2M1 product.
//
// Structure (one CTA per SM, persistent over 128 x BN output tiles):
//   warp 0     TMA producer: 128-byte-swizzled 128 x 256 and BN x 256 FP4
//              tiles of A and W^T into a kStages-deep shared-memory ring
//   warp 1     TMEM allocator and MMA issuer (one thread): 4 MMAs of
//              K = 64 per 256-wide k-block, accumulating in TMEM
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (one TMEM lane
//              quarter each), scale, add C, store fp32 / bf16
// Every mbarrier wait is bounded; a wait that gives up sets the timeout bit in
// the status word, raises a CTA-wide abort flag, waits (bounded) for copies
// and MMAs in flight, frees TMEM and returns.
#include <cuda.h>

#include "qg_internal.cuh"

namespace qg {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK_BYTES = 128;       // 256 E2M1 values per row per k-block
constexpr int UMMA_K_BYTES = 32;    // 64 E2M1 values per MMA
constexpr int kStages = 4;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kTmemCols = 512;
constexpr int kSfaCol = 448;        // constant block-scale region (0x7F = 2^0)
constexpr int kSfbCol = 480;
constexpr long long kWaitLimit = 2000000000LL;  // SM clocks (~1-2 s)

constexpr int kStageABytes = BM * BK_BYTES;
constexpr int kStageBBytes = BN * BK_BYTES;

struct alignas(8) Barriers {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t acc_full;
    uint64_t acc_empty;
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kSmemBytes =
    1024 /*alignment slack*/ + (size_t)kStages * (kStageABytes + kStageBBytes) + sizeof(Barriers);

// ------------------------------------------------------------------ PTX wraps
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait.  Returns false when the CTA is aborting or the limit passed.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Barriers* B,
                                          uint32_t* status) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*reinterpret_cast<volatile int*>(&B->abort)) return false;
        if (clock64() - t0 > kWaitLimit) {
            *reinterpret_cast<volatile int*>(&B->abort) = 1;
            flag_status(status, kStatusTimeout);
            return false;
        }
    }
}
// Bounded wait used during teardown (ignores the abort flag).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > kWaitLimit) return;
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint64_t* bar, void* dst,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (tile base 1024-byte aligned).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;             // leading byte offset (unused for this layout)
    d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset
    d |= (uint64_t)1 << 46;             // descriptor version
    d |= (uint64_t)2 << 61;             // 128-byte swizzle
    return d;
}

// Instruction descriptor of the block-scaled MMA: E2M1 x E2M1, UE8M0 scales,
// both operands K-major, M = 128, N = BN, dense K = 64.
__device__ __forceinline__ uint32_t mma_idesc() {
    return (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | (1u << 23) |
           ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;"
        "\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb));
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
          "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
          "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
          "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st32_const(uint32_t taddr, uint32_t c) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,"
        "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
        "r"(c)
        : "memory");
}

// ------------------------------------------------------------------ kernel
struct Params {
    const float* sA;
    const float* sW;
    const float* C;      // nullable
    void* Y;             // nullable
    float* raw_acc;      // nullable
    uint32_t* status;
    int M, N, K;
    int y_bf16;
};

__device__ __forceinline__ void tile_coords(int tile, int num_m, int& m_blk, int& n_blk) {
    m_blk = tile % num_m;
    n_blk = tile / num_m;
}

__global__ void __launch_bounds__(kThreads, 1)
fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                const __grid_constant__ CUtensorMap tmap_b, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* sa = smem;
    uint8_t* sb = smem + (size_t)kStages * kStageABytes;
    Barriers* B = reinterpret_cast<Barriers*>(sb + (size_t)kStages * kStageBBytes);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_m = (p.M + BM - 1) / BM;
    const int num_n = (p.N + BN - 1) / BN;
    const int num_tiles = num_m * num_n;
    const int num_kb = (p.K / 2 + BK_BYTES - 1) / BK_BYTES;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&B->full[s], 1);
            mbar_init(&B->empty[s], 1);
        }
        mbar_init(&B->acc_full, 1);
        mbar_init(&B->acc_empty, kEpiWarps);
        mbar_init(&B->mma_done, 1);
        B->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_b)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&B->tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = B->tmem_base;

    if (warp >= 2) {
        // constant block scales: every byte 0x7F (UE8M0 2^0) in the scale region
        const uint32_t q = (uint32_t)(warp & 3);
        tmem_st32_const(tmem + ((32u * q) << 16) + kSfaCol, 0x7F7F7F7Fu);
        tmem_st32_const(tmem + ((32u * q) << 16) + kSfbCol, 0x7F7F7F7Fu);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            bool pend[kStages];
            uint32_t pend_par[kStages];
            for (int s = 0; s < kStages; ++s) pend[s] = false, pend_par[s] = 0;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                int m_blk, n_blk;
                tile_coords(tile, num_m, m_blk, n_blk);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&B->empty[stage], phase ^ 1u, B, p.status)) {
                        ok = false;
                        break;
                    }
                    pend[stage] = false;
                    mbar_expect_tx(&B->full[stage], (uint32_t)(kStageABytes + kStageBBytes));
                    tma_load_2d(&tmap_a, &B->full[stage], sa + (size_t)stage * kStageABytes,
                                kb * BK_BYTES, m_blk * BM);
                    tma_load_2d(&tmap_b, &B->full[stage], sb + (size_t)stage * kStageBBytes,
                                kb * BK_BYTES, n_blk * BN);
                    pend[stage] = true;
                    pend_par[stage] = phase;
                    if (++stage == kStages) stage = 0, phase ^= 1u;
                }
            }
            // copies still in flight complete before the CTA exits
            for (int s = 0; s < kStages; ++s)
                if (pend[s]) mbar_drain(&B->full[s], pend_par[s]);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = mma_idesc();
            const uint32_t sfa = tmem + kSfaCol, sfb = tmem + kSfbCol;
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                if (!mbar_wait(&B->acc_empty, acc_phase ^ 1u, B, p.status)) break;
                tc_fence_after();
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&B->full[stage], phase, B, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sa + (size_t)stage * kStageABytes);
                    const uint32_t b0 = smem_u32(sb + (size_t)stage * kStageBBytes);
#pragma unroll
                    for (int ks = 0; ks < BK_BYTES / UMMA_K_BYTES; ++ks) {
                        mma_mxf4(tmem, smem_desc(a0 + ks * UMMA_K_BYTES),
                                 smem_desc(b0 + ks * UMMA_K_BYTES), idesc, sfa, sfb,
                                 (kb > 0 || ks > 0) ? 1u : 0u);
                    }
                    tc_commit(&B->empty[stage]);   // frees the stage when the MMAs finish
                    if (++stage == kStages) stage = 0, phase ^= 1u;
                }
                if (!ok) break;
                tc_commit(&B->acc_full);
                acc_phase ^= 1u;
            }
            // all issued MMAs complete before TMEM is released
            tc_commit(&B->mma_done);
            mbar_drain(&B->mma_done, 0);
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        uint32_t acc_phase = 0;
        const bool vec = (p.N % 8) == 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            int m_blk, n_blk;
            tile_coords(tile, num_m, m_blk, n_blk);
            if (!mbar_wait(&B->acc_full, acc_phase, B, p.status)) break;
            acc_phase ^= 1u;
            tc_fence_after();
            const int row = m_blk * BM + 32 * q + lane;
            const bool row_ok = row < p.M;
            const float s_row = row_ok ? p.sA[row] : 0.0f;
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + (uint32_t)(c * 32), v);
                if (c == BN / 32 - 1) {
                    // accumulator fully read: let the next tile's MMAs start
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&B->acc_empty);
                }
                const int col0 = n_blk * BN + c * 32;
                if (!row_ok || col0 >= p.N) continue;
                const bool full = vec && (col0 + 32 <= p.N);
                const int64_t off = (int64_t)row * p.N + col0;
                if (p.raw_acc) {
                    if (full) {
                        float4* d = reinterpret_cast<float4*>(p.raw_acc + off);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            d[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                               __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (col0 + j < p.N) p.raw_acc[off + j] = __uint_as_float(v[j]);
                    }
                }
                if (p.Y == nullptr) continue;
                float y[32];
                if (full) {
                    const float4* tw = reinterpret_cast<const float4*>(p.sW + col0);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 t = __ldg(tw + j);
                        y[4 * j + 0] = __fmul_rn(__fmul_rn(__uint_as_float(v[4 * j + 0]), s_row), t.x);
                        y[4 * j + 1] = __fmul_rn(__fmul_rn(__uint_as_float(v[4 * j + 1]), s_row), t.y);
                        y[4 * j + 2] = __fmul_rn(__fmul_rn(__uint_as_float(v[4 * j + 2]), s_row), t.z);
                        y[4 * j + 3] = __fmul_rn(__fmul_rn(__uint_as_float(v[4 * j + 3]), s_row), t.w);
                    }
                    if (p.C) {
                        const float4* cc = reinterpret_cast<const float4*>(p.C + off);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float4 t = __ldg(cc + j);
                            y[4 * j + 0] = __fadd_rn(y[4 * j + 0], t.x);
                            y[4 * j + 1] = __fadd_rn(y[4 * j + 1], t.y);
                            y[4 * j + 2] = __fadd_rn(y[4 * j + 2], t.z);
                            y[4 * j + 3] = __fadd_rn(y[4 * j + 3], t.w);
                        }
                    }
                    if (p.y_bf16) {
                        uint4* d = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.Y) + off);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint32_t w[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                __nv_bfloat162 h = __floats2bfloat162_rn(y[8 * j + 2 * i], y[8 * j + 2 * i + 1]);
                                w[i] = *reinterpret_cast<uint32_t*>(&h);
                            }
                            d[j] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    } else {
                        float4* d = reinterpret_cast<float4*>(static_cast<float*>(p.Y) + off);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            d[j] = make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (col0 + j >= p.N) continue;
                        float yy = __fmul_rn(__fmul_rn(__uint_as_float(v[j]), s_row), p.sW[col0 + j]);
                        if (p.C) yy = __fadd_rn(yy, p.C[off + j]);
                        if (p.y_bf16) static_cast<__nv_bfloat16*>(p.Y)[off + j] = __float2bfloat16_rn(yy);
                        else static_cast<float*>(p.Y)[off + j] = yy;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                                "r"(kTmemCols));
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2-D map over packed codes: rows x (K/2) bytes, box (128 bytes) x box_rows.
static bool make_code_map(CUtensorMap* map, const uint8_t* base, int64_t rows, int64_t kbytes,
                          int box_rows) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)kbytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)kbytes};
    cuuint32_t box[2] = {(cuuint32_t)BK_BYTES, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace gemm

cudaError_t gemm_setup() {
    return cudaFuncSetAttribute(gemm::fp4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)gemm::kSmemBytes);
}

// Returns cudaErrorInvalidValue when the tensor maps cannot be built.
cudaError_t launch_fp4_gemm(const uint8_t* codesA, const float* sA, const uint8_t* codesWT,
                            const float* sW, int64_t M, int64_t N, int64_t K, const float* C,
                            void* Y, qg_dtype y_dtype, float* raw_acc, uint32_t* status,
                            cudaStream_t s) {
    using namespace gemm;
    CUtensorMap ta, tb;
    if (!make_code_map(&ta, codesA, M, K / 2, BM)) return cudaErrorInvalidValue;
    if (!make_code_map(&tb, codesWT, N, K / 2, BN)) return cudaErrorInvalidValue;
    Params p;
    p.sA = sA;
    p.sW = sW;
    p.C = C;
    p.Y = Y;
    p.raw_acc = raw_acc;
    p.status = status;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.y_bf16 = (y_dtype == QG_BF16) ? 1 : 0;
    const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    const int grid = (int)std::min<int64_t>(tiles, num_sms());
    fp4_gemm_kernel<<<grid, kThreads, kSmemBytes, s>>>(ta, tb, p);
    count_launch(1);
    return cudaGetLastError();
}

}  // namespace qg
