// mma_peak.cu -- the E2M1 rate of the tensor cores alone: a measurement
// kernel for the roofline of the FP4 GEMM, not a step of the layer.
//
// Method: the FP4 GEMM paragraph of the QbitAI write-up of "Optimizing LLM
// Training Using FP4 Quantization" (news.movedaos.com/post/4103) names the
// matrix product as the part that FP4 speeds up; its ceiling on this GPU is
// the rate at which the tensor pipe retires E2M1 MMAs, measured here.
//
// Every CTA (one per SM: its shared-memory request is more than half of an
// SM's) keeps one FP4 tile of each operand in shared memory, and one thread
// issues the block-scaled E2M1 MMA (tcgen05.mma kind::mxf4, every scale a
// constant UE8M0 1.0 in TMEM) on them back to back into one TMEM accumulator,
// with the FP4 GEMM's instruction shape: 128 x 224 x 64 per CTA, or
// 256 x 224 x 64 per 2-SM pair (cta_group::2).  Nothing is read from or
// written to global memory except the status word, so the launch time is the
// tensor pipe's time for the MMAs.  The wait for the last MMA is bounded; a
// wait that runs out sets the timeout bit of the status word, and a second
// bounded wait lets MMAs still in flight finish before TMEM is released.
// Optionally (acc_out != NULL) CTA 0 copies its accumulator, 128 rows x 224
// columns, to global memory afterwards, so a test can check the MMAs against
// a CPU product of the same operand tiles.
#include "qg_internal.cuh"

namespace qg {
namespace peak {

constexpr int kThreads = 128;            // four warps, one per TMEM lane quarter
constexpr int kTmemCols = 512;
constexpr int kSfaCol = 448;             // constant A scales (32 columns)
constexpr int kSfbCol = 480;             // constant B scales (32 columns)
constexpr int kBN = 224;                 // the GEMM's widest tile
constexpr int kRowBytes = 128;           // 256 E2M1 values per operand row: four K = 64 MMAs
constexpr int kATileBytes = 128 * kRowBytes;
constexpr int kBTileBytes = kBN * kRowBytes;   // solo: all 224 rows; a pair uses half per CTA
constexpr int kOffBar = kATileBytes + kBTileBytes;
constexpr size_t kSmemBytes = 120 * 1024;     // > half of an SM's 228 KB: one CTA per SM
constexpr long long kWaitLimit = 4000000000LL;   // SM clocks (~2 s)
static_assert(kOffBar + 16 + 1024 <= (int)kSmemBytes, "tiles + barrier + alignment slack");

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
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

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// K-major operand rows, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

template <bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
fp4_mma_loop_kernel(long long iters, uint32_t* status, float* acc_out) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* sa = smem;
    uint8_t* sb = smem + kATileBytes;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + 8);
    const int warp = threadIdx.x >> 5;
    uint32_t rank = 0;
    if constexpr (PAIR) asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));

    // operands: arbitrary E2M1 codes (every nibble is a finite value)
    uint32_t* words = reinterpret_cast<uint32_t*>(smem);
    for (int i = threadIdx.x; i < kOffBar / 4; i += kThreads) {
        uint32_t h = (uint32_t)i * 2654435761u + blockIdx.x;
        h ^= h >> 15;
        words[i] = h * 2246822519u;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor pipe
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        if constexpr (PAIR) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(tmem_slot)),
                         "r"(kTmemCols));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(tmem_slot)),
                         "r"(kTmemCols));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;

    // constant block scales (UE8M0 2^0) in this warp's lane quarter
    {
        const uint32_t lanes = (uint32_t)(32 * warp) << 16;
        const uint32_t c = 0x7F7F7F7Fu;
#pragma unroll
        for (int col = 0; col < 2; ++col)
            asm volatile(
                "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,"
                "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(
                    tmem + lanes + (uint32_t)(col == 0 ? kSfaCol : kSfbCol)),
                "r"(c)
                : "memory");
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if constexpr (PAIR) cluster_sync();   // both CTAs' operands, barriers and scales are ready
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

    if (threadIdx.x == 0 && rank == 0) {
        constexpr uint32_t kM = PAIR ? 256u : 128u;
        // E2M1 x E2M1, UE8M0 scales, K-major operands, M x 224, dense K = 64
        const uint32_t idesc =
            (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) | (1u << 23) | ((kM >> 4) << 24);
        uint64_t ad[4], bd[4];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            ad[ks] = smem_desc(smem_u32(sa) + 32u * ks);
            bd[ks] = smem_desc(smem_u32(sb) + 32u * ks);
        }
        const uint32_t sfa = tmem + kSfaCol, sfb = tmem + kSfbCol;
        for (long long it = 0; it < iters; ++it) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint32_t acc = (it > 0 || ks > 0) ? 1u : 0u;
                if constexpr (PAIR)
                    asm volatile(
                        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                        "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, "
                        "[%5], [%6], p;\n\t}" ::"r"(tmem),
                        "l"(ad[ks]), "l"(bd[ks]), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
                else
                    asm volatile(
                        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, "
                        "[%5], [%6], p;\n\t}" ::"r"(tmem),
                        "l"(ad[ks]), "l"(bd[ks]), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
            }
        }
        // completion of every MMA above arrives on the barrier (a pair: on both CTAs')
        if constexpr (PAIR)
            asm volatile(
                "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
                " [%0], %1;" ::"r"(smem_u32(bar)),
                "h"((uint16_t)0x3)
                : "memory");
        else
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                             smem_u32(bar))
                         : "memory");
    }
    // every thread waits (bounded) for the MMAs to complete; after a timeout a
    // second bounded wait gives MMAs still in flight time to finish before
    // the accumulator is read or TMEM is released
    bool done = mbar_try_wait(bar, 0);
    if (!done) {
        const long long t0 = clock64();
        while (!(done = mbar_try_wait(bar, 0))) {
            if (clock64() - t0 > kWaitLimit) {
                if ((threadIdx.x & 31) == 0) flag_status(status, kStatusTimeout);
                break;
            }
        }
        if (!done) {
            const long long t1 = clock64();
            while (!(done = mbar_try_wait(bar, 0)) && clock64() - t1 < kWaitLimit) {
            }
        }
    }
    __syncwarp();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (acc_out != nullptr && blockIdx.x == 0 && __all_sync(0xFFFFFFFFu, done)) {
        // warp w holds accumulator rows 32 w .. 32 w + 31 (one per lane)
        const int row = 32 * warp + (threadIdx.x & 31);
        const uint32_t lanes = (uint32_t)(32 * warp) << 16;
        for (int c0 = 0; c0 < kBN; c0 += 32) {
            uint32_t v[32];
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,"
                "%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,"
                "%31}, [%32];"
                : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                  "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
                  "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]),
                  "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
                  "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),
                  "=r"(v[30]), "=r"(v[31])
                : "r"(tmem + lanes + (uint32_t)c0));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            float4* d = reinterpret_cast<float4*>(acc_out + (size_t)row * kBN + c0);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                d[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                   __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if constexpr (PAIR) cluster_sync();   // the peer's MMAs no longer use this CTA
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 0) {
        if constexpr (PAIR)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                         "r"(kTmemCols));
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                         "r"(kTmemCols));
    }
}

// The shared-memory size is set here, on use, rather than in the library's
// device setup, which the layer's calls share.
static cudaError_t set_smem_attr(bool pair) {
    return cudaFuncSetAttribute(pair ? (const void*)fp4_mma_loop_kernel<true>
                                     : (const void*)fp4_mma_loop_kernel<false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
}

}  // namespace peak

// One launch over the whole GPU: a CTA per SM (pair: as many 2-CTA clusters as
// can be resident at once).  *flops = 2 x 128 x 224 x 64 x 4 x iters per CTA.
// acc_out (nullable): CTA 0's accumulator, 128 x 224 fp32, row-major.
cudaError_t launch_fp4_mma_loop(int64_t iters, bool pair, double* flops, float* acc_out,
                                uint32_t* status, cudaStream_t s) {
    using namespace peak;
    cudaError_t e = set_smem_attr(pair);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pair ? 2 : 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int ctas = num_sms();
    if (pair) {
        cfg.gridDim = dim3(2);
        int clusters = 0;
        e = cudaOccupancyMaxActiveClusters(&clusters, fp4_mma_loop_kernel<true>, &cfg);
        if (e != cudaSuccess) return e;
        if (clusters < 1) return cudaErrorInvalidConfiguration;
        ctas = std::min(2 * clusters, ctas / 2 * 2);
    }
    cfg.gridDim = dim3((unsigned)ctas);
    e = pair ? cudaLaunchKernelEx(&cfg, fp4_mma_loop_kernel<true>, (long long)iters, status, acc_out)
             : cudaLaunchKernelEx(&cfg, fp4_mma_loop_kernel<false>, (long long)iters, status, acc_out);
    count_launch(1);
    if (flops) *flops = 2.0 * 128.0 * kBN * 64.0 * 4.0 * (double)iters * (double)ctas;
    return e;
}

}  // namespace qg
