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
// Two variants of one kernel template, persistent over output tiles:
//   PAIR = false  one CTA per SM computes 128 x BN tiles (tcgen05 cta_group::1)
//   PAIR = true   a cluster of two CTAs (two SMs) computes 256 x BN tiles with
//                 the 2-SM MMA (cta_group::2): each CTA loads its 128 rows of A
//                 and half of the BN rows of W^T, so operand traffic from L2
//                 per output element drops by about a third.  The leader CTA
//                 (rank 0) issues the MMAs; the TMA loads of both CTAs signal
//                 the leader's barriers; the leader's MMA commits signal both
//                 CTAs' barriers.  Loads use no multicast.
// Warp roles (64 + 32 * kEpiWarps threads per CTA, kEpiWarps = 4 by default):
//   warp 0     TMA producer: 128-byte-swizzled FP4 tiles (256 values deep)
//              into a kStages-deep shared-memory ring
//   warp 1     TMEM allocator; in the (leader) CTA one thread issues the MMAs,
//              K = 64 each, into one of two TMEM accumulators so the next
//              tile's MMAs run while the epilogue drains this one
//   warps 2..  epilogue, one (or, with 8 warps, two) per TMEM lane quarter of
//              32 rows, 32 columns at a time: tcgen05.ld, the C sub-tile
//              arrives by TMA in swizzled shared memory, Y = acc * s_i * t_j
//              + C goes back into the same buffer and leaves by a TMA store
//              (kEpiBufs buffers per warp, C requested kEpiBufs - 1 chunks
//              ahead, TMEM loads one chunk ahead, the next tile's scales
//              loaded while this tile drains).  A separate instantiation
//              (TMA_EPI = false) stores registers directly, for the raw-
//              accumulator output and row pitches that TMA cannot describe.
// TMEM: accumulators at columns [0, BN) and [BN, 2 BN), constant block
// scales (every byte 0x7F = 2^0) at [448, 512).
// MX = true (MXFP4 operands, solo CTAs, BN = 128): every stage also brings the
// stage's E8M0 block scales of both operands (two 512-byte atoms each, see
// qg_mx_quantize_rows) by a bulk copy; the MMA thread moves them into a TMEM
// slot of the stage with tcgen05.cp (32 rows x 16 bytes, repeated into the four
// lane quarters) and points each MMA at them.  The block-scaled MMA reads the
// scales of row r from lane r, column slot + r / 32, and the scale-factor id
// of the instruction descriptor picks the byte pair of its two 32-blocks.
// The epilogue then writes the accumulator as is (+ C).
// CORR = true (the layer's compensated GEMM): kCorrWarps more warps compute
// the compensation dA . W of each output tile on the CUDA cores while the
// tensor pipe runs the tile's MMAs.  A correction warp owns a contiguous block
// of the CTA's 128 rows, split into four quarter-warp row blocks; a quarter
// walks its rows' CSR entries as one stream, each of its lanes summing 32 of
// the tile's columns, with the W-row chunks in flight copied L2 -> shared
// memory by cp.async into a per-warp ring (corr_rows4s; bf16 W with N and
// its pitch multiples of 8), or, otherwise, a warp walks its rows with 8
// columns per lane and a register ring (corr_rows).  Each row is an fp32 FMA
// chain in CSR order.  Finished rows go to this CTA's slot of a small
// scratch ring in global memory (2 slots of 128 x BN fp32 per CTA, rewritten
// every other tile, so it stays in L2), and the epilogue TMA-loads them
// exactly as it loads a caller's C.  Two barrier pairs (corr_full /
// corr_empty) hand the slots between the two roles.  The dense M x N fp32
// correction never exists.
// Every mbarrier wait is bounded; a wait that gives up sets the timeout bit in
// the status word, raises a CTA-wide abort flag, waits (bounded) for copies
// and MMAs in flight, frees TMEM and returns.
#include <cuda.h>

#include "qg_internal.cuh"

namespace qg {
namespace gemm {

constexpr int BM = 128;             // rows of A per CTA
constexpr int BK_BYTES = 128;       // 256 E2M1 values per row per k-block
constexpr int UMMA_K_BYTES = 32;    // 64 E2M1 values per MMA
constexpr int kAccStages = 2;
#ifndef QG_GEMM_EPI_WARPS
#define QG_GEMM_EPI_WARPS 4
#endif
constexpr int kEpiWarps = QG_GEMM_EPI_WARPS;     // 4 or 8 (one or two per TMEM lane quarter)
constexpr int kEpiSplit = kEpiWarps / 4;         // chunk stride of one epilogue warp
static_assert(kEpiWarps == 4 || kEpiWarps == 8, "one or two epilogue warps per lane quarter");
constexpr int kCorrWarps = 6;                    // correction warps (CORR)
// Threads of a CTA: producer, MMA, epilogue warps (+ correction warps).  With
// the correction warps a CTA has 384 threads, which leaves 168 registers per
// thread: what the TMA epilogue needs.
template <bool CORR>
constexpr int threads_of() { return 64 + 32 * kEpiWarps + (CORR ? 32 * kCorrWarps : 0); }
constexpr int kThreads = threads_of<false>();
constexpr int kCorrMaxCtas = 160;                // scratch slots are sized for this many CTAs
constexpr int kCorrSlots = 2;
constexpr int kTmemCols = 512;
constexpr int kSfaCol = 448;
constexpr int kSfbCol = 480;
// Pipeline depths (overridable at build time for tuning sweeps).
#ifndef QG_GEMM_PAIR_STAGES
#define QG_GEMM_PAIR_STAGES 5
#endif
#ifndef QG_GEMM_SOLO_STAGES
#define QG_GEMM_SOLO_STAGES 3
#endif
#ifndef QG_GEMM_EPI_BUFS
#define QG_GEMM_EPI_BUFS 4
#endif
#ifndef QG_GEMM_PAIR_EPI_BUFS
#define QG_GEMM_PAIR_EPI_BUFS QG_GEMM_EPI_BUFS
#endif
// The pair GEMM without C (Y written, nothing read in the epilogue) takes a
// deeper operand ring and two sub-tile buffers per epilogue warp: with no C
// sub-tiles to bring ahead, the epilogue needs only double buffering, and the
// freed shared memory keeps more k-blocks in flight.  Used for BN = 192 tiles
// (measured 5 % faster on the 7B block's qkv and gate_up at M = 16384; the
// BN = 224 down projection ran 4 % slower with it, and with a C to read, fewer
// C loads in flight cost more).
#ifndef QG_GEMM_PAIR_DEEP_STAGES
#define QG_GEMM_PAIR_DEEP_STAGES 6
#endif
#ifndef QG_GEMM_FORCE_BN
#define QG_GEMM_FORCE_BN 0
#endif
#ifndef QG_GEMM_MX_STAGES
#define QG_GEMM_MX_STAGES 4
#endif
constexpr int kMxSfCol = 256;        // MX: per-stage scale slots, 16 columns each
constexpr int kMxAtom = 512;         // 32 rows x 16 bytes of E8M0 scales (128 rows x 4 blocks)
constexpr int kMxStageSf = 4 * kMxAtom;   // two atoms of A, two of W^T per 256-deep stage
constexpr int kEpiBuf = 32 * 32 * 4;   // one 32 x 32 fp32 sub-tile
constexpr int kEpiBufs = QG_GEMM_EPI_BUFS;   // sub-tile buffers per epilogue warp (>= 2)
constexpr long long kWaitLimit = 2000000000LL;  // SM clocks (~1-2 s)
constexpr int kStageABytes = BM * BK_BYTES;

#ifndef QG_CORR_D
#define QG_CORR_D 4              // W-row entries in flight per quarter-warp (bf16 W, fused path)
#endif
// Shared-memory ring of one correction warp: QG_CORR_D steps x 4 quarters x
// 448 bytes (a 224-column bf16 W row segment per quarter).
constexpr int kCorrRingBytes = QG_CORR_D * 4 * 448;

// Shared-memory plan.  With the fused correction (CORR) the operand ring is
// one stage shorter (pairs) or two (single CTAs) and the pair's epilogue has
// three sub-tile buffers per warp, which frees room for the correction
// warps' W-row rings.
template <int BN, bool PAIR, bool MX = false, bool CORR = false, bool DEEP = false>
struct Cfg {
    static_assert(BN % 32 == 0 && BN <= 224, "two accumulators + scales must fit in TMEM");
    static_assert(!MX || (!PAIR && BN == 128), "MX tiles: one CTA, 128 x 128");
    static_assert(!DEEP || (PAIR && !MX && !CORR), "the deep ring: pair GEMMs without C");
    static constexpr int kStages = MX ? QG_GEMM_MX_STAGES
                                      : CORR ? (PAIR ? QG_GEMM_PAIR_STAGES - 1 : QG_GEMM_SOLO_STAGES - 1)
                                             : DEEP ? QG_GEMM_PAIR_DEEP_STAGES
                                                    : (PAIR ? QG_GEMM_PAIR_STAGES : QG_GEMM_SOLO_STAGES);
    // sub-tile buffers per epilogue warp (C loads in flight: kEpiB - 1 per warp)
    static constexpr int kEpiB = DEEP ? 2 : (CORR && PAIR) ? 3 : PAIR ? QG_GEMM_PAIR_EPI_BUFS : kEpiBufs;
    static_assert(kEpiB >= 2 && kStages >= 2, "double buffering at least");
    static_assert(!MX || kMxSfCol + 16 * kStages <= kSfaCol, "MX scale slots below the constant scales");
    static constexpr int kBRows = PAIR ? BN / 2 : BN;   // rows of W^T loaded by one CTA
    static constexpr int kStageBBytes = kBRows * BK_BYTES;
    static constexpr int kStageSfBytes = MX ? kMxStageSf : 0;
    static constexpr uint32_t kTxBytes = (PAIR ? 2u : 1u) * (kStageABytes + kStageBBytes) + kStageSfBytes;
    static constexpr int kTileRows = PAIR ? 2 * BM : BM;
    static constexpr size_t kOffB = (size_t)kStages * kStageABytes;
    static constexpr size_t kOffSf = kOffB + (size_t)kStages * kStageBBytes;
    static constexpr size_t kOffEpi = kOffSf + (size_t)kStages * kStageSfBytes;
    static constexpr size_t kOffSw = kOffEpi + (size_t)kEpiWarps * kEpiB * kEpiBuf;
    static constexpr size_t kOffRing = kOffSw + (size_t)kEpiWarps * ((BN / 32 + kEpiSplit - 1) / kEpiSplit) * 32 * 4;
    static constexpr size_t kOffBar = kOffRing + (CORR ? (size_t)kCorrWarps * kCorrRingBytes : 0);
};

template <int S, int EB>
struct alignas(8) Barriers {
    uint64_t full[S];
    uint64_t empty[S];
    uint64_t acc_full[kAccStages];
    uint64_t acc_empty[kAccStages];
    uint64_t cbar[kEpiWarps][EB];
    uint64_t corr_full[kCorrSlots];    // a tile's correction rows are in its scratch slot
    uint64_t corr_empty[kCorrSlots];   // the epilogue has loaded them: the slot is free
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort;
};

template <int BN, bool PAIR, bool MX = false, bool CORR = false, bool DEEP = false>
constexpr size_t smem_bytes() {
    using CF = Cfg<BN, PAIR, MX, CORR, DEEP>;
    return 1024 + CF::kOffBar + sizeof(Barriers<CF::kStages, CF::kEpiB>);
}
static_assert(smem_bytes<224, true>() <= 232448 && smem_bytes<224, false>() <= 232448 &&
                  smem_bytes<192, true, false, false, true>() <= 232448 &&
                  smem_bytes<128, false, true>() <= 232448 &&
                  smem_bytes<224, true, false, true>() <= 232448 &&
                  smem_bytes<224, false, false, true>() <= 232448,
              "pipeline stages and epilogue buffers must fit in 227 KB of shared memory");

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
// Arrive on a barrier given by its shared::cluster address (maybe the peer's).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
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
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* abort,
                                          uint32_t* status) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*reinterpret_cast<volatile int*>(abort)) return false;
        if (clock64() - t0 > kWaitLimit) {
            *reinterpret_cast<volatile int*>(abort) = 1;
            flag_status(status, kStatusTimeout);
            return false;
        }
    }
}
// The same wait by a whole warp, with one verdict for all its lanes.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, int* abort,
                                               uint32_t* status) {
    const bool ok = mbar_wait(bar, parity, abort, status);
    return __all_sync(0xFFFFFFFFu, ok);
}
// Bounded wait used during teardown (ignores the abort flag).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > kWaitLimit) return;
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}
// shared::cluster address of the same shared-memory object in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_rank(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint64_t* bar, void* dst,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// Load into this CTA's shared memory, completing on the leader CTA's barrier.
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap* map, uint32_t bar_cluster,
                                                 void* dst, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
        : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(smem_u32(src))
                 : "memory");
}
// The same box added into global memory: the memory system reads the
// destination, adds the shared-memory tile element by element and writes it
// back (fp32, round to nearest).
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int x,
                                                  int y) {
    asm volatile(
        "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(x), "r"(y), "r"(smem_u32(src))
        : "memory");
}
// Plain bulk copy global -> this CTA's shared memory (16-byte aligned, size a
// multiple of 16), completing on a barrier of this CTA.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// One scale atom (32 rows x 16 bytes, no swizzle, 8-row groups 128 bytes
// apart) from shared memory into TMEM columns [taddr, taddr + 4) of all four
// lane quarters.
__device__ __forceinline__ void tc_cp_scales(uint32_t taddr, uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)(2048 >> 4) << 16;   // leading byte offset (one 16-byte column: unused)
    d |= (uint64_t)(128 >> 4) << 32;    // stride byte offset: next 8-row group
    d |= (uint64_t)1 << 46;             // descriptor version, no swizzle
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Commit this thread's outstanding MMAs to a barrier of this CTA (PAIR: the
// barriers at the same offset in both CTAs of the pair).
template <bool PAIR>
__device__ __forceinline__ void tc_commit_all(uint64_t* bar) {
    if constexpr (PAIR) {
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
            " [%0], %1;" ::"r"(smem_u32(bar)),
            "h"((uint16_t)0x3)
            : "memory");
    } else {
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(bar))
                     : "memory");
    }
}
template <bool PAIR>
__device__ __forceinline__ void tc_commit_local(uint64_t* bar) {
    if constexpr (PAIR)
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(bar))
                     : "memory");
    else
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(bar))
                     : "memory");
}

template <bool PAIR>
__device__ __forceinline__ void tmem_alloc(uint32_t* dst) {
    if constexpr (PAIR) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(dst)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    } else {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(dst)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
}
template <bool PAIR>
__device__ __forceinline__ void tmem_free(uint32_t taddr) {
    if constexpr (PAIR)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr),
                     "r"(kTmemCols));
    else
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr),
                     "r"(kTmemCols));
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
// both operands K-major, M = 128 (256 for the pair), N = BN, dense K = 64.
template <int BN, bool PAIR>
__device__ __forceinline__ uint32_t mma_idesc() {
    constexpr uint32_t kM = PAIR ? 256u : 128u;
    return (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | (1u << 23) | ((kM >> 4) << 24);
}

template <bool PAIR>
__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                         uint32_t accumulate) {
    if constexpr (PAIR)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;"
            "\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb));
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;"
            "\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb));
}

// Start a load of 32 accumulator columns (this warp's 32 lanes) into v; the
// registers are valid only after tmem_ld_wait(v).
__device__ __forceinline__ void tmem_ld32_issue(uint32_t taddr, uint32_t (&v)[32]) {
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
}
// Wait for the loads issued so far; v is named so that no use of it can be
// scheduled before the wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&v)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                   "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                   "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]), "+r"(v[16]), "+r"(v[17]),
                   "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]), "+r"(v[22]), "+r"(v[23]),
                   "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]), "+r"(v[29]),
                   "+r"(v[30]), "+r"(v[31])
                 :
                 : "memory");
}
__device__ __forceinline__ void tmem_ld_wait_all() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
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

// Byte offset of 16-byte chunk `c` of row `r` in a 32-row TMA box with the
// 128-byte (fp32 rows) or 64-byte (bf16 rows) swizzle.
__device__ __forceinline__ uint32_t swz128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }
__device__ __forceinline__ uint32_t swz64(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }

// ------------------------------------------------------------------ correction
// acc (an fp32 pair) += v * (lo(w), hi(w)) for a bf16 pair w: one rounding per
// product-sum, as fmaf.
__device__ __forceinline__ void fma2_bf16(uint64_t& acc, uint64_t vv, uint32_t w) {
    asm("{\n\t.reg .b32 lo, hi;\n\t.reg .b64 x;\n\t"
        "shl.b32 lo, %2, 16;\n\tand.b32 hi, %2, 0xFFFF0000;\n\t"
        "mov.b64 x, {lo, hi};\n\tfma.rn.f32x2 %0, x, %1, %0;\n\t}"
        : "+l"(acc)
        : "l"(vv), "r"(w));
}
// acc += v * (a, b) for an fp32 pair (a in the low word).
__device__ __forceinline__ void fma2_f32(uint64_t& acc, uint64_t vv, uint32_t a, uint32_t b) {
    asm("{\n\t.reg .b64 x;\n\tmov.b64 x, {%2, %3};\n\tfma.rn.f32x2 %0, x, %1, %0;\n\t}"
        : "+l"(acc)
        : "l"(vv), "r"(a), "r"(b));
}

#ifndef QG_CORR_LDG
#define QG_CORR_LDG 0
#endif
// A 16-byte W segment load (read-only data)
__device__ __forceinline__ uint4 ld_w16(const void* p) {
#if QG_CORR_LDG == 1
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
#elif QG_CORR_LDG == 2
    return __ldcg(reinterpret_cast<const uint4*>(p));
#else
    return __ldg(reinterpret_cast<const uint4*>(p));
#endif
}

// The compensation rows r_begin .. r_end - 1 (at most 31 rows) of dA . W,
// 8 columns per lane starting at c0: for each row, the fp32 FMA chain over the
// row's CSR entries in order, value (fp32 of the stored double) times the W
// row segment.  The warp's entries form one contiguous CSR range, consumed as
// a stream in groups of G entries; NG groups of W-row segments (16 bytes per
// lane per entry) are in flight.  A group's G loads are issued together and
// its G entries consumed together, so a group needs one load scoreboard and
// the wait for the oldest group never waits for a newer one.  Ring positions
// are compile-time indices (the loop is unrolled by NG groups).  Lane l holds
// entry values and the columns of the entries NG * G ahead, batch by batch
// of 32.  Row r's 8 sums go to dst + (r - r_begin) * dst_ld (lanes with
// lane_on).  fast: every W row segment the warp reads is 16-byte aligned and
// inside W for the lanes that are on (the caller checks N and ldw); lanes
// that are off then read the warp's first segment (column c_safe) instead,
// so the loads are not divergent.  Otherwise element loads, zero past N.
template <bool WBF16, int NG, int G>
__device__ __forceinline__ void corr_rows(const int32_t* __restrict__ row_ptr,
                                          const int32_t* __restrict__ col,
                                          const double* __restrict__ val,
                                          const void* __restrict__ W, int64_t ldw, int r_begin,
                                          int r_end, int N, int c0, int c_safe, bool lane_on,
                                          bool fast, float* __restrict__ dst, int dst_ld) {
    constexpr int D = NG * G;                   // entries in flight
    static_assert(32 % D == 0, "entry batches of 32 hold whole ring turns");
    constexpr int SEG = WBF16 ? 1 : 2;          // 16-byte words per lane per W row segment
    const int lane = threadIdx.x & 31;
    const int nrows = r_end - r_begin;
    const int rp = (lane <= nrows) ? __ldg(row_ptr + r_begin + lane) : 0;
    const int P0 = __shfl_sync(0xFFFFFFFFu, rp, 0);
    const int n = __shfl_sync(0xFFFFFFFFu, rp, nrows) - P0;
    int kc = (lane < n) ? __ldg(col + P0 + lane) : 0;
    float vc = (lane < n) ? (float)__ldg(val + P0 + lane) : 0.0f;
    int ks;
    {
        const int kn = (32 + lane < n) ? __ldg(col + P0 + 32 + lane) : 0;
        const int a = __shfl_sync(0xFFFFFFFFu, kc, (lane + D) & 31);
        const int b = __shfl_sync(0xFFFFFFFFu, kn, (lane + D) & 31);
        ks = (lane + D < 32) ? a : b;
    }
    const int cl = lane_on ? c0 : c_safe;       // this lane's load column
    auto fetch = [&](uint4 (&d)[SEG], int k) {
        if constexpr (WBF16) {
            const uint16_t* src = static_cast<const uint16_t*>(W) + (int64_t)k * ldw + cl;
            if (fast) {
                d[0] = ld_w16(src);
            } else {
                uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (lane_on && c0 + e < N) w[e >> 1] |= (uint32_t)__ldg(src + e) << (16 * (e & 1));
                d[0] = make_uint4(w[0], w[1], w[2], w[3]);
            }
        } else {
            const float* src = static_cast<const float*>(W) + (int64_t)k * ldw + cl;
            if (fast) {
                d[0] = ld_w16(src);
                d[1] = ld_w16(src + 4);
            } else {
                uint32_t w[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    w[e] = (lane_on && c0 + e < N) ? __float_as_uint(__ldg(src + e)) : 0u;
                d[0] = make_uint4(w[0], w[1], w[2], w[3]);
                d[1] = make_uint4(w[4], w[5], w[6], w[7]);
            }
        }
    };
    uint4 buf[NG][G][SEG];
#pragma unroll
    for (int g = 0; g < NG; ++g)
#pragma unroll
        for (int i = 0; i < G; ++i)
            if (g * G + i < n) fetch(buf[g][i], __shfl_sync(0xFFFFFFFFu, kc, g * G + i));
    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
    int row = r_begin;
    int rend = __shfl_sync(0xFFFFFFFFu, rp, 1) - P0;   // entries of rows <= row end here
    auto store_row = [&](int r) {
        if (lane_on) {
            ulonglong2* d = reinterpret_cast<ulonglong2*>(dst + (int64_t)(r - r_begin) * dst_ld);
            d[0] = make_ulonglong2(acc[0], acc[1]);
            d[1] = make_ulonglong2(acc[2], acc[3]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] = 0ull;
    };
    for (int q = 0; q < n; q += D) {
#pragma unroll
        for (int g = 0; g < NG; ++g) {
#pragma unroll
            for (int i = 0; i < G; ++i) {           // consume group g
                const int j = q + g * G + i;         // entry index within the warp's range
                if (j < n) {
                    while (j >= rend) {              // rows that end before entry j
                        store_row(row);
                        ++row;
                        rend = __shfl_sync(0xFFFFFFFFu, rp, row - r_begin + 1) - P0;
                    }
                    const float v = __shfl_sync(0xFFFFFFFFu, vc, (q & 31) + g * G + i);
                    uint64_t vv;
                    asm("mov.b64 %0, {%1, %1};" : "=l"(vv) : "f"(v));
                    if constexpr (WBF16) {
                        fma2_bf16(acc[0], vv, buf[g][i][0].x);
                        fma2_bf16(acc[1], vv, buf[g][i][0].y);
                        fma2_bf16(acc[2], vv, buf[g][i][0].z);
                        fma2_bf16(acc[3], vv, buf[g][i][0].w);
                    } else {
                        fma2_f32(acc[0], vv, buf[g][i][0].x, buf[g][i][0].y);
                        fma2_f32(acc[1], vv, buf[g][i][0].z, buf[g][i][0].w);
                        fma2_f32(acc[2], vv, buf[g][i][SEG - 1].x, buf[g][i][SEG - 1].y);
                        fma2_f32(acc[3], vv, buf[g][i][SEG - 1].z, buf[g][i][SEG - 1].w);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < G; ++i) {           // refill group g, entries D ahead
                const int j = q + g * G + i;
                const int kf = __shfl_sync(0xFFFFFFFFu, ks, (q & 31) + g * G + i);
                if (j + D < n) fetch(buf[g][i], kf);
            }
        }
        if ((q & 31) == 32 - D) {                // batch done: load the next one
            const int Bn = q + D;
            kc = (Bn + lane < n) ? __ldg(col + P0 + Bn + lane) : 0;
            vc = (Bn + lane < n) ? (float)__ldg(val + P0 + Bn + lane) : 0.0f;
            const int kn = (Bn + 32 + lane < n) ? __ldg(col + P0 + Bn + 32 + lane) : 0;
            const int a = __shfl_sync(0xFFFFFFFFu, kc, (lane + D) & 31);
            const int b = __shfl_sync(0xFFFFFFFFu, kn, (lane + D) & 31);
            ks = (lane + D < 32) ? a : b;
        }
    }
    while (row < r_end) {                        // the last rows (and empty ones)
        store_row(row);
        ++row;
    }
}

// The compensation rows of a warp for a tile of 224 (or 192) bf16 columns,
// four row blocks at a time.  Quarter-warp qd (lanes 8 qd .. 8 qd + 7) walks
// the contiguous CSR range of its rows [rq0, rq1) (at most 7 rows); lane
// lq < 7 of a quarter owns the four 8-column groups lq, lq + 7, lq + 14,
// lq + 21 of the tile, so each of a quarter's four 16-byte copies covers 112
// contiguous bytes of the W row and a lane sums 32 columns per entry.  The W
// segments in flight live in shared memory, not registers: every lane copies
// its chunks of an entry with cp.async (L2 -> shared memory), one commit
// group per ring step, D steps ahead, and waits with cp.async.wait_group for
// the oldest step before reading it back; each lane reads only what it
// copied, so no other synchronisation is needed.  Entry values and columns
// are held by the quarter's lanes, batch by batch of 8, and broadcast with
// 8-lane shuffles.  Each row is an fp32 FMA chain over its entries in CSR
// order; its sums go to dst + (r - r_base) * dst_ld at the lane's columns.
// ring: this warp's D x 4 x 448 bytes of shared memory.  The loop runs until
// the warp's longest quarter is done; the other quarters idle meanwhile.
template <int D>
__device__ __forceinline__ void corr_rows4s(const int32_t* __restrict__ row_ptr,
                                            const int32_t* __restrict__ col,
                                            const double* __restrict__ val,
                                            const uint16_t* __restrict__ W, int64_t ldw, int rq0,
                                            int rq1, int n0, int N, int r_base,
                                            float* __restrict__ dst, int dst_ld, int BNr,
                                            uint8_t* ring) {
    static_assert(8 % D == 0, "entry batches of 8 hold whole ring turns");
    const int lane = threadIdx.x & 31;
    const int lq = lane & 7, qd = lane >> 3;
    const unsigned FULL = 0xFFFFFFFFu;
    const int nrows = rq1 - rq0;
    const int rp = (lq <= nrows) ? __ldg(row_ptr + rq0 + lq) : 0;
    const int P0 = __shfl_sync(FULL, rp, 0, 8);
    const int n = __shfl_sync(FULL, rp, nrows, 8) - P0;
    int nmax = n;
#pragma unroll
    for (int d = 8; d < 32; d <<= 1) nmax = max(nmax, __shfl_xor_sync(FULL, nmax, d));
    bool on[4];
    int cg[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        cg[h] = 8 * (lq + 7 * h);
        on[h] = lq < 7 && cg[h] < BNr && n0 + cg[h] < N;
        if (!on[h]) cg[h] = 0;
    }
    int kc = (lq < n) ? __ldg(col + P0 + lq) : 0;
    float vc = (lq < n) ? (float)__ldg(val + P0 + lq) : 0.0f;
    int ks;
    {
        const int kn = (8 + lq < n) ? __ldg(col + P0 + 8 + lq) : 0;
        const int a = __shfl_sync(FULL, kc, (lq + D) & 7, 8);
        const int b = __shfl_sync(FULL, kn, (lq + D) & 7, 8);
        ks = (lq + D < 8) ? a : b;
    }
    const uint16_t* wl = W + n0;
    // slot u of this lane: 4 chunks, lane-private, conflict-free per quarter
    // (lane 7 of a quarter owns no columns: it mirrors lane 6's slots, which
    // keeps its reads inside the quarter's region; it never copies or stores)
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(ring) + (uint32_t)(qd * 448 + min(lq, 6) * 16);
    auto slot_addr = [&](int u, int h) { return sbase + (uint32_t)(u * 4 * 448 + h * 112); };
    auto fetch = [&](int u, int k, bool valid) {
        const uint16_t* src = wl + (int64_t)k * ldw;
#pragma unroll
        for (int h = 0; h < 4; ++h)
            if (valid && on[h])
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(slot_addr(u, h)),
                             "l"(src + cg[h])
                             : "memory");
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
#pragma unroll
    for (int u = 0; u < D; ++u) fetch(u, __shfl_sync(FULL, kc, u, 8), u < n);
    uint64_t acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0ull;
    int row = rq0;
    int rend = __shfl_sync(FULL, rp, 1, 8) - P0;
    auto store_row = [&](int r) {
        float* d = dst + (int64_t)(r - r_base) * dst_ld;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            if (on[h]) {
                ulonglong2* p = reinterpret_cast<ulonglong2*>(d + cg[h]);
                p[0] = make_ulonglong2(acc[4 * h + 0], acc[4 * h + 1]);
                p[1] = make_ulonglong2(acc[4 * h + 2], acc[4 * h + 3]);
            }
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = 0ull;
    };
    for (int q = 0; q < nmax; q += D) {
#pragma unroll
        for (int u = 0; u < D; ++u) {
            const int j = q + u;
            const int t = (q & 7) + u;
            const float v = __shfl_sync(FULL, vc, t, 8);
            const int kf = __shfl_sync(FULL, ks, t, 8);
            // the oldest of the D groups in flight is slot u's
            asm volatile("cp.async.wait_group %0;" ::"n"(D - 1) : "memory");
            if (j < n) {
                while (j >= rend) {
                    store_row(row);
                    ++row;
                    rend = __shfl_sync(__activemask(), rp, row - rq0 + 1, 8) - P0;
                }
                uint64_t vv;
                asm("mov.b64 %0, {%1, %1};" : "=l"(vv) : "f"(v));
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    uint4 w;
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                                 : "r"(slot_addr(u, h)));
                    fma2_bf16(acc[4 * h + 0], vv, w.x);
                    fma2_bf16(acc[4 * h + 1], vv, w.y);
                    fma2_bf16(acc[4 * h + 2], vv, w.z);
                    fma2_bf16(acc[4 * h + 3], vv, w.w);
                }
            }
            fetch(u, kf, j + D < n);             // refill slot u (an empty group if none)
        }
        if ((q & 7) == 8 - D) {
            const int Bn = q + D;
            kc = (Bn + lq < n) ? __ldg(col + P0 + Bn + lq) : 0;
            vc = (Bn + lq < n) ? (float)__ldg(val + P0 + Bn + lq) : 0.0f;
            const int kn = (Bn + 8 + lq < n) ? __ldg(col + P0 + Bn + 8 + lq) : 0;
            const int a = __shfl_sync(FULL, kc, (lq + D) & 7, 8);
            const int b = __shfl_sync(FULL, kn, (lq + D) & 7, 8);
            ks = (lq + D < 8) ? a : b;
        }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    while (row < rq1) {
        store_row(row);
        ++row;
    }
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
    int tma_epi;         // Y (and C) through TMA
    int y_add;           // TMA epilogue, fp32 Y, no C: add the product into Y instead of storing it
    int unit_scales;     // MX: no row / column scales in the epilogue
    const uint8_t* sfA;  // MX: E8M0 scale atoms of A, [row block][k group]
    const uint8_t* sfB;  // MX: the same for W^T
    int sf_groups;       // MX: 128-deep k groups per row block (even)
    // Tile order of the persistent grid: m fastest (consecutive tiles share a
    // column block: W's codes for it stay in L2 while A's codes stream) or n
    // fastest (consecutive tiles share a row block: A's codes stay in L2).
    // The host picks the order that keeps the larger code matrix streaming
    // once and the smaller one resident.
    int n_fastest;
    // CORR: dA in CSR, the unquantized W (K x N, row pitch ldw elements, bf16
    // or fp32) and the scratch slots (kCorrSlots x 128 x BN fp32 per CTA)
    const int32_t* row_ptr;
    const int32_t* col;
    const double* val;
    const void* Wc;
    int64_t ldw;
    int w_bf16;
    float* corr;
};

// Direct epilogue of one 32-column chunk: registers -> global (row per lane).
// crow: this row's correction at column col0 (a caller's C or a scratch slot),
// or null; read with coherent loads, since a slot is rewritten in the kernel.
__device__ __forceinline__ void epi_direct(const Params& p, const uint32_t (&v)[32], int row,
                                           int col0, float s_row, const float* crow) {
    const bool full = (p.N % 8) == 0 && (col0 + 32 <= p.N);
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
    if (p.Y == nullptr) return;
    if (full && !p.y_bf16) {
        // 16-byte loads of C and the column scales, 16-byte stores of Y
        float* yrow = static_cast<float*>(p.Y) + off;
        const float4* tw = reinterpret_cast<const float4*>(p.sW + col0);
        const float4* c4 = reinterpret_cast<const float4*>(crow);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 t = p.unit_scales ? make_float4(1.0f, 1.0f, 1.0f, 1.0f) : __ldg(tw + j);
            float4 y = make_float4(__fmul_rn(__fmul_rn(__uint_as_float(v[4 * j]), s_row), t.x),
                                   __fmul_rn(__fmul_rn(__uint_as_float(v[4 * j + 1]), s_row), t.y),
                                   __fmul_rn(__fmul_rn(__uint_as_float(v[4 * j + 2]), s_row), t.z),
                                   __fmul_rn(__fmul_rn(__uint_as_float(v[4 * j + 3]), s_row), t.w));
            if (c4) {
                const float4 c = __ldcg(c4 + j);
                y.x = __fadd_rn(y.x, c.x);
                y.y = __fadd_rn(y.y, c.y);
                y.z = __fadd_rn(y.z, c.z);
                y.w = __fadd_rn(y.w, c.w);
            }
            reinterpret_cast<float4*>(yrow)[j] = y;
        }
        return;
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        if (col0 + j >= p.N) continue;
        const float tj = p.unit_scales ? 1.0f : __ldg(p.sW + col0 + j);
        float yy = __fmul_rn(__fmul_rn(__uint_as_float(v[j]), s_row), tj);
        if (crow) yy = __fadd_rn(yy, __ldcg(crow + j));
        if (p.y_bf16) static_cast<__nv_bfloat16*>(p.Y)[off + j] = __float2bfloat16_rn(yy);
        else static_cast<float*>(p.Y)[off + j] = yy;
    }
}

// TMA_EPI: Y (and C) go through the swizzled sub-tile buffers and TMA; the
// other instantiation stores registers directly (raw accumulator output, or
// row pitches TMA cannot describe), so neither path's registers burden the other.
template <int BN, bool PAIR, bool TMA_EPI, bool MX = false, bool CORR = false, bool DEEP = false>
__global__ void __launch_bounds__(threads_of<CORR>(), 1)
fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                const __grid_constant__ CUtensorMap tmap_b,
                const __grid_constant__ CUtensorMap tmap_y,
                const __grid_constant__ CUtensorMap tmap_c, const Params p) {
    using CF = Cfg<BN, PAIR, MX, CORR, DEEP>;
    constexpr int S = CF::kStages;
    constexpr int EB = CF::kEpiB;
    static_assert(!(CORR && MX), "the compensated GEMM uses per-row / per-column scales");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* sa = smem;
    uint8_t* sb = smem + CF::kOffB;
    uint8_t* ssf = smem + CF::kOffSf;
    uint8_t* sepi = smem + CF::kOffEpi;
    Barriers<S, EB>* B = reinterpret_cast<Barriers<S, EB>*>(smem + CF::kOffBar);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = PAIR ? cluster_rank() : 0u;
    const bool leader = rank == 0;
    const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;    // CTA or CTA pair
    const int n_units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    const int num_m = (p.M + CF::kTileRows - 1) / CF::kTileRows;
    const int num_n = (p.N + BN - 1) / BN;
    const int num_tiles = num_m * num_n;
    const int num_kb = (p.K / 2 + BK_BYTES - 1) / BK_BYTES;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&B->full[s], 1);
            mbar_init(&B->empty[s], 1);
        }
        for (int s = 0; s < kAccStages; ++s) {
            mbar_init(&B->acc_full[s], 1);
            mbar_init(&B->acc_empty[s], (PAIR ? 2 : 1) * kEpiWarps);
        }
        for (int w = 0; w < kEpiWarps; ++w)
            for (int b = 0; b < EB; ++b) mbar_init(&B->cbar[w][b], 1);
        for (int s = 0; s < kCorrSlots; ++s) {
            mbar_init(&B->corr_full[s], kCorrWarps);
            mbar_init(&B->corr_empty[s], kEpiWarps);
        }
        mbar_init(&B->mma_done, 1);
        B->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_b)) : "memory");
    }
    if (warp == 1) tmem_alloc<PAIR>(&B->tmem_base);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = B->tmem_base;

    if (warp >= 2 && warp < 2 + kEpiWarps) {
        // constant block scales: every byte 0x7F (UE8M0 2^0) in the scale region
        const uint32_t q = (uint32_t)(warp & 3);
        tmem_st32_const(tmem + ((32u * q) << 16) + kSfaCol, 0x7F7F7F7Fu);
        tmem_st32_const(tmem + ((32u * q) << 16) + kSfbCol, 0x7F7F7F7Fu);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();   // both CTAs' barriers and scales are ready
    tc_fence_after();

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            uint32_t pend = 0, pend_par = 0;     // per stage: load in flight / its parity
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = unit; ok && tile < num_tiles; tile += n_units) {
                const int m_blk = p.n_fastest ? tile / num_n : tile % num_m;
                const int n_blk = p.n_fastest ? tile % num_n : tile / num_m;
                const int a_row = m_blk * CF::kTileRows + (int)rank * BM;
                const int b_row = n_blk * BN + (int)rank * CF::kBRows;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&B->empty[stage], phase ^ 1u, &B->abort, p.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t* da = sa + (size_t)stage * kStageABytes;
                    uint8_t* db = sb + (size_t)stage * CF::kStageBBytes;
                    if constexpr (PAIR) {
                        if (leader) mbar_expect_tx(&B->full[stage], CF::kTxBytes);
                        const uint32_t lb = map_to_rank(&B->full[stage], 0);
                        tma_load_2d_pair(&tmap_a, lb, da, kb * BK_BYTES, a_row);
                        tma_load_2d_pair(&tmap_b, lb, db, kb * BK_BYTES, b_row);
                    } else {
                        mbar_expect_tx(&B->full[stage], CF::kTxBytes);
                        tma_load_2d(&tmap_a, &B->full[stage], da, kb * BK_BYTES, a_row);
                        tma_load_2d(&tmap_b, &B->full[stage], db, kb * BK_BYTES, b_row);
                        if constexpr (MX) {
                            // the stage's two k groups are adjacent atoms
                            uint8_t* ds = ssf + (size_t)stage * kMxStageSf;
                            const size_t ka = (size_t)2 * kb * kMxAtom;
                            bulk_load(ds, p.sfA + (size_t)m_blk * p.sf_groups * kMxAtom + ka,
                                      2 * kMxAtom, &B->full[stage]);
                            bulk_load(ds + 2 * kMxAtom, p.sfB + (size_t)n_blk * p.sf_groups * kMxAtom + ka,
                                      2 * kMxAtom, &B->full[stage]);
                        }
                    }
                    pend |= 1u << stage;
                    pend_par = (pend_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) stage = 0, phase ^= 1u;
                }
            }
            if (!ok) {
                // on abort, copies still in flight land before the CTA exits
                if (!PAIR || leader) {
                    for (int s = 0; s < S; ++s)
                        if ((pend >> s) & 1u) mbar_drain(&B->full[s], (pend_par >> s) & 1u);
                } else {
                    // the peer's loads complete on the leader's barriers: give
                    // them a fixed grace period instead
                    const long long t0 = clock64();
                    while (clock64() - t0 < 2000000LL) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0 && leader) {
            const uint32_t idesc = mma_idesc<BN, PAIR>();
            const uint32_t sfa = tmem + kSfaCol, sfb = tmem + kSfbCol;
            int stage = 0, as = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            // MX: a stage's four scale atoms go into its TMEM slot with
            // tcgen05.cp right before its MMAs (issuing them one stage early,
            // when the next stage's data had landed, measured 13 % slower)
            auto copy_scales = [&](int st) {
                const uint32_t slot = tmem + (uint32_t)(kMxSfCol + 16 * st);
                const uint32_t s0 = smem_u32(ssf + (size_t)st * kMxStageSf);
#pragma unroll
                for (int g = 0; g < 4; ++g) tc_cp_scales(slot + 4u * g, s0 + kMxAtom * g);
            };
            for (int tile = unit; ok && tile < num_tiles; tile += n_units) {
                if (!mbar_wait(&B->acc_empty[as], acc_phase ^ 1u, &B->abort, p.status)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(as * BN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&B->full[stage], phase, &B->abort, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sa + (size_t)stage * kStageABytes);
                    const uint32_t b0 = smem_u32(sb + (size_t)stage * CF::kStageBBytes);
                    if constexpr (MX) {
                        // this stage's scales into its TMEM slot: A atoms at +0, +4,
                        // W^T atoms at +8, +12; the copies run before the MMAs
                        const uint32_t slot = tmem + (uint32_t)(kMxSfCol + 16 * stage);
                        copy_scales(stage);
#pragma unroll
                        for (int ks = 0; ks < BK_BYTES / UMMA_K_BYTES; ++ks) {
                            // MMA ks covers 32-blocks 2 ks, 2 ks + 1: atom ks / 2, bytes
                            // 2 (ks % 2) and up (scale-factor ids, bits 29-30 and 4-5)
                            const uint32_t id = 2u * (uint32_t)(ks & 1);
                            mma_mxf4<PAIR>(d_tmem, smem_desc(a0 + ks * UMMA_K_BYTES),
                                           smem_desc(b0 + ks * UMMA_K_BYTES),
                                           idesc | (id << 29) | (id << 4),
                                           slot + 4u * (uint32_t)(ks >> 1),
                                           slot + 8u + 4u * (uint32_t)(ks >> 1),
                                           (kb > 0 || ks > 0) ? 1u : 0u);
                        }
                    } else {
#pragma unroll
                        for (int ks = 0; ks < BK_BYTES / UMMA_K_BYTES; ++ks) {
                            mma_mxf4<PAIR>(d_tmem, smem_desc(a0 + ks * UMMA_K_BYTES),
                                           smem_desc(b0 + ks * UMMA_K_BYTES), idesc, sfa, sfb,
                                           (kb > 0 || ks > 0) ? 1u : 0u);
                        }
                    }
                    tc_commit_all<PAIR>(&B->empty[stage]);   // frees the stage (both CTAs)
                    if (++stage == S) stage = 0, phase ^= 1u;
                }
                if (!ok) break;
                tc_commit_all<PAIR>(&B->acc_full[as]);
                if (++as == kAccStages) as = 0, acc_phase ^= 1u;
            }
            // all issued MMAs complete before TMEM is released
            tc_commit_local<PAIR>(&B->mma_done);
            mbar_drain(&B->mma_done, 0);
        }
    } else if (warp < 2 + kEpiWarps) {
        // ---------------------------------------------------------- epilogue
        // Two warps per TMEM lane quarter when kEpiSplit == 2: warp ew takes
        // the chunks c with c % kEpiSplit == ew / 4.  Each warp walks its
        // chunks of all its tiles as one stream: chunk g uses sub-tile buffer
        // g % EB; with a correction C, the C sub-tile of chunk
        // g + EB - 1 is requested once chunk g is stored.  The next
        // tile's row and column scales are loaded while this tile is drained.
        constexpr int NC = BN / 32;
        constexpr int SWR = (NC + kEpiSplit - 1) / kEpiSplit;   // this warp's chunks per tile, at most
        const int ew = warp - 2;               // epilogue warp index (buffers)
        const int q = warp & 3;                // TMEM lane quarter
        const int par = ew / 4;                // chunk residue class of this warp
        const int my_nc = (NC - par + kEpiSplit - 1) / kEpiSplit;   // its chunks per tile
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        uint8_t* bufs = sepi + (size_t)ew * EB * kEpiBuf;
        float* sw = reinterpret_cast<float*>(smem + CF::kOffSw) + ew * SWR * 32;
        const bool use_c = TMA_EPI && (CORR || p.C != nullptr);
        const int my_tiles = unit < num_tiles ? (num_tiles - unit + n_units - 1) / n_units : 0;
        const int total = my_tiles * my_nc;
        uint32_t cphase = 0;                   // bit b: parity of the next wait on cbar[ew][b]
        uint32_t cpend = 0;                    // bit b: a C load into buffer b not yet waited for
        // C sub-tile of chunk g: from the caller's C, or (CORR) from this CTA's
        // scratch slot of the chunk's tile, once the correction warps have
        // filled it.  False when a wait gave up.
        auto c_load = [&](int g) -> bool {
            const int ti = g / my_nc, c = par + kEpiSplit * (g - ti * my_nc);
            const int tile = unit + ti * n_units;
            const int mb = p.n_fastest ? tile / num_n : tile % num_m;
            const int nbk = p.n_fastest ? tile % num_n : tile / num_m;
            const int b = g % EB;
            int x = nbk * BN + c * 32, y = mb * CF::kTileRows + (int)rank * BM + 32 * q;
            if constexpr (CORR) {
                if (g == ti * my_nc &&
                    !mbar_wait_warp(&B->corr_full[ti & 1], (uint32_t)(ti >> 1) & 1u, &B->abort,
                                    p.status))
                    return false;
                x = c * 32;
                y = ((int)blockIdx.x * kCorrSlots + (ti & 1)) * BM + 32 * q;
            }
            if (lane == 0) {
                mbar_expect_tx(&B->cbar[ew][b], kEpiBuf);
                tma_load_2d(&tmap_c, &B->cbar[ew][b], bufs + b * kEpiBuf, x, y);
            }
            cpend |= 1u << b;
            return true;
        };
        bool ok = true;
        if (use_c)
            for (int g = 0; ok && g < EB - 1 && g < total; ++g) ok = c_load(g);
        // scales of tile ti into registers (consumed one tile later)
        float swr[SWR];
        float srow_next = 0.0f;
        auto fetch_scales = [&](int ti) {
            const int tile = unit + ti * n_units;
            const int m_blk = p.n_fastest ? tile / num_n : tile % num_m;
            const int n_blk = p.n_fastest ? tile % num_n : tile / num_m;
#pragma unroll
            for (int k = 0; k < SWR; ++k) {
                const int c = par + kEpiSplit * k;           // k-th chunk of this warp
                const int n = n_blk * BN + c * 32 + lane;
                if constexpr (MX) swr[k] = 1.0f;
                else swr[k] = (k < my_nc && n < p.N) ? __ldg(p.sW + n) : 0.0f;
            }
            const int r = m_blk * CF::kTileRows + (int)rank * BM + 32 * q + lane;
            if constexpr (MX) srow_next = 1.0f;
            else srow_next = r < p.M ? __ldg(p.sA + r) : 0.0f;
        };
        if (my_tiles > 0) fetch_scales(0);
        int as = 0;
        uint32_t acc_phase = 0;
        uint32_t va[32], vb[32];
        for (int ti = 0; ok && ti < my_tiles; ++ti) {
            const int tile = unit + ti * n_units;
            const int m_blk = p.n_fastest ? tile / num_n : tile % num_m;
            const int n_blk = p.n_fastest ? tile % num_n : tile / num_m;
            const int row0 = m_blk * CF::kTileRows + (int)rank * BM + 32 * q;
            const int row = row0 + lane;
            // this tile's column scales into the warp's shared-memory copy
            __syncwarp();   // the previous tile's chunks have read sw
#pragma unroll
            for (int k = 0; k < SWR; ++k) sw[32 * k + lane] = swr[k];   // chunk h's scales at sw[32 h]
            const float s_row = srow_next;
            __syncwarp();
            if (ti + 1 < my_tiles) fetch_scales(ti + 1);
            if (!mbar_wait_warp(&B->acc_full[as], acc_phase, &B->abort, p.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // direct epilogue with the fused correction: this tile's slot rows
            const float* cslot = nullptr;
            if constexpr (CORR && !TMA_EPI) {
                if (!mbar_wait_warp(&B->corr_full[ti & 1], (uint32_t)(ti >> 1) & 1u, &B->abort,
                                    p.status)) {
                    ok = false;
                    break;
                }
                cslot = p.corr + ((size_t)((int)blockIdx.x * kCorrSlots + (ti & 1)) * BM +
                                  32 * q + lane) * BN;
            }
            const uint32_t tbase = tmem + lane_base + (uint32_t)(as * BN);
            auto release_acc = [&]() {
                // this warp's chunks fully read: the next tile's MMAs may reuse
                // the accumulator once every epilogue warp has arrived
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (PAIR) mbar_arrive_cluster(map_to_rank(&B->acc_empty[as], 0));
                    else mbar_arrive(&B->acc_empty[as]);
                }
            };
            // one 32-column chunk: Y = acc * s_i * t_j (+ C), staged and stored by TMA
            auto chunk = [&](uint32_t (&v)[32], int h) -> bool {
                const int c = par + kEpiSplit * h;
                const int col0 = n_blk * BN + c * 32;
                if constexpr (!TMA_EPI) {
                    const float* crow = CORR ? cslot + c * 32
                                             : (p.C ? p.C + (int64_t)row * p.N + col0 : nullptr);
                    if (row < p.M && col0 < p.N) epi_direct(p, v, row, col0, s_row, crow);
                    if (CORR && h == my_nc - 1) {
                        // every chunk of the tile is read: the slot may be refilled
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&B->corr_empty[ti & 1]);
                    }
                    return true;
                }
                const int g = ti * my_nc + h;
                const int b = g % EB;
                uint8_t* buf = bufs + b * kEpiBuf;
                // y overwrites the accumulator registers (as fp32 bit patterns)
                const float4* tw = reinterpret_cast<const float4*>(sw + h * 32);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 t = tw[j];
                    const float tt[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        v[4 * j + e] = __float_as_uint(
                            __fmul_rn(__fmul_rn(__uint_as_float(v[4 * j + e]), s_row), tt[e]));
                }
                if (use_c) {
                    if (!mbar_wait_warp(&B->cbar[ew][b], (cphase >> b) & 1u, &B->abort, p.status))
                        return false;
                    cphase ^= 1u << b;
                    cpend &= ~(1u << b);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 t = *reinterpret_cast<const float4*>(buf + swz128(lane, j));
                        const float tt[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            v[4 * j + e] = __float_as_uint(__fadd_rn(__uint_as_float(v[4 * j + e]), tt[e]));
                    }
                    if (CORR && h == my_nc - 1 && lane == 0) {
                        // the tile's last C sub-tile has landed: every TMA read of
                        // its scratch slot is done, the slot may be refilled
                        mbar_arrive(&B->corr_empty[ti & 1]);
                    }
                } else {
                    // buffer b was last read by the store of chunk g - EB
                    if (lane == 0) bulk_wait_read<EB - 1>();
                }
                __syncwarp();   // every lane has read its C row before the buffer is overwritten
                if (p.y_bf16) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t w[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            __nv_bfloat162 hh = __floats2bfloat162_rn(__uint_as_float(v[8 * j + 2 * i]),
                                                                      __uint_as_float(v[8 * j + 2 * i + 1]));
                            w[i] = *reinterpret_cast<uint32_t*>(&hh);
                        }
                        *reinterpret_cast<uint4*>(buf + swz64(lane, j)) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<uint4*>(buf + swz128(lane, j)) =
                            make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (p.y_add) tma_reduce_add_2d(&tmap_y, buf, col0, row0);
                    else tma_store_2d(&tmap_y, buf, col0, row0);
                    bulk_commit();
                }
                if (use_c && g + EB - 1 < total) {
                    // that buffer was last read by the store of chunk g - 1
                    if (lane == 0) bulk_wait_read<1>();
                    if (!c_load(g + EB - 1)) return false;
                }
                return true;
            };
            const uint32_t coff = (uint32_t)(par * 32), cstep = (uint32_t)(kEpiSplit * 32);
            tmem_ld32_issue(tbase + coff, va);
            for (int h = 0; h < my_nc; h += 2) {
                tmem_ld_wait(va);
                if (h + 1 < my_nc) tmem_ld32_issue(tbase + coff + (uint32_t)(h + 1) * cstep, vb);
                else release_acc();
                if (!chunk(va, h)) {
                    ok = false;
                    break;
                }
                if (h + 1 < my_nc) {
                    tmem_ld_wait(vb);
                    if (h + 2 < my_nc) tmem_ld32_issue(tbase + coff + (uint32_t)(h + 2) * cstep, va);
                    else release_acc();
                    if (!chunk(vb, h + 1)) {
                        ok = false;
                        break;
                    }
                }
            }
            if (++as == kAccStages) as = 0, acc_phase ^= 1u;
        }
        tmem_ld_wait_all();
        if (TMA_EPI && lane == 0) {
            bulk_wait_all();
            // on abort, C loads still in flight land before the CTA exits
            for (int b = 0; b < EB; ++b)
                if ((cpend >> b) & 1u) mbar_drain(&B->cbar[ew][b], (cphase >> b) & 1u);
        }
        __syncwarp();
    } else if constexpr (CORR) {
        // ---------------------------------------------------------- correction
        // Warp cw owns rows [r_lo, r_hi) of the CTA's 128 (one contiguous CSR
        // range per tile); tiles in the CTA's order, slot ti % 2.
        const int cw = warp - 2 - kEpiWarps;
        const int r_lo = (cw * BM) / kCorrWarps, r_hi = ((cw + 1) * BM) / kCorrWarps;
        const int my_tiles = unit < num_tiles ? (num_tiles - unit + n_units - 1) / n_units : 0;
        const bool lane_on = lane * 8 < BN;
        for (int ti = 0; ti < my_tiles; ++ti) {
            const int tile = unit + ti * n_units;
            const int m_blk = p.n_fastest ? tile / num_n : tile % num_m;
            const int n_blk = p.n_fastest ? tile % num_n : tile / num_m;
            const int slot = ti & 1;
            if (!mbar_wait_warp(&B->corr_empty[slot], ((uint32_t)(ti >> 1) & 1u) ^ 1u, &B->abort,
                                p.status))
                break;
            const int row0 = m_blk * CF::kTileRows + (int)rank * BM;
            const int rb = min(p.M, row0 + r_lo), re = min(p.M, row0 + r_hi);
            const int c0 = n_blk * BN + lane * 8;
            float* dst = p.corr + ((size_t)((int)blockIdx.x * kCorrSlots + slot) * BM + r_lo) * BN +
                         lane * 8;
            const bool on = lane_on && c0 < p.N;
            const int c_safe = n_blk * BN;           // inside W: the tile exists
            if (p.w_bf16 && (p.N % 8) == 0 && (p.ldw % 8) == 0) {
                // bf16 W with whole, aligned 8-column groups: the quarter-warp
                // loop with its shared-memory ring (every lane of the warp
                // takes part, also when its quarter has no rows)
                const int span = r_hi - r_lo, qd = lane >> 3;
                const int q_lo = r_lo + (qd * span) / 4, q_hi = r_lo + ((qd + 1) * span) / 4;
                corr_rows4s<QG_CORR_D>(p.row_ptr, p.col, p.val, static_cast<const uint16_t*>(p.Wc),
                                       p.ldw, min(p.M, row0 + q_lo), min(p.M, row0 + q_hi),
                                       n_blk * BN, p.N, row0,
                                       p.corr + (size_t)((int)blockIdx.x * kCorrSlots + slot) * BM * BN,
                                       BN, BN, smem + CF::kOffRing + (size_t)cw * kCorrRingBytes);
            } else if (rb < re) {
                if (p.w_bf16) {
                    corr_rows<true, 2, 4>(p.row_ptr, p.col, p.val, p.Wc, p.ldw, rb, re, p.N, c0,
                                          c_safe, on, false, dst, BN);
                } else {
                    const bool fast = (p.N % 8) == 0 && (p.ldw % 4) == 0;
                    corr_rows<false, 2, 2>(p.row_ptr, p.col, p.val, p.Wc, p.ldw, rb, re, p.N, c0,
                                           c_safe, on, fast, dst, BN);
                }
            }
            // the rows are written (generic proxy); the epilogue reads them by
            // TMA (async proxy) once every correction warp has arrived
            asm volatile("fence.proxy.async.global;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&B->corr_full[slot]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();   // the peer no longer touches this CTA
    tc_fence_after();
    if (warp == 1) tmem_free<PAIR>(tmem);
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

static bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                      uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
                      CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tile order: m fastest re-reads A's codes once per column block, n fastest
// W's once per row block.  Both code matrices of the block16k qkv and o
// layers (25-34 MB) stay in L2 beside the output stream either way, and m
// fastest measured slightly better there; A's codes of the down layer
// (16384 x 11008: 90 MB) do not, and n fastest cut that GEMM by a quarter.
// So: n fastest when A's codes exceed 48 MB and W's codes are the smaller.
static int n_fastest_order(int64_t M, int64_t N, int64_t K) {
    const int64_t a_codes = M * (K / 2), w_codes = N * (K / 2);
    return (a_codes > ((int64_t)48 << 20) && w_codes < a_codes) ? 1 : 0;
}

// Tile width: the persistent grid runs ceil(tiles / units) rounds of tiles
// whose time grows with BN, so pick the width with the smaller rounds x BN;
// on a tie, the one that pads N less.
static int pick_bn(int64_t M, int64_t N, bool pair) {
    const int64_t row_tiles = (M + (pair ? 255 : 127)) / (pair ? 256 : 128);
    const int64_t units = std::max<int64_t>(1, num_sms() / (pair ? 2 : 1));
    auto cost = [&](int64_t bn) {
        const int64_t tiles = row_tiles * ((N + bn - 1) / bn);
        return ((tiles + units - 1) / units) * bn;
    };
    const int64_t c224 = cost(224), c192 = cost(192);
    if (c224 != c192) return c224 < c192 ? 224 : 192;
    const int64_t w224 = ((N + 223) / 224) * 224 - N;
    const int64_t w192 = ((N + 191) / 192) * 192 - N;
    return (w192 < w224) ? 192 : 224;
}

// CTAs of the persistent grid (units of one CTA or one pair, at most one per
// SM, and at most kCorrMaxCtas with the fused correction).
template <int BN, bool PAIR, bool CORR = false>
static int grid_ctas(int64_t M, int64_t N) {
    using CF = Cfg<BN, PAIR, false>;
    const int64_t tiles = ((M + CF::kTileRows - 1) / CF::kTileRows) * ((N + BN - 1) / BN);
    const int per_unit = PAIR ? 2 : 1;
    int64_t units = std::min<int64_t>(tiles, num_sms() / per_unit);
    if (CORR) units = std::min<int64_t>(units, kCorrMaxCtas / per_unit);
    return (int)std::max<int64_t>(units, 1) * per_unit;
}

template <int BN, bool PAIR, bool TMA_EPI, bool MX = false, bool CORR = false, bool DEEP = false>
static cudaError_t launch_variant(const CUtensorMap& ta, const uint8_t* codesWT, int64_t N,
                                  int64_t K, const CUtensorMap& ty, const CUtensorMap& tc,
                                  const Params& p, cudaStream_t s) {
    using CF = Cfg<BN, PAIR, MX>;
    CUtensorMap tb;
    if (!encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, codesWT, K / 2, N, K / 2, BK_BYTES,
                   CF::kBRows, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int64_t tiles = ((p.M + CF::kTileRows - 1) / CF::kTileRows) * ((N + BN - 1) / BN);
    const int per_unit = PAIR ? 2 : 1;
    int64_t max_units = num_sms() / per_unit;
    if (CORR) max_units = std::min<int64_t>(max_units, kCorrMaxCtas / per_unit);
    const int units = (int)std::min<int64_t>(tiles, max_units);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(units * per_unit));
    cfg.blockDim = dim3(threads_of<CORR>());
    cfg.dynamicSmemBytes = smem_bytes<BN, PAIR, MX, CORR, DEEP>();
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = per_unit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, fp4_gemm_kernel<BN, PAIR, TMA_EPI, MX, CORR, DEEP>, ta, tb,
                                       ty, tc, p);
    count_launch(1);
    return e;
}

template <int BN, bool PAIR, bool MX = false, bool CORR = false>
static cudaError_t set_smem_attr() {
    if constexpr (BN == 192 && PAIR && !MX && !CORR) {
        const cudaError_t d = cudaFuncSetAttribute(fp4_gemm_kernel<BN, true, true, false, false, true>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)smem_bytes<BN, true, false, false, true>());
        if (d != cudaSuccess) return d;
    }
    cudaError_t e = cudaFuncSetAttribute(fp4_gemm_kernel<BN, PAIR, true, MX, CORR>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_bytes<BN, PAIR, MX, CORR>());
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(fp4_gemm_kernel<BN, PAIR, false, MX, CORR>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem_bytes<BN, PAIR, MX, CORR>());
}

}  // namespace gemm

cudaError_t gemm_setup() {
    using namespace gemm;
    cudaError_t e;
    if ((e = set_smem_attr<224, false>()) != cudaSuccess) return e;
    if ((e = set_smem_attr<192, false>()) != cudaSuccess) return e;
    if ((e = set_smem_attr<224, true>()) != cudaSuccess) return e;
    if ((e = set_smem_attr<128, false, true>()) != cudaSuccess) return e;
    if ((e = set_smem_attr<192, true>()) != cudaSuccess) return e;
    if ((e = set_smem_attr<224, false, false, true>()) != cudaSuccess) return e;
    if ((e = set_smem_attr<192, false, false, true>()) != cudaSuccess) return e;
    if ((e = set_smem_attr<224, true, false, true>()) != cudaSuccess) return e;
    return set_smem_attr<192, true, false, true>();
}

static_assert(kCorrScratchBytes ==
                  (size_t)gemm::kCorrMaxCtas * gemm::kCorrSlots * gemm::BM * 224 * sizeof(float),
              "scratch of the fused correction: two 128 x 224 fp32 slots per CTA");

// Returns cudaErrorInvalidValue when the tensor maps cannot be built.
cudaError_t launch_fp4_gemm(const uint8_t* codesA, const float* sA, const uint8_t* codesWT,
                            const float* sW, int64_t M, int64_t N, int64_t K, const float* C,
                            void* Y, qg_dtype y_dtype, float* raw_acc, uint32_t* status,
                            cudaStream_t s, bool y_add) {
    using namespace gemm;
    Params p{};
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
    p.unit_scales = 0;
    p.sfA = nullptr;
    p.sfB = nullptr;
    p.sf_groups = 0;
    p.n_fastest = n_fastest_order(M, N, K);
    // TMA epilogue: the row pitches of Y and C must be multiples of 16 bytes
    const size_t ysz = (y_dtype == QG_BF16) ? 2 : 4;
#ifndef QG_GEMM_DIRECT_EPI
#define QG_GEMM_DIRECT_EPI 0
#endif
    p.tma_epi = (!QG_GEMM_DIRECT_EPI && Y != nullptr && raw_acc == nullptr &&
                 ((size_t)N * ysz) % 16 == 0 && ((size_t)N * 4) % 16 == 0)
                    ? 1
                    : 0;
    // adding into Y: through the TMA epilogue only, fp32 Y, no C
    if (y_add && (!p.tma_epi || y_dtype != QG_F32 || C != nullptr)) return cudaErrorInvalidValue;
    p.y_add = y_add ? 1 : 0;
    CUtensorMap ta, ty, tc;
    if (!encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, codesA, K / 2, M, K / 2, BK_BYTES, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    ty = ta;
    tc = ta;
    if (p.tma_epi) {
        if (y_dtype == QG_BF16) {
            if (!encode_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, N * 2, 32, 32,
                           CU_TENSOR_MAP_SWIZZLE_64B))
                return cudaErrorInvalidValue;
        } else {
            if (!encode_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Y, N, M, N * 4, 32, 32,
                           CU_TENSOR_MAP_SWIZZLE_128B))
                return cudaErrorInvalidValue;
        }
        if (C != nullptr &&
            !encode_2d(&tc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, C, N, M, N * 4, 32, 32,
                       CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    // the CTA pair when there are enough 256-row tiles to fill the SMs in pairs
    const bool pair = M > BM;
    const int bn = QG_GEMM_FORCE_BN ? QG_GEMM_FORCE_BN : pick_bn(p.M, N, pair);
    if (pair) {
        if (p.tma_epi && C == nullptr && bn == 192)
            return launch_variant<192, true, true, false, false, true>(ta, codesWT, N, K, ty, tc, p, s);
        if (p.tma_epi) {
            if (bn == 192) return launch_variant<192, true, true>(ta, codesWT, N, K, ty, tc, p, s);
            return launch_variant<224, true, true>(ta, codesWT, N, K, ty, tc, p, s);
        }
        if (bn == 192) return launch_variant<192, true, false>(ta, codesWT, N, K, ty, tc, p, s);
        return launch_variant<224, true, false>(ta, codesWT, N, K, ty, tc, p, s);
    }
    if (p.tma_epi) {
        if (bn == 192) return launch_variant<192, false, true>(ta, codesWT, N, K, ty, tc, p, s);
        return launch_variant<224, false, true>(ta, codesWT, N, K, ty, tc, p, s);
    }
    if (bn == 192) return launch_variant<192, false, false>(ta, codesWT, N, K, ty, tc, p, s);
    return launch_variant<224, false, false>(ta, codesWT, N, K, ty, tc, p, s);
}

// The compensated GEMM: Y = acc * sA_i * sW_j + (dA . W)_ij, the correction
// computed inside the GEMM kernel (CORR) into scratch slots of `scratch`
// (corr_scratch_bytes()).  Returns cudaErrorInvalidValue when the tensor maps
// cannot be built.
cudaError_t launch_fp4_gemm_corr(const uint8_t* codesA, const float* sA, const uint8_t* codesWT,
                                 const float* sW, int64_t M, int64_t N, int64_t K,
                                 const qg_csr* dA, const void* W, qg_dtype w_dtype, int64_t ldw,
                                 float* scratch, void* Y, qg_dtype y_dtype, uint32_t* status,
                                 cudaStream_t s) {
    using namespace gemm;
    Params p{};
    p.sA = sA;
    p.sW = sW;
    p.C = nullptr;
    p.Y = Y;
    p.raw_acc = nullptr;
    p.status = status;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.y_bf16 = (y_dtype == QG_BF16) ? 1 : 0;
    p.unit_scales = 0;
    p.sfA = nullptr;
    p.sfB = nullptr;
    p.sf_groups = 0;
    p.row_ptr = dA->row_ptr;
    p.col = dA->col;
    p.val = dA->val;
    p.Wc = W;
    p.ldw = ldw;
    p.w_bf16 = (w_dtype == QG_BF16) ? 1 : 0;
    p.corr = scratch;
    p.n_fastest = n_fastest_order(M, N, K);
    const size_t ysz = (y_dtype == QG_BF16) ? 2 : 4;
    p.tma_epi = (!QG_GEMM_DIRECT_EPI && ((size_t)N * ysz) % 16 == 0) ? 1 : 0;
    const bool pair = M > BM;
    const int bn = QG_GEMM_FORCE_BN ? QG_GEMM_FORCE_BN : pick_bn(p.M, N, pair);
    const int ctas = pair ? (bn == 192 ? grid_ctas<192, true, true>(M, N) : grid_ctas<224, true, true>(M, N))
                          : (bn == 192 ? grid_ctas<192, false, true>(M, N) : grid_ctas<224, false, true>(M, N));
    CUtensorMap ta, ty, tc;
    if (!encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, codesA, K / 2, M, K / 2, BK_BYTES, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    ty = ta;
    tc = ta;
    if (p.tma_epi) {
        if (y_dtype == QG_BF16) {
            if (!encode_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, N * 2, 32, 32,
                           CU_TENSOR_MAP_SWIZZLE_64B))
                return cudaErrorInvalidValue;
        } else {
            if (!encode_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Y, N, M, N * 4, 32, 32,
                           CU_TENSOR_MAP_SWIZZLE_128B))
                return cudaErrorInvalidValue;
        }
        // the scratch as a (ctas x slots x 128) x bn fp32 matrix
        if (!encode_2d(&tc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, scratch, bn,
                       (uint64_t)ctas * kCorrSlots * BM, (uint64_t)bn * 4, 32, 32,
                       CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    if (pair) {
        if (p.tma_epi) {
            if (bn == 192) return launch_variant<192, true, true, false, true>(ta, codesWT, N, K, ty, tc, p, s);
            return launch_variant<224, true, true, false, true>(ta, codesWT, N, K, ty, tc, p, s);
        }
        if (bn == 192) return launch_variant<192, true, false, false, true>(ta, codesWT, N, K, ty, tc, p, s);
        return launch_variant<224, true, false, false, true>(ta, codesWT, N, K, ty, tc, p, s);
    }
    if (p.tma_epi) {
        if (bn == 192) return launch_variant<192, false, true, false, true>(ta, codesWT, N, K, ty, tc, p, s);
        return launch_variant<224, false, true, false, true>(ta, codesWT, N, K, ty, tc, p, s);
    }
    if (bn == 192) return launch_variant<192, false, false, false, true>(ta, codesWT, N, K, ty, tc, p, s);
    return launch_variant<224, false, false, false, true>(ta, codesWT, N, K, ty, tc, p, s);
}

// MXFP4 GEMM: Y = sum over 32-blocks of 2^(eA + eW) * (block product) (+ C).
cudaError_t launch_fp4_gemm_mx(const uint8_t* codesA, const uint8_t* sfA, const uint8_t* codesWT,
                               const uint8_t* sfW, int64_t M, int64_t N, int64_t K, const float* C,
                               void* Y, qg_dtype y_dtype, float* raw_acc, uint32_t* status,
                               cudaStream_t s) {
    using namespace gemm;
    Params p{};
    p.sA = nullptr;
    p.sW = nullptr;
    p.C = C;
    p.Y = Y;
    p.raw_acc = raw_acc;
    p.status = status;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.y_bf16 = (y_dtype == QG_BF16) ? 1 : 0;
    p.unit_scales = 1;
    p.sfA = sfA;
    p.sfB = sfW;
    p.sf_groups = (int)(2 * ((K + 255) / 256));
    const size_t ysz = (y_dtype == QG_BF16) ? 2 : 4;
    p.tma_epi = (!QG_GEMM_DIRECT_EPI && Y != nullptr && raw_acc == nullptr &&
                 ((size_t)N * ysz) % 16 == 0 && ((size_t)N * 4) % 16 == 0)
                    ? 1
                    : 0;
    CUtensorMap ta, ty, tc;
    if (!encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, codesA, K / 2, M, K / 2, BK_BYTES, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    ty = ta;
    tc = ta;
    if (p.tma_epi) {
        if (y_dtype == QG_BF16) {
            if (!encode_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, N * 2, 32, 32,
                           CU_TENSOR_MAP_SWIZZLE_64B))
                return cudaErrorInvalidValue;
        } else {
            if (!encode_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Y, N, M, N * 4, 32, 32,
                           CU_TENSOR_MAP_SWIZZLE_128B))
                return cudaErrorInvalidValue;
        }
        if (C != nullptr &&
            !encode_2d(&tc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, C, N, M, N * 4, 32, 32,
                       CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        return launch_variant<128, false, true, true>(ta, codesWT, N, K, ty, tc, p, s);
    }
    return launch_variant<128, false, false, true>(ta, codesWT, N, K, ty, tc, p, s);
}

}  // namespace qg
