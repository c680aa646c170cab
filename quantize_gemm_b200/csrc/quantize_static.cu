// quantize_static.cu -- qg_quantize_cols_static: the channel-wise weight
// quantizer with its scratch memory in a fixed device array instead of a
// caller-provided workspace, for callers that cannot allocate device memory.
//
// The scratch is the per-column maximum written by the first pass and read
// by the second.  It lives in g_colmax_scratch below (kStaticColsMax uint32,
// 256 KB), which every GPU that loads this library holds until the process
// exits.  Host code cannot use the array's name as a device address, so the
// address is looked up once per device (cudaGetSymbolAddress, with that device
// current) on the first call made on that device, and cached; a
// cudaDeviceReset ends the context that address belongs to, so the cache is
// only valid until then.  Both dtypes run the two-pass kernels of
// qg_quantize_cols's fp32 path (column maxima, then codes): the cooperative
// bf16 kernel of qg_quantize_cols keeps per-split maxima and a grid barrier in
// its workspace, which would need a larger fixed array.
#include <mutex>

#include "qg_internal.cuh"

namespace qg {

constexpr int64_t kStaticColsMax = 65536;

static __device__ __align__(256) uint32_t g_colmax_scratch[kStaticColsMax];

static std::mutex g_static_mu;
static uint32_t* g_static_ptr[64];     // device address of the array, per device

// Device address of g_colmax_scratch on the current device (nullptr on error).
static uint32_t* static_scratch() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (g_static_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_colmax_scratch) != cudaSuccess || p == nullptr)
            return nullptr;
        g_static_ptr[dev] = static_cast<uint32_t*>(p);
    }
    return g_static_ptr[dev];
}

}  // namespace qg

using namespace qg;

extern "C" qg_status qg_quantize_cols_static(const void* W, qg_dtype dtype, int64_t K, int64_t N,
                                             int64_t ldw, uint8_t* codesT, float* scales,
                                             cudaStream_t stream) {
    // the checks of qg_quantize_cols (same helpers), then the array's capacity
    if (!dtype_ok(dtype)) return QG_ERR_INVALID_ARG;
    qg_status st = check_mk(N, K);
    if (st != QG_OK) return st;
    if (N > kStaticColsMax) return QG_ERR_UNSUPPORTED_SHAPE;
    if (W == nullptr || !aligned16(W) || ldw < N) return QG_ERR_INVALID_ARG;
    if (!codesT || !scales || !aligned16(codesT)) return QG_ERR_INVALID_ARG;
    if (device_setup() != cudaSuccess) return QG_ERR_CUDA;
    uint32_t* colmax = static_scratch();
    if (colmax == nullptr) return QG_ERR_CUDA;
    // the same two kernels as qg_quantize_cols; the column maxima are zeroed
    // first, since the array keeps whatever the previous call left in it
    launch_quantize_cols(W, dtype, K, N, ldw, codesT, scales, colmax, stream);
    return cuda_status(cudaGetLastError());
}
