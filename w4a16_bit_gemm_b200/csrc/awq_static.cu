// awq_static.cu -- the AWQ scaling search with library-owned scratch.
//
// wq_awq_search_static runs wq_awq_search on a file-scope device array
// instead of a caller workspace, for callers that cannot allocate device
// memory (they run under an allocator they may not bypass, or must not grow
// their device footprint after start-up); the search itself allocates
// nothing.  The array is reserved when the CUDA module holding it is loaded
// on a device: at the first call under lazy module loading (the default), at
// context creation under CUDA_MODULE_LOADING=EAGER.  Every call on a device
// shares the array: calls whose work overlaps on the GPU race (queue them on
// one stream).
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/wq.h"
#include "wq_kernels.h"

namespace {

constexpr size_t kAwqStaticScratchBytes = 80ull << 20;  // the 4096 x 4096 layer with 512 tokens needs ~61 MB
static __device__ __align__(256) uint8_t g_awq_static_scratch[kAwqStaticScratchBytes];

}  // namespace

extern "C" size_t wq_awq_static_scratch_bytes(void) { return kAwqStaticScratchBytes; }

extern "C" wq_status wq_awq_search_static(const void* W_bf16, int64_t d_out, int64_t d_in, const void* X_bf16,
                                          int64_t T, int32_t group_size, int32_t symmetric, uint32_t* qweight,
                                          void* scales_fp16, void* zeros_fp16, void* s_bf16, double* losses,
                                          int32_t* best, void* stream) {
    wq_status v = wq::awq_check_args(W_bf16, d_out, d_in, X_bf16, T, group_size, symmetric, qweight, scales_fp16,
                                     zeros_fp16, s_bf16, losses, best);
    if (v != WQ_OK) return v;
    if (wq_awq_workspace_bytes(d_out, d_in, T, group_size) > kAwqStaticScratchBytes) return WQ_ERR_UNSUPPORTED;
    // the scratch's set-up (symbol lookup) comes before the search's own: both
    // injected faults land here
    if (wq::fault_injected(wq::kFaultAlloc) || wq::fault_injected(wq::kFaultLaunch)) return WQ_ERR_CUDA;
    void* ws = nullptr;
    if (cudaGetSymbolAddress(&ws, g_awq_static_scratch) != cudaSuccess) return WQ_ERR_CUDA;
    return wq_awq_search(W_bf16, d_out, d_in, X_bf16, T, group_size, symmetric, qweight, scales_fp16, zeros_fp16,
                         s_bf16, losses, best, ws, kAwqStaticScratchBytes, stream);
}
