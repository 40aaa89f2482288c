// wq_kernels.h -- host-side launch functions of the libwq kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/wq.h"

namespace wq {

// Host-side fault injection (WQ_FAULT_INJECT): true when the named step is to
// fail in this process (the failure is counted for wq_fault_injections).
enum FaultStep { kFaultNone = 0, kFaultLaunch = 1, kFaultAlloc = 2 };
bool fault_injected(int step);

cudaError_t launch_quantize(const void* W, int64_t d_out, int64_t d_in, int g, int symmetric, uint32_t* qweight,
                            uint16_t* scales, uint16_t* zeros, uint32_t* status, int num_sms, cudaStream_t stream);

// Quantize with the per-group MSE-optimal clipping search; g in {32, 64, 128, 256}
// (cudaErrorNotSupported otherwise).
cudaError_t launch_quantize_clip(const void* W, int64_t d_out, int64_t d_in, int g, int symmetric,
                                 uint32_t* qweight, uint16_t* scales, uint16_t* zeros, uint32_t* status,
                                 int num_sms, cudaStream_t stream);

cudaError_t launch_dequantize(const uint32_t* qweight, const uint16_t* scales, const uint16_t* zeros,
                              int64_t d_out, int64_t d_in, int g, int symmetric, void* W_hat, int num_sms,
                              cudaStream_t stream);

// Decode GEMV, M <= 16.
struct GemvArgs {
    const void* X;           // bf16 [M][K]
    const uint16_t* scales;  // fp16 [N][G]
    const uint16_t* zeros;   // fp16 [N][G] or nullptr (symmetric)
    void* Y;                 // [M][N] bf16 or fp32
    uint32_t* status;
    int M, N, K, G, g;
    int g_shift;       // log2(g) when g is a power of two, else -1
    int rows_per_cta;  // npass * BR
    int BR;            // rows per pass, <= 64
    int T;             // tiles per pass
    int BRT;           // rows per tile (TMA box height), <= 16
    int npass;
    int nkb;           // ceil(K / 128)
    int nks;           // row segments of 2048 k per row
    int pitch;         // padded shared-memory row pitch of a slot (bytes)
    int nslots;        // smem slots (ring when fewer than the chunks)
    int slot_bytes;
    int xs_bytes;      // activations staged in smem (0: read from global)
    int symmetric;
    int y_fp32;
};

struct LaunchOptions {
    bool pdl;  // programmatic dependent launch (prefetch weights before the previous kernel ends)
};

cudaError_t launch_gemv(const uint32_t* qweight, const GemvArgs& base, int num_sms, const LaunchOptions& opt,
                        cudaStream_t stream);

// Decode GEMV for M <= 8 whose MMA tiles mix rows and k ranges (gemv_ksplit.cu);
// two CTAs per SM when they fit, so consecutive launches overlap.
struct KsArgs {
    const void* X;           // bf16 [M][K]
    const uint16_t* scales;  // fp16 [N][G]
    const uint16_t* zeros;   // fp16 [N][G] or nullptr (symmetric)
    void* Y;                 // [M][N] bf16 or fp32
    uint32_t* status;
    int M, N, K, G, g;
    int g_shift;     // log2(g) when g is a power of two, else -1
    int R;           // rows per CTA (set by the launcher)
    int RC;          // rows per chunk (set by the launcher)
    int nslots;      // shared-memory slots (set by the launcher)
    int slot_bytes;  // (set by the launcher)
    int pre;         // ring kernel: park leading chunks in tensor memory before the
                     // wait (two CTAs per SM, so the next launch overlaps; set by the launcher)
    int symmetric;
    int y_fp32;
};

cudaError_t launch_gemv_ksplit(const uint32_t* qweight, const KsArgs& a, int num_sms, const LaunchOptions& opt,
                               cudaStream_t stream);

// Decode GEMV for a few tokens, weights streamed k-major (gemv_kmajor.cu):
// M <= 16, K >= 2048, N >= 16, power-of-two g; cudaErrorNotSupported otherwise.
struct KmArgs {
    const void* X;           // bf16 [M][K]
    const uint16_t* scales;  // fp16 [N][G]
    const uint16_t* zeros;   // fp16 [N][G] or nullptr (symmetric)
    void* Y;                 // [M][N] bf16 or fp32
    uint32_t* status;
    int M, N, K, G, g;
    int g_shift;  // log2(g)
    int symmetric;
    int y_fp32;
    int gpc;        // groups per row of a 1024-k chunk (set by the launcher)
    int gpc_shift;  // log2(gpc)
    int prb;      // 16-row blocks per pass (set by the launcher)
    int nslots;   // shared-memory slots (set by the launcher)
};

cudaError_t launch_gemv_kmajor(const uint32_t* qweight, const KmArgs& a, int num_sms, const LaunchOptions& opt,
                               cudaStream_t stream);

// M <= 2 on tensor cores (dequantized weights as the A operand in tensor
// memory); cudaErrorNotSupported for shapes it does not take.
cudaError_t launch_gemv_tc(const uint32_t* qweight, const GemvArgs& a, int num_sms, const LaunchOptions& opt,
                           cudaStream_t stream);

// WQ_GEMV_TC=0 in the environment keeps M <= 2 off the tensor-memory kernel
// (read once per process).
bool gemv_tc_disabled();
// WQ_GEMV_KSPLIT=0 keeps M <= 8 off the k-split kernel (read once per process).
bool gemv_ksplit_disabled();
// WQ_GEMV_KMAJOR=0 keeps M >= 2 off the k-major kernel (read once per process).
bool gemv_kmajor_disabled();

// Prefill GEMM on tcgen05 tensor cores, any M (used for M > 16).
struct GemmArgs {
    const void* X;           // bf16 [M][K]
    const uint32_t* qweight; // [N][K/8]
    const uint16_t* scales;  // fp16 [N][G]
    const uint16_t* zeros;   // fp16 [N][G] or nullptr
    void* Y;                 // [M][N]
    uint32_t* status;
    int M, N, K, G, g;
    int symmetric;
    int y_fp32;
    int bits;  // 4 (qweight [N][K/8], nibbles), 8 (qweight [N][K/4], symmetric bytes) or
               // 16 (qweight: unquantized bf16 [N][K]; scales, zeros unused)
};

cudaError_t launch_gemm(const GemmArgs& a, int num_sms, const LaunchOptions& opt, cudaStream_t stream);

// AWQ search pieces (awq.cu).
cudaError_t launch_awq_colstats(const uint16_t* X, int64_t T, int64_t K, double* lnm, double* mean_ln,
                                cudaStream_t stream);
cudaError_t launch_awq_scale_apply(const uint16_t* W, int64_t N, const uint16_t* X, int64_t T, int64_t K,
                                   const double* lnm, const double* mean_ln, int alpha_idx, const int32_t* best,
                                   uint16_t* s, uint16_t* Wp, uint16_t* Xp, int num_sms, cudaStream_t stream);
cudaError_t launch_awq_divide(const uint16_t* X, int64_t T, int64_t K, const uint16_t* s, uint16_t* Xp, int num_sms,
                              cudaStream_t stream);
cudaError_t launch_awq_loss(const float* Yref, const float* Y, int64_t n, double* part, double* out,
                            cudaStream_t stream);
cudaError_t launch_awq_select(const double* losses, int n, int32_t* best, cudaStream_t stream);
int awq_loss_partials();
// Argument checks of the AWQ search (everything except the workspace).
wq_status awq_check_args(const void* W_bf16, int64_t d_out, int64_t d_in, const void* X_bf16, int64_t T,
                         int32_t group_size, int32_t symmetric, const uint32_t* qweight, const void* scales_fp16,
                         const void* zeros_fp16, const void* s_bf16, const double* losses, const int32_t* best);

// W8A16 (w8.cu): symmetric INT8 [-127, 127], 4 codes per word.
struct W8Args {
    const void* X;           // bf16 [M][K]
    const uint32_t* qweight; // [N][K/4]
    const uint16_t* scales;  // fp16 [N][G]
    void* Y;                 // [M][N] bf16 or fp32
    uint32_t* status;
    int64_t N, K, G;
    int M, g, y_fp32;
};
cudaError_t launch_quantize_w8(const void* W, int64_t N, int64_t K, int g, uint32_t* qweight, uint16_t* scales,
                               uint32_t* status, int num_sms, cudaStream_t stream);
cudaError_t launch_dequantize_w8(const uint32_t* qweight, const uint16_t* scales, int64_t N, int64_t K, int g,
                                 void* out, int num_sms, cudaStream_t stream);
cudaError_t launch_gemv_w8a16(const W8Args& a, cudaStream_t stream);  // M <= 16

// GPTQ (gptq.cu): scales/zeros must already hold the RTN parameters of W.
size_t gptq_workspace_bytes(int64_t N, int64_t K);
cudaError_t launch_gptq(const uint16_t* W, int64_t N, int64_t K, const uint16_t* X, int64_t T, int g, int symmetric,
                        int act_order, uint32_t* qweight, const uint16_t* scales, const uint16_t* zeros,
                        int32_t* perm_out, void* workspace, uint32_t* status, cudaStream_t stream);

cudaError_t launch_bounded_wait_selftest(uint32_t* status, uint32_t limit_us, cudaStream_t stream);

// Driver entry point for tensor-map encoding (resolved once through the runtime).
CUresult encode_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                              uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                              CUtensorMapSwizzle swizzle);

}  // namespace wq
