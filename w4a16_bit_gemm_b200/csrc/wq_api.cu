// wq_api.cu -- the extern "C" boundary of libwq (declared in include/wq.h).
//
// Host-side argument validation, the per-device status word, tensor-map
// encoding through the driver entry point, and dispatch to the kernels.
// No entry point allocates device memory: the status word is a static device
// variable and every other buffer belongs to the caller.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/wq.h"
#include "wq_kernels.h"

namespace wq {

// Device status word (WQ_DEVFLAG_* bits), one per device that loads the library.
__device__ uint32_t g_status_word;

// Host-side fault injection (WQ_FAULT_INJECT=launch|alloc, read once per
// process): the named step fails as a CUDA error would, before anything is
// enqueued, and the call returns WQ_ERR_CUDA; every such failure is counted.
namespace {
std::atomic<uint64_t> g_fault_count{0};
int fault_mode() {
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("WQ_FAULT_INJECT");
        v = !e ? kFaultNone : strcmp(e, "launch") == 0 ? kFaultLaunch : strcmp(e, "alloc") == 0 ? kFaultAlloc : kFaultNone;
    }
    return v;
}
}  // namespace

bool fault_injected(int step) {
    if (fault_mode() != step) return false;
    g_fault_count.fetch_add(1);
    return true;
}

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint32_t* g_status_ptr[kMaxDevices];
int g_num_sms[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct DeviceState {
    int dev;
    uint32_t* status;
    int num_sms;
};

// Per-device set-up on first use: address of the status word, SM count.
// Must not run inside a stream capture (it may load the module).
wq_status device_state(DeviceState* st) {
    // the per-device set-up reserves device memory (module load) and is the
    // last host step before every launch: both injected faults land here
    if (fault_injected(kFaultAlloc) || fault_injected(kFaultLaunch)) return WQ_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return WQ_ERR_CUDA;
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return WQ_ERR_CUDA;
        g_num_sms[dev] = sms;
        g_status_ptr[dev] = static_cast<uint32_t*>(p);
    }
    st->dev = dev;
    st->status = g_status_ptr[dev];
    st->num_sms = g_num_sms[dev];
    return WQ_OK;
}

bool group_size_ok(int64_t d_in, int32_t g) {
    if (g <= 0 || d_in % g != 0) return false;
    if (g == 32 || g == 64 || g == 128 || g == 256) return true;
    return g % 256 == 0;
}

wq_status check_artifact(const void* qweight, const void* scales, const void* zeros, int64_t d_out, int64_t d_in,
                         int32_t g, int32_t symmetric) {
    if (!qweight || !scales) return WQ_ERR_INVALID_ARG;
    if (d_out < 1 || d_in < 1 || d_out > (1ll << 31) - 1 || d_in > (1ll << 31) - 1) return WQ_ERR_INVALID_ARG;
    if (symmetric != 0 && symmetric != 1) return WQ_ERR_INVALID_ARG;
    if (!group_size_ok(d_in, g)) return WQ_ERR_INVALID_ARG;
    if (symmetric == 0 && !zeros) return WQ_ERR_INVALID_ARG;
    if (symmetric == 1 && zeros) return WQ_ERR_INVALID_ARG;
    if (!aligned(qweight, 16) || !aligned(scales, 2) || (zeros && !aligned(zeros, 2))) return WQ_ERR_INVALID_ARG;
    return WQ_OK;
}

bool pdl_enabled() {
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("WQ_DISABLE_PDL");
        v = (e && e[0] == '1') ? 0 : 1;
    }
    return v == 1;
}

}  // namespace

bool gemv_tc_disabled() {
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("WQ_GEMV_TC");
        v = (e && e[0] == '0') ? 1 : 0;
    }
    return v == 1;
}

bool gemv_ksplit_disabled() {
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("WQ_GEMV_KSPLIT");
        v = (e && e[0] == '0') ? 1 : 0;
    }
    return v == 1;
}

bool gemv_kmajor_disabled() {
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("WQ_GEMV_KMAJOR");
        v = (e && e[0] == '0') ? 1 : 0;
    }
    return v == 1;
}

CUresult encode_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                              uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                              CUtensorMapSwizzle swizzle) {
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
                    cudaSuccess ||
                q != cudaDriverEntryPointSuccess || !fn)
                return CUDA_ERROR_NOT_FOUND;
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
    }
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

wq_status awq_check_args(const void* W_bf16, int64_t d_out, int64_t d_in, const void* X_bf16, int64_t T,
                         int32_t group_size, int32_t symmetric, const uint32_t* qweight, const void* scales_fp16,
                         const void* zeros_fp16, const void* s_bf16, const double* losses, const int32_t* best) {
    wq_status v = check_artifact(qweight, scales_fp16, zeros_fp16, d_out, d_in, group_size, symmetric);
    if (v != WQ_OK) return v;
    if (!W_bf16 || !X_bf16 || !s_bf16 || !aligned(W_bf16, 16) || !aligned(X_bf16, 16) || !aligned(s_bf16, 2))
        return WQ_ERR_INVALID_ARG;
    if (T < 1 || T > (1ll << 31) - 1 || (d_in % 8) != 0) return WQ_ERR_INVALID_ARG;
    if ((losses && !aligned(losses, 8)) || (best && !aligned(best, 4))) return WQ_ERR_INVALID_ARG;
    return WQ_OK;
}

}  // namespace wq

using namespace wq;

extern "C" {

int32_t wq_abi_version(void) { return WQ_ABI_VERSION; }

uint64_t wq_fault_injections(void) { return g_fault_count.load(); }

const char* wq_status_string(wq_status s) {
    switch (s) {
        case WQ_OK: return "WQ_OK";
        case WQ_ERR_INVALID_ARG: return "WQ_ERR_INVALID_ARG";
        case WQ_ERR_UNSUPPORTED: return "WQ_ERR_UNSUPPORTED";
        case WQ_ERR_CUDA: return "WQ_ERR_CUDA";
        case WQ_ERR_NONFINITE: return "WQ_ERR_NONFINITE";
        case WQ_ERR_TIMEOUT: return "WQ_ERR_TIMEOUT";
        case WQ_ERR_RANGE: return "WQ_ERR_RANGE";
    }
    return "WQ_ERR_UNKNOWN";
}

wq_status wq_quantize_rtn(const void* W_bf16, int64_t d_out, int64_t d_in, int32_t group_size, int32_t symmetric,
                          uint32_t* qweight, void* scales_fp16, void* zeros_fp16, void* stream) {
    if (!W_bf16 || !aligned(W_bf16, 16)) return WQ_ERR_INVALID_ARG;
    wq_status v = check_artifact(qweight, scales_fp16, zeros_fp16, d_out, d_in, group_size, symmetric);
    if (v != WQ_OK) return v;
    DeviceState st;
    if ((v = device_state(&st)) != WQ_OK) return v;
    cudaError_t e = launch_quantize(W_bf16, d_out, d_in, group_size, symmetric, qweight,
                                    static_cast<uint16_t*>(scales_fp16), static_cast<uint16_t*>(zeros_fp16), st.status,
                                    st.num_sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

wq_status wq_quantize_clip_mse(const void* W_bf16, int64_t d_out, int64_t d_in, int32_t group_size,
                               int32_t symmetric, uint32_t* qweight, void* scales_fp16, void* zeros_fp16,
                               void* stream) {
    if (!W_bf16 || !aligned(W_bf16, 16)) return WQ_ERR_INVALID_ARG;
    wq_status v = check_artifact(qweight, scales_fp16, zeros_fp16, d_out, d_in, group_size, symmetric);
    if (v != WQ_OK) return v;
    if (group_size != 32 && group_size != 64 && group_size != 128 && group_size != 256) return WQ_ERR_UNSUPPORTED;
    DeviceState st;
    if ((v = device_state(&st)) != WQ_OK) return v;
    cudaError_t e = launch_quantize_clip(W_bf16, d_out, d_in, group_size, symmetric, qweight,
                                         static_cast<uint16_t*>(scales_fp16), static_cast<uint16_t*>(zeros_fp16),
                                         st.status, st.num_sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

wq_status wq_dequantize(const uint32_t* qweight, const void* scales_fp16, const void* zeros_fp16, int64_t d_out,
                        int64_t d_in, int32_t group_size, int32_t symmetric, void* W_hat_bf16, void* stream) {
    wq_status v = check_artifact(qweight, scales_fp16, zeros_fp16, d_out, d_in, group_size, symmetric);
    if (v != WQ_OK) return v;
    if (!W_hat_bf16 || !aligned(W_hat_bf16, 16)) return WQ_ERR_INVALID_ARG;
    DeviceState st;
    if ((v = device_state(&st)) != WQ_OK) return v;
    cudaError_t e = launch_dequantize(qweight, static_cast<const uint16_t*>(scales_fp16),
                                      static_cast<const uint16_t*>(zeros_fp16), d_out, d_in, group_size, symmetric,
                                      W_hat_bf16, st.num_sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

size_t wq_linear_workspace_bytes(int64_t M, int64_t d_out, int64_t d_in) {
    (void)M;
    (void)d_out;
    (void)d_in;
    return 0;
}

namespace {

// The linear layer after argument checks: GEMV for M <= 16, tcgen05 GEMM above.
cudaError_t run_linear(const DeviceState& st, const void* X_bf16, int64_t M, const uint32_t* qweight,
                       const void* scales_fp16, const void* zeros_fp16, int64_t d_out, int64_t d_in,
                       int32_t group_size, int32_t symmetric, void* Y, int32_t y_dtype, cudaStream_t s) {
    LaunchOptions opt;
    opt.pdl = pdl_enabled();
    if (M <= 16) {
        GemvArgs a = {};
        a.X = X_bf16;
        a.scales = static_cast<const uint16_t*>(scales_fp16);
        a.zeros = static_cast<const uint16_t*>(zeros_fp16);
        a.Y = Y;
        a.status = st.status;
        a.M = (int)M;
        a.N = (int)d_out;
        a.K = (int)d_in;
        a.g = group_size;
        a.G = (int)(d_in / group_size);
        a.g_shift = -1;
        for (int sh = 0; sh < 31; ++sh)
            if ((1 << sh) == group_size) a.g_shift = sh;
        a.symmetric = symmetric;
        a.y_fp32 = y_dtype == WQ_OUT_FP32;
        return launch_gemv(qweight, a, st.num_sms, opt, s);
    }
    GemmArgs a = {};
    a.X = X_bf16;
    a.qweight = qweight;
    a.scales = static_cast<const uint16_t*>(scales_fp16);
    a.zeros = static_cast<const uint16_t*>(zeros_fp16);
    a.Y = Y;
    a.status = st.status;
    a.M = (int)M;
    a.N = (int)d_out;
    a.K = (int)d_in;
    a.g = group_size;
    a.G = (int)(d_in / group_size);
    a.symmetric = symmetric;
    a.y_fp32 = y_dtype == WQ_OUT_FP32;
    a.bits = 4;
    return launch_gemm(a, st.num_sms, opt, s);
}

}  // namespace

wq_status wq_linear_w4a16(const void* X_bf16, int64_t M, const uint32_t* qweight, const void* scales_fp16,
                          const void* zeros_fp16, int64_t d_out, int64_t d_in, int32_t group_size, int32_t symmetric,
                          void* Y, int32_t y_dtype, void* workspace, size_t workspace_bytes, void* stream) {
    wq_status v = check_artifact(qweight, scales_fp16, zeros_fp16, d_out, d_in, group_size, symmetric);
    if (v != WQ_OK) return v;
    if (!X_bf16 || !Y || !aligned(X_bf16, 16) || !aligned(Y, 16)) return WQ_ERR_INVALID_ARG;
    if (M < 1 || M > (1ll << 31) - 1) return WQ_ERR_INVALID_ARG;
    if (y_dtype != WQ_OUT_BF16 && y_dtype != WQ_OUT_FP32) return WQ_ERR_INVALID_ARG;
    if (workspace_bytes < wq_linear_workspace_bytes(M, d_out, d_in)) return WQ_ERR_INVALID_ARG;
    (void)workspace;
    DeviceState st;
    if ((v = device_state(&st)) != WQ_OK) return v;
    const cudaError_t e = run_linear(st, X_bf16, M, qweight, scales_fp16, zeros_fp16, d_out, d_in, group_size,
                                     symmetric, Y, y_dtype, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// AWQ search
// ---------------------------------------------------------------------------

namespace {

constexpr int kAwqAlphas = 11;

struct AwqWorkspace {
    size_t wp, qa, sa, za, xp, yref, ya, lnm, red, scal, total;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

AwqWorkspace awq_workspace(int64_t N, int64_t K, int64_t T, int64_t g) {
    AwqWorkspace w;
    size_t o = 0;
    const int64_t G = K / g;
    w.wp = o;   o += align256((size_t)(N * K) * 2);
    w.qa = o;   o += align256((size_t)(N * K) / 2);
    w.sa = o;   o += align256((size_t)(N * G) * 2);
    w.za = o;   o += align256((size_t)(N * G) * 2);
    w.xp = o;   o += align256((size_t)(T * K) * 2);
    w.yref = o; o += align256((size_t)(T * N) * 4);
    w.ya = o;   o += align256((size_t)(T * N) * 4);
    w.lnm = o;  o += align256((size_t)K * 8);
    w.red = o;  o += align256((size_t)(awq_loss_partials() + 64) * 8);
    w.scal = o; o += align256((size_t)K * 2);
    w.total = o;
    return w;
}

}  // namespace

size_t wq_awq_workspace_bytes(int64_t d_out, int64_t d_in, int64_t T, int32_t group_size) {
    if (d_out < 1 || d_in < 1 || T < 1 || group_size < 1 || d_in % group_size != 0) return 0;
    return awq_workspace(d_out, d_in, T, group_size).total;
}

wq_status wq_awq_search(const void* W_bf16, int64_t d_out, int64_t d_in, const void* X_bf16, int64_t T,
                        int32_t group_size, int32_t symmetric, uint32_t* qweight, void* scales_fp16,
                        void* zeros_fp16, void* s_bf16, double* losses, int32_t* best, void* workspace,
                        size_t workspace_bytes, void* stream) {
    wq_status v = awq_check_args(W_bf16, d_out, d_in, X_bf16, T, group_size, symmetric, qweight, scales_fp16,
                                 zeros_fp16, s_bf16, losses, best);
    if (v != WQ_OK) return v;
    if (!workspace || !aligned(workspace, 256)) return WQ_ERR_INVALID_ARG;
    const AwqWorkspace L = awq_workspace(d_out, d_in, T, group_size);
    if (workspace_bytes < L.total) return WQ_ERR_INVALID_ARG;
    DeviceState st;
    if ((v = device_state(&st)) != WQ_OK) return v;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint16_t* Wp = reinterpret_cast<uint16_t*>(ws + L.wp);
    uint32_t* qa = reinterpret_cast<uint32_t*>(ws + L.qa);
    uint16_t* sa = reinterpret_cast<uint16_t*>(ws + L.sa);
    uint16_t* za = symmetric ? nullptr : reinterpret_cast<uint16_t*>(ws + L.za);
    uint16_t* Xp = reinterpret_cast<uint16_t*>(ws + L.xp);
    float* Yref = reinterpret_cast<float*>(ws + L.yref);
    float* Ya = reinterpret_cast<float*>(ws + L.ya);
    double* lnm = reinterpret_cast<double*>(ws + L.lnm);
    double* red = reinterpret_cast<double*>(ws + L.red);
    double* mean_ln = red + awq_loss_partials();
    double* loss_buf = losses ? losses : mean_ln + 8;
    int32_t* best_buf = best ? best : reinterpret_cast<int32_t*>(mean_ln + 32);
    uint16_t* sbuf = reinterpret_cast<uint16_t*>(ws + L.scal);
    const uint16_t* W = static_cast<const uint16_t*>(W_bf16);
    const uint16_t* X = static_cast<const uint16_t*>(X_bf16);

    // reference output Y = X W^T on the unquantized weights (fp32 accumulation):
    // the tcgen05 GEMM with bf16 B tiles loaded by TMA
    GemmArgs ga = {};
    ga.X = X;
    ga.qweight = reinterpret_cast<const uint32_t*>(W);
    ga.Y = Yref;
    ga.status = st.status;
    ga.M = (int)T;
    ga.N = (int)d_out;
    ga.K = (int)d_in;
    ga.g = (int)d_in;
    ga.G = 1;
    ga.y_fp32 = 1;
    ga.bits = 16;
    LaunchOptions gopt;
    gopt.pdl = false;
    cudaError_t e = launch_gemm(ga, st.num_sms, gopt, s);
    if (e == cudaSuccess) e = launch_awq_colstats(X, T, d_in, lnm, mean_ln, s);
    for (int i = 0; e == cudaSuccess && i < kAwqAlphas; ++i) {
        e = launch_awq_scale_apply(W, d_out, X, T, d_in, lnm, mean_ln, i, nullptr, sbuf, Wp, Xp, st.num_sms, s);
        if (e == cudaSuccess)
            e = launch_quantize(Wp, d_out, d_in, group_size, symmetric, qa, sa, za, st.status, st.num_sms, s);
        if (e == cudaSuccess)
            e = run_linear(st, Xp, T, qa, sa, za, d_out, d_in, group_size, symmetric, Ya, WQ_OUT_FP32, s);
        if (e == cudaSuccess) e = launch_awq_loss(Yref, Ya, T * d_out, red, loss_buf + i, s);
    }
    if (e == cudaSuccess) e = launch_awq_select(loss_buf, kAwqAlphas, best_buf, s);
    // the kept alpha: its scales and the RTN artifact of W diag(s) into the caller's buffers
    if (e == cudaSuccess)
        e = launch_awq_scale_apply(W, d_out, nullptr, 0, d_in, lnm, mean_ln, 0, best_buf,
                                   static_cast<uint16_t*>(s_bf16), Wp, nullptr, st.num_sms, s);
    if (e == cudaSuccess)
        e = launch_quantize(Wp, d_out, d_in, group_size, symmetric, qweight, static_cast<uint16_t*>(scales_fp16),
                            static_cast<uint16_t*>(zeros_fp16), st.status, st.num_sms, s);
    return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// W8A16
// ---------------------------------------------------------------------------

namespace {

wq_status check_w8_artifact(const void* qweight, const void* scales, int64_t d_out, int64_t d_in, int32_t g) {
    if (!qweight || !scales) return WQ_ERR_INVALID_ARG;
    if (d_out < 1 || d_in < 1 || d_out > (1ll << 31) - 1 || d_in > (1ll << 31) - 1) return WQ_ERR_INVALID_ARG;
    if (d_in % 32 != 0 || g < 32 || g % 32 != 0 || d_in % g != 0) return WQ_ERR_INVALID_ARG;
    if (!aligned(qweight, 16) || !aligned(scales, 2)) return WQ_ERR_INVALID_ARG;
    return WQ_OK;
}

}  // namespace

wq_status wq_quantize_w8(const void* W_bf16, int64_t d_out, int64_t d_in, int32_t group_size, uint32_t* qweight,
                         void* scales_fp16, void* stream) {
    wq_status v = check_w8_artifact(qweight, scales_fp16, d_out, d_in, group_size);
    if (v != WQ_OK) return v;
    if (!W_bf16 || !aligned(W_bf16, 16)) return WQ_ERR_INVALID_ARG;
    DeviceState st;
    if ((v = device_state(&st)) != WQ_OK) return v;
    const cudaError_t e = launch_quantize_w8(W_bf16, d_out, d_in, group_size, qweight,
                                             static_cast<uint16_t*>(scales_fp16), st.status, st.num_sms,
                                             static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

wq_status wq_dequantize_w8(const uint32_t* qweight, const void* scales_fp16, int64_t d_out, int64_t d_in,
                           int32_t group_size, void* W_hat_bf16, void* stream) {
    wq_status v = check_w8_artifact(qweight, scales_fp16, d_out, d_in, group_size);
    if (v != WQ_OK) return v;
    if (!W_hat_bf16 || !aligned(W_hat_bf16, 16)) return WQ_ERR_INVALID_ARG;
    DeviceState st;
    if ((v = device_state(&st)) != WQ_OK) return v;
    const cudaError_t e = launch_dequantize_w8(qweight, static_cast<const uint16_t*>(scales_fp16), d_out, d_in,
                                               group_size, W_hat_bf16, st.num_sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

wq_status wq_linear_w8a16(const void* X_bf16, int64_t M, const uint32_t* qweight, const void* scales_fp16,
                          int64_t d_out, int64_t d_in, int32_t group_size, void* Y, int32_t y_dtype, void* stream) {
    wq_status v = check_w8_artifact(qweight, scales_fp16, d_out, d_in, group_size);
    if (v != WQ_OK) return v;
    if (!X_bf16 || !Y || !aligned(X_bf16, 16) || !aligned(Y, 16)) return WQ_ERR_INVALID_ARG;
    if (M < 1 || M > (1ll << 31) - 1) return WQ_ERR_INVALID_ARG;
    if (y_dtype != WQ_OUT_BF16 && y_dtype != WQ_OUT_FP32) return WQ_ERR_INVALID_ARG;
    DeviceState st;
    if ((v = device_state(&st)) != WQ_OK) return v;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (M <= 16) {
        W8Args a = {};
        a.X = X_bf16;
        a.qweight = qweight;
        a.scales = static_cast<const uint16_t*>(scales_fp16);
        a.Y = Y;
        a.status = st.status;
        a.N = d_out;
        a.K = d_in;
        a.G = d_in / group_size;
        a.M = (int)M;
        a.g = group_size;
        a.y_fp32 = y_dtype == WQ_OUT_FP32;
        e = launch_gemv_w8a16(a, s);
    } else {
        GemmArgs a = {};
        a.X = X_bf16;
        a.qweight = qweight;
        a.scales = static_cast<const uint16_t*>(scales_fp16);
        a.zeros = nullptr;
        a.Y = Y;
        a.status = st.status;
        a.M = (int)M;
        a.N = (int)d_out;
        a.K = (int)d_in;
        a.g = group_size;
        a.G = (int)(d_in / group_size);
        a.symmetric = 1;
        a.y_fp32 = y_dtype == WQ_OUT_FP32;
        a.bits = 8;
        LaunchOptions opt;
        opt.pdl = false;
        e = launch_gemm(a, st.num_sms, opt, s);
    }
    return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

size_t wq_gptq_workspace_bytes(int64_t d_out, int64_t d_in) {
    if (d_out < 1 || d_in < 1) return 0;
    return gptq_workspace_bytes(d_out, d_in);
}

wq_status wq_gptq(const void* W_bf16, int64_t d_out, int64_t d_in, const void* X_bf16, int64_t T, int32_t group_size,
                  int32_t symmetric, int32_t act_order, uint32_t* qweight, void* scales_fp16, void* zeros_fp16,
                  int32_t* perm, void* workspace, size_t workspace_bytes, void* stream) {
    wq_status v = check_artifact(qweight, scales_fp16, zeros_fp16, d_out, d_in, group_size, symmetric);
    if (v != WQ_OK) return v;
    if (!W_bf16 || !X_bf16 || !workspace || !aligned(W_bf16, 16) || !aligned(X_bf16, 16) || !aligned(workspace, 256))
        return WQ_ERR_INVALID_ARG;
    if (T < 1 || T > (1ll << 31) - 1 || (act_order != 0 && act_order != 1)) return WQ_ERR_INVALID_ARG;
    if (perm && !aligned(perm, 4)) return WQ_ERR_INVALID_ARG;
    if (workspace_bytes < gptq_workspace_bytes(d_out, d_in)) return WQ_ERR_INVALID_ARG;
    DeviceState st;
    if ((v = device_state(&st)) != WQ_OK) return v;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // static group parameters: plain RTN of W (its codes are replaced below)
    cudaError_t e = launch_quantize(W_bf16, d_out, d_in, group_size, symmetric, qweight,
                                    static_cast<uint16_t*>(scales_fp16), static_cast<uint16_t*>(zeros_fp16), st.status,
                                    st.num_sms, s);
    if (e == cudaSuccess)
        e = launch_gptq(static_cast<const uint16_t*>(W_bf16), d_out, d_in, static_cast<const uint16_t*>(X_bf16), T,
                        group_size, symmetric, act_order, qweight, static_cast<const uint16_t*>(scales_fp16),
                        static_cast<const uint16_t*>(zeros_fp16), perm, workspace, st.status, s);
    return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

wq_status wq_awq_scale_activations(const void* X_bf16, int64_t T, int64_t d_in, const void* s_bf16, void* Xp_bf16,
                                    void* stream) {
    if (!X_bf16 || !s_bf16 || !Xp_bf16 || !aligned(X_bf16, 16) || !aligned(Xp_bf16, 16) || !aligned(s_bf16, 2))
        return WQ_ERR_INVALID_ARG;
    if (T < 1 || d_in < 8 || d_in % 8 != 0) return WQ_ERR_INVALID_ARG;
    DeviceState st;
    wq_status v = device_state(&st);
    if (v != WQ_OK) return v;
    const cudaError_t e = launch_awq_divide(static_cast<const uint16_t*>(X_bf16), T, d_in,
                                            static_cast<const uint16_t*>(s_bf16), static_cast<uint16_t*>(Xp_bf16),
                                            st.num_sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

wq_status wq_selftest_bounded_wait(uint32_t limit_us, void* stream) {
    if (limit_us < 1 || limit_us > 1000000) return WQ_ERR_INVALID_ARG;
    DeviceState st;
    wq_status v = device_state(&st);
    if (v != WQ_OK) return v;
    cudaError_t e = launch_bounded_wait_selftest(st.status, limit_us, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

wq_status wq_get_device_error(uint32_t* flags, void* stream) {
    DeviceState st;
    wq_status v = device_state(&st);
    if (v != WQ_OK) return v;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t h = 0;
    if (cudaMemcpyAsync(&h, st.status, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return WQ_ERR_CUDA;
    if (cudaMemsetAsync(st.status, 0, sizeof(uint32_t), s) != cudaSuccess) return WQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return WQ_ERR_CUDA;
    if (flags) *flags = h;
    if (h & WQ_DEVFLAG_TIMEOUT) return WQ_ERR_TIMEOUT;
    if (h & WQ_DEVFLAG_NONFINITE) return WQ_ERR_NONFINITE;
    if (h & WQ_DEVFLAG_RANGE) return WQ_ERR_RANGE;
    return WQ_OK;
}

}  // extern "C"
