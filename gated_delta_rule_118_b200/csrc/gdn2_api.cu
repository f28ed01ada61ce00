// gdn2_api.cu -- the C ABI of libgdn2.so: argument checks, the device error
// word, and the launch of the forward and decode kernels on the caller's stream.
#include <cuda_runtime.h>

#include <mutex>
#include <stdint.h>

#include "gdn2.h"
#include "common.cuh"
#include "launch.h"

namespace gdn2 {

// Device-side error word: kernels OR bits into it (kErrTimeout);
// gdn2_check_device_error() reads and clears it.  One per device (module global).
__device__ unsigned int g_device_error = 0;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_init_mutex;
unsigned int *g_err_ptr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

// Address of the error word and the SM count on the current device.
gdn2_status device_context(unsigned int **err, int *num_sms)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDN2_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_init_mutex);
    if (!g_err_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return GDN2_ERR_CUDA;
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return GDN2_ERR_CUDA;
        g_err_ptr[dev] = static_cast<unsigned int *>(p);
        g_num_sms[dev] = sms;
    }
    *err = g_err_ptr[dev];
    *num_sms = g_num_sms[dev];
    return GDN2_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool head_dim_ok(int d) { return d == 64 || d == 128; }

gdn2_status check_dims(int dk, int dv)
{
    if (dk <= 0 || dv <= 0) return GDN2_ERR_SHAPE;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return GDN2_ERR_UNSUPPORTED;
    return GDN2_OK;
}

}  // namespace

// Device address of the error word on the current device (for other entry points).
bool device_error_word(unsigned int **err)
{
    int sms = 0;
    return device_context(err, &sms) == GDN2_OK;
}

}  // namespace gdn2

using namespace gdn2;

namespace {

constexpr unsigned kLayoutBits = GDN2_ERASE_SCALAR | GDN2_WRITE_SCALAR | GDN2_DECAY_SCALAR;

// The chunked forward; with `epi` (gdn2_layer_fwd) the inputs are the layer's
// raw ones and the outputs get the layer's RMS norm and output gate.
struct LayerEpi {
    const void *g;
    const float *weight;
    float eps;
};

gdn2_status fwd_chunked(const void *q, const void *k, const void *v, const void *b, const void *w,
                        const float *log_alpha, const float *S0, void *o, float *S_T, int B, int T, int H, int dk,
                        int dv, gdn2_dtype dtype, unsigned layout, gdn2_stream_t stream,
                        const LayerEpi *epi = nullptr)
{
    if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_DTYPE;
    if (B <= 0 || H <= 0 || T < 0) return GDN2_ERR_SHAPE;
    if (layout & ~kLayoutBits) return GDN2_ERR_UNSUPPORTED;
    gdn2_status st = check_dims(dk, dv);
    if (st != GDN2_OK) return st;
    if (B > 65535 || H > 65535) return GDN2_ERR_UNSUPPORTED;  // grid y/z limits
    const void *ins[] = {q, k, v, b, w, log_alpha, o, epi ? epi->g : q, epi ? epi->weight : q};
    if (T > 0)
        for (const void *p : ins)
            if (!p) return GDN2_ERR_NULL;
    const void *all[] = {q, k, v, b, w, log_alpha, o, S0, S_T, epi ? epi->g : nullptr, epi ? epi->weight : nullptr};
    for (const void *p : all)
        if (p && !aligned16(p)) return GDN2_ERR_ALIGN;
    if (epi && !(epi->eps >= 0.f)) return GDN2_ERR_SHAPE;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) {  // nothing to run: S_T = S0 (or zeros)
        if (!S_T) return GDN2_OK;
        const size_t bytes = sizeof(float) * (size_t)B * H * dk * dv;
        cudaError_t e = S0 ? (S0 == S_T ? cudaSuccess
                                        : cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, s))
                           : cudaMemsetAsync(S_T, 0, bytes, s);
        return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
    }

    FwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.b = b; a.w = w; a.log_alpha = log_alpha;
    a.S0 = S0; a.o = o; a.S_T = S_T;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv;
    a.bf16 = (dtype == GDN2_BF16);
    a.layout = layout;
    a.stream = s;
    if (epi) {
        a.layout |= kLayerInputsBit;
        a.g = epi->g;
        a.norm_weight = epi->weight;
        a.eps = epi->eps;
    }
    st = device_context(&a.err, &a.num_sms);
    if (st != GDN2_OK) return st;
    // bf16 inputs with dk = 128 run on the tensor cores (the output processing
    // inside the output work); fp32 inputs (and dk = 64) run on the fp32 pipes,
    // which meet the fp32 tolerance, with the output processing as a row kernel.
    cudaError_t e;
    if (a.bf16 && dk == 128) {
        e = launch_fwd_tc(a);
    } else {
        e = launch_fwd_simt(a);
        if (e == cudaSuccess && epi) e = launch_layer_epilogue_rows(a);
    }
    return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

gdn2_status decode(const void *q, const void *k, const void *v, const void *b, const void *w,
                   const float *log_alpha, float *S, void *o, int B, int T, int H, int dk, int dv,
                   gdn2_dtype dtype, unsigned layout, gdn2_stream_t stream)
{
    if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_DTYPE;
    if (B <= 0 || H <= 0 || T <= 0) return GDN2_ERR_SHAPE;
    if (layout & ~kLayoutBits) return GDN2_ERR_UNSUPPORTED;
    gdn2_status st = check_dims(dk, dv);
    if (st != GDN2_OK) return st;
    if ((long long)B * H > 0x7fffffffLL) return GDN2_ERR_UNSUPPORTED;  // grid x limit
    const void *all[] = {q, k, v, b, w, log_alpha, S, o};
    for (const void *p : all) {
        if (!p) return GDN2_ERR_NULL;
        if (!aligned16(p)) return GDN2_ERR_ALIGN;
    }
    DecodeArgs a{};
    a.q = q; a.k = k; a.v = v; a.b = b; a.w = w; a.log_alpha = log_alpha;
    a.S = S; a.o = o; a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv;
    a.bf16 = (dtype == GDN2_BF16);
    a.layout = layout;
    a.stream = reinterpret_cast<cudaStream_t>(stream);
    return launch_decode(a) == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

}  // namespace

extern "C" gdn2_status gdn2_fwd_chunked(const void *q, const void *k, const void *v,
                                        const void *b, const void *w, const float *log_alpha,
                                        const float *S0, void *o, float *S_T,
                                        int B, int T, int H, int dk, int dv,
                                        gdn2_dtype dtype, gdn2_stream_t stream)
{
    return fwd_chunked(q, k, v, b, w, log_alpha, S0, o, S_T, B, T, H, dk, dv, dtype, 0u, stream);
}

extern "C" gdn2_status gdn2_fwd_chunked_gates(const void *q, const void *k, const void *v,
                                              const void *b, const void *w, const float *log_alpha,
                                              const float *S0, void *o, float *S_T,
                                              int B, int T, int H, int dk, int dv,
                                              gdn2_dtype dtype, unsigned int layout, gdn2_stream_t stream)
{
    return fwd_chunked(q, k, v, b, w, log_alpha, S0, o, S_T, B, T, H, dk, dv, dtype, layout, stream);
}

extern "C" gdn2_status gdn2_layer_fwd(const void *q, const void *k, const void *v, const void *b_logit,
                                      const void *w_logit, const float *decay_logit, const void *g_logit,
                                      const float *norm_weight, float eps, const float *S0, void *y, float *S_T,
                                      int B, int T, int H, int dk, int dv, gdn2_dtype dtype,
                                      gdn2_stream_t stream)
{
    const LayerEpi epi{g_logit, norm_weight, eps};
    return fwd_chunked(q, k, v, b_logit, w_logit, decay_logit, S0, y, S_T, B, T, H, dk, dv, dtype, 0u, stream,
                       &epi);
}

extern "C" gdn2_status gdn2_bwd_chunked(const void *q, const void *k, const void *v, const void *b, const void *w,
                                        const float *log_alpha, const float *S0, const void *dO,
                                        const float *dS_T, float *dq, float *dk_, float *dv_, float *db, float *dw,
                                        float *dlog_alpha, float *dS0, int B, int T, int H, int dk, int dv,
                                        gdn2_dtype dtype, gdn2_stream_t stream)
{
    if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_DTYPE;
    if (B <= 0 || H <= 0 || T < 0) return GDN2_ERR_SHAPE;
    gdn2_status st = check_dims(dk, dv);
    if (st != GDN2_OK) return st;
    if (B > 65535 || H > 65535) return GDN2_ERR_UNSUPPORTED;
    const void *req[] = {q, k, v, b, w, log_alpha, dO, dq, dk_, dv_, db, dw, dlog_alpha};
    if (T > 0)
        for (const void *p : req)
            if (!p) return GDN2_ERR_NULL;
    const void *all[] = {q, k, v, b, w, log_alpha, dO, dq, dk_, dv_, db, dw, dlog_alpha, S0, dS_T, dS0};
    for (const void *p : all)
        if (p && !aligned16(p)) return GDN2_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t DD = sizeof(float) * (size_t)dk * dv;
    if (T == 0) {  // o is empty and S_T = S0: dS0 = dS_T
        if (!dS0) return GDN2_OK;
        cudaError_t e = dS_T ? cudaMemcpyAsync(dS0, dS_T, DD * B * H, cudaMemcpyDeviceToDevice, s)
                             : cudaMemsetAsync(dS0, 0, DD * B * H, s);
        return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN2_ERR_CUDA;
    cudaMemPool_t pool = workspace_pool(dev);
    if (!pool) return GDN2_ERR_CUDA;
    // bf16 inputs with dk = 128 run on the tensor cores (workspace: the prep
    // records with T and P (and T - bf16(T) where T is far from the identity),
    // and the state and dS' images of every chunk); fp32
    // inputs and dk = 64 on the fp32 pipes (per chunk: T and P, the state
    // entering it, U, dU and the adjoint at its end)
    const bool tc = dtype == GDN2_BF16 && dk == 128;
    unsigned int *err = nullptr;
    int num_sms = 0;
    if (tc && device_context(&err, &num_sms) != GDN2_OK) return GDN2_ERR_CUDA;
    const size_t ws_bytes = tc ? bwd_tc_workspace_bytes(B, T, H, dv) : sizeof(float) * bwd_workspace_floats(B, T, H, dk, dv);
    void *ws = nullptr;
    cudaError_t e = cudaMallocFromPoolAsync(&ws, ws_bytes, pool, s);
    if (e != cudaSuccess) return GDN2_ERR_CUDA;
    BwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.b = b; a.w = w; a.log_alpha = log_alpha; a.S0 = S0;
    a.dO = dO; a.dS_T = dS_T; a.ws = tc ? nullptr : static_cast<float *>(ws);
    a.gq = dq; a.gk = dk_; a.gv = dv_; a.gb = db; a.gw = dw; a.gla = dlog_alpha; a.dS0 = dS0;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv;
    a.bf16 = (dtype == GDN2_BF16);
    a.stream = s;
    e = tc ? launch_bwd_tc(a, static_cast<uint8_t *>(ws), err, num_sms) : launch_bwd_simt(a);
    const cudaError_t fe = cudaFreeAsync(ws, s);
    return (e == cudaSuccess && fe == cudaSuccess) ? GDN2_OK : GDN2_ERR_CUDA;
}

extern "C" gdn2_status gdn2_decode_step(const void *q, const void *k, const void *v,
                                        const void *b, const void *w, const float *log_alpha,
                                        float *S, void *o, int B, int H, int dk, int dv,
                                        gdn2_dtype dtype, gdn2_stream_t stream)
{
    return decode(q, k, v, b, w, log_alpha, S, o, B, 1, H, dk, dv, dtype, 0u, stream);
}

extern "C" gdn2_status gdn2_decode_tokens(const void *q, const void *k, const void *v,
                                          const void *b, const void *w, const float *log_alpha,
                                          float *S, void *o, int B, int T, int H, int dk, int dv,
                                          gdn2_dtype dtype, unsigned int layout, gdn2_stream_t stream)
{
    return decode(q, k, v, b, w, log_alpha, S, o, B, T, H, dk, dv, dtype, layout, stream);
}

extern "C" gdn2_status gdn2_check_device_error(gdn2_stream_t stream)
{
    unsigned int *err = nullptr;
    int sms = 0;
    if (device_context(&err, &sms) != GDN2_OK) return GDN2_ERR_CUDA;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return GDN2_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpy(&word, err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return GDN2_ERR_CUDA;
    if (word && cudaMemset(err, 0, sizeof(word)) != cudaSuccess) return GDN2_ERR_CUDA;
    if (word & kErrTimeout) return GDN2_ERR_DEVICE_TIMEOUT;
    return GDN2_OK;
}

extern "C" gdn2_status gdn2_selftest_bounded_wait(gdn2_stream_t stream)
{
    unsigned int *err = nullptr;
    int sms = 0;
    if (device_context(&err, &sms) != GDN2_OK) return GDN2_ERR_CUDA;
    return launch_selftest_wait(reinterpret_cast<cudaStream_t>(stream), err) == cudaSuccess ? GDN2_OK
                                                                                            : GDN2_ERR_CUDA;
}

extern "C" int gdn2_fwd_chunked_launches(int B, int T, int H, int dk, int dv, gdn2_dtype dtype)
{
    if ((dtype != GDN2_F32 && dtype != GDN2_BF16) || B <= 0 || H <= 0 || T < 0) return -1;
    if (check_dims(dk, dv) != GDN2_OK || B > 65535 || H > 65535) return -1;
    if (T == 0) return 0;
    if (dtype == GDN2_BF16 && dk == 128) {
        // the window plan depends on the SM count of the current device (none: plan for 148)
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            sms = 0;
            cudaGetLastError();
        }
        if (sms <= 0) sms = 148;
        if (plan_fwd_persist(B, T, H, dv, sms).use) return 1;
        // per window: prep and chain with the outputs (wide batches), or prep, chain and outputs
        const FwdTcPlan p = plan_fwd_tc(B, T, H, dv, kWindowBudgetBytes, sms);
        return (p.overlap ? 3 : 2) * p.nwindows;
    }
    return 1;
}

extern "C" const char *gdn2_status_string(gdn2_status status)
{
    switch (status) {
    case GDN2_OK: return "GDN2_OK";
    case GDN2_ERR_NULL: return "GDN2_ERR_NULL: a required pointer is NULL";
    case GDN2_ERR_SHAPE: return "GDN2_ERR_SHAPE: a size is out of range";
    case GDN2_ERR_DTYPE: return "GDN2_ERR_DTYPE: unknown dtype code";
    case GDN2_ERR_ALIGN: return "GDN2_ERR_ALIGN: a pointer is not 16-byte aligned";
    case GDN2_ERR_UNSUPPORTED: return "GDN2_ERR_UNSUPPORTED: request outside the implemented set";
    case GDN2_ERR_CUDA: return "GDN2_ERR_CUDA: a CUDA runtime call or launch failed";
    case GDN2_ERR_DEVICE_TIMEOUT: return "GDN2_ERR_DEVICE_TIMEOUT: a device-side bounded wait gave up";
    case GDN2_ERR_RANGE: return "GDN2_ERR_RANGE: reserved (no longer reported)";
    case GDN2_ERR_SCRATCH_LIMIT: return "GDN2_ERR_SCRATCH_LIMIT: the problem needs more than the fixed scratch buffer";
    }
    return "GDN2 unknown status";
}
