// fwd_noalloc.cu -- gdn2_fwd_chunked_noalloc: the chunked forward with no
// device allocation at all.
//
// gdn2_fwd_chunked draws the workspace of its bf16 tensor-core path (the
// per-chunk prep records, the exported state images and the state carried
// between windows) from a stream-ordered memory pool.  Some callers cannot let
// a library allocate: a runtime that hands out all device memory itself at
// start-up, code that must never enter the driver's allocator on its hot loop
// (allocation can block, or fail when memory is fragmented), or a process that
// has to know its full device footprint before it runs.  This entry point
// gives them the same computation with the workspace in a fixed buffer that
// lives in this library's device image: `g_noalloc_scratch` below.
//
// The buffer holds kNoAllocScratchBytes on every GPU that loads the library,
// until the process exits.  The sequence is processed in as many windows as
// it takes to fit the buffer; a problem whose single chunk-column (all batch x
// head records of one chunk, plus the carried state) does not fit is rejected
// with GDN2_ERR_SCRATCH_LIMIT before anything is launched.
#include <cuda_runtime.h>

#include <mutex>
#include <stdint.h>

#include "gdn2.h"
#include "launch.h"
#include "tc_common.cuh"

namespace gdn2 {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB per device

// The workspace.  In host code this name is only a stand-in for the device
// symbol: its device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint8_t *g_scratch[kMaxDevices] = {};

// Device address of the scratch buffer, looked up the first time this entry
// point runs on the current device (with that device current), and the
// device error word.
gdn2_status noalloc_setup(uint8_t **scratch, unsigned int **err)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDN2_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_scratch[dev]) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GDN2_ERR_CUDA;
            g_scratch[dev] = static_cast<uint8_t *>(p);
        }
        *scratch = g_scratch[dev];
    }
    return device_error_word(err) ? GDN2_OK : GDN2_ERR_CUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool head_dim_ok(int d) { return d == 64 || d == 128; }

}  // namespace
}  // namespace gdn2

using namespace gdn2;

extern "C" gdn2_status gdn2_fwd_chunked_noalloc(const void *q, const void *k, const void *v, const void *b,
                                                const void *w, const float *log_alpha, const float *S0, void *o,
                                                float *S_T, int B, int T, int H, int dk, int dv,
                                                gdn2_dtype dtype, gdn2_stream_t stream)
{
    if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_DTYPE;
    if (B <= 0 || H <= 0 || T < 0 || dk <= 0 || dv <= 0) return GDN2_ERR_SHAPE;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return GDN2_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535) return GDN2_ERR_UNSUPPORTED;
    const void *ins[] = {q, k, v, b, w, log_alpha, o};
    if (T > 0)
        for (const void *p : ins)
            if (!p) return GDN2_ERR_NULL;
    const void *all[] = {q, k, v, b, w, log_alpha, o, S0, S_T};
    for (const void *p : all)
        if (p && !aligned16(p)) return GDN2_ERR_ALIGN;

    const bool tensor_cores = (dtype == GDN2_BF16 && dk == 128);
    FwdTcPlan plan{};
    if (tensor_cores && T > 0) {
        // Records of as many chunks as fit, after room for the carried state.
        const size_t carry = (size_t)B * H * 128 * dv * sizeof(float);
        const size_t rec = (dv == 128) ? Record<128>::BYTES : Record<64>::BYTES;
        const size_t sx = (dv == 128) ? SxSlot<128>::BYTES : SxSlot<64>::BYTES;
        const size_t per_chunk = (size_t)B * H * (rec + sx);
        if (carry >= kNoAllocScratchBytes || per_chunk > kNoAllocScratchBytes - carry) return GDN2_ERR_SCRATCH_LIMIT;
        plan = plan_fwd_tc(B, T, H, dv, kNoAllocScratchBytes - carry, 0);
        if (plan.ws_bytes > kNoAllocScratchBytes) return GDN2_ERR_SCRATCH_LIMIT;
    }

    uint8_t *scratch = nullptr;
    unsigned int *errword = nullptr;
    gdn2_status st = noalloc_setup(&scratch, &errword);
    if (st != GDN2_OK) return st;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) {
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
    a.stream = s;
    a.err = errword;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return GDN2_ERR_CUDA;
    a.num_sms = sms;
    const cudaError_t e = tensor_cores ? run_fwd_tc(a, plan, scratch) : launch_fwd_simt(a);
    return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}
