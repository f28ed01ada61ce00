// fwd_tc.cu -- host orchestration of the bf16 tensor-core forward.
//
// The forward of a sequence is split into its state-independent part (the
// prep kernel, fully parallel over (batch, head, chunk)) and its state-carrying
// part (the chain kernel, one CTA per (batch, head, value tile) walking the
// chunks in order).  Prep records travel through a workspace in device memory.
// The sequence is processed in windows of WC chunks so that the workspace of
// one window stays small enough to live in L2 between the kernels; the state
// crosses window boundaries through a carry buffer (or S_T / S0).  The
// allocating entry point overlaps the windows on internal streams; the
// no-allocation entry point runs them in order on the caller's stream.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "launch.h"
#include "tc_common.cuh"

namespace gdn2 {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 4-D map over a [B][T][H][d] tensor: dims (d, H, T, B), box (box_d, 1, 64, 1).
bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, int d, int H, int T, int B,
              int box_d, CUtensorMapSwizzle swz)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * esize, (cuuint64_t)H * d * esize, (cuuint64_t)T * H * d * esize};
    cuuint32_t box[4] = {(cuuint32_t)box_d, 1, 64, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, dt, 4, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Stream-ordered pool for the workspace; it keeps freed blocks for reuse.
cudaMemPool_t workspace_pool(int dev)
{
    static std::mutex mu;
    static cudaMemPool_t pools[64] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return nullptr;
    if (!pools[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t p = nullptr;
        if (cudaMemPoolCreate(&p, &props) != cudaSuccess) return nullptr;
        uint64_t keep = ~0ull;
        cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
        pools[dev] = p;
    }
    return pools[dev];
}

}  // namespace

FwdTcPlan plan_fwd_tc(int B, int T, int H, int dv, size_t window_budget)
{
    FwdTcPlan p{};
    const long bh = (long)B * H;
    // The serial chain costs about the same per UMMA instruction for 64 and 128
    // columns; 64-wide tiles halve each thread's epilogue when SMs are plentiful.
    p.dvt = (dv == 64 || bh * 2 <= 148) ? 64 : 128;
    p.nchunks = (T + kChunk - 1) / kChunk;
    p.rec_bytes = (dv == 128) ? Record<128>::BYTES : Record<64>::BYTES;
    p.sx_bytes = (dv == 128) ? SxSlot<128>::BYTES : SxSlot<64>::BYTES;
    const size_t per_chunk = (size_t)bh * (p.rec_bytes + p.sx_bytes);
    long wc = per_chunk ? (long)(window_budget / per_chunk) : 0;
    if (wc < 1) wc = 1;
    if (wc > p.nchunks) wc = p.nchunks;
    p.wc = (int)wc;
    p.nwindows = p.nchunks ? (p.nchunks + p.wc - 1) / p.wc : 0;
    p.rec_total = (size_t)p.wc * bh * p.rec_bytes;
    p.sx_total = (size_t)p.wc * bh * p.sx_bytes;
    p.carry_bytes = p.nwindows > 1 ? (size_t)bh * 128 * dv * sizeof(float) : 0;
    p.ws_bytes = p.rec_total + p.sx_total + p.carry_bytes;
    return p;
}

cudaError_t run_fwd_tc(const FwdArgs &a, const FwdTcPlan &p, uint8_t *ws)
{
    CUtensorMap maps[6];
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!make_map(&maps[0], a.q, BF, 2, 128, a.H, a.T, a.B, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&maps[1], a.k, BF, 2, 128, a.H, a.T, a.B, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&maps[2], a.b, BF, 2, 128, a.H, a.T, a.B, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&maps[3], a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 128, a.H, a.T, a.B, 128,
                  CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&maps[4], a.v, BF, 2, a.dv, a.H, a.T, a.B, a.dv, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&maps[5], a.w, BF, 2, a.dv, a.H, a.T, a.B, a.dv, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    uint8_t *recs = ws, *sxs = ws + p.rec_total;
    float *carry = p.carry_bytes ? reinterpret_cast<float *>(ws + p.rec_total + p.sx_total) : nullptr;
    for (int w = 0; w < p.nwindows; ++w) {
        const int c0 = w * p.wc;
        const int ncw = (p.nchunks - c0 < p.wc) ? p.nchunks - c0 : p.wc;
        const float *S_in = (w == 0) ? a.S0 : carry;
        float *S_out = (w == p.nwindows - 1) ? a.S_T : carry;
        cudaError_t e = launch_prep(a, maps, recs, c0, ncw, p.wc, false);
        if (e == cudaSuccess) e = launch_chain(a, p.dvt, recs, sxs, S_in, S_out, ncw, p.wc);
        if (e == cudaSuccess) e = launch_out(a, recs, sxs, c0, ncw, p.wc, false);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

namespace {

// Streams and events of the overlapped schedule, one set per device, created on
// first use and kept for the life of the process.  The chain stream has the
// highest priority so that its CTAs are dispatched ahead of pending prep CTAs.
struct StreamSet {
    std::mutex mu;
    cudaStream_t prep = nullptr, chain = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, ev_p[4] = {}, ev_c[4] = {}, ev_o[4] = {};
    bool ready = false;
};

StreamSet *stream_set(int dev)
{
    static StreamSet sets[64];
    if (dev < 0 || dev >= 64) return nullptr;
    StreamSet &ss = sets[dev];
    std::lock_guard<std::mutex> lock(ss.mu);
    if (!ss.ready) {
        int lo = 0, hi = 0;
        if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) return nullptr;
        if (cudaStreamCreateWithPriority(&ss.chain, cudaStreamNonBlocking, hi) != cudaSuccess ||
            cudaStreamCreateWithFlags(&ss.prep, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&ss.out, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&ss.start, cudaEventDisableTiming) != cudaSuccess)
            return nullptr;
        for (int i = 0; i < 4; ++i)
            if (cudaEventCreateWithFlags(&ss.ev_p[i], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&ss.ev_c[i], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&ss.ev_o[i], cudaEventDisableTiming) != cudaSuccess)
                return nullptr;
        ss.ready = true;
    }
    return &ss;
}

// Overlapped schedule over two workspace halves (window w uses half w % 2):
//   prep stream:   [wait chain(w-2), out(w-2)]  prep(w)  -> ev_p[w]
//   chain stream:  [wait prep(w)]               chain(w) -> ev_c[w]
//   out stream:    [wait chain(w)]              out(w)   -> ev_o[w]
// so prep of the next window runs while the chain walks the current one.  The
// caller's stream forks into the three at the start and joins them at the end.
cudaError_t run_fwd_tc_overlapped(const FwdArgs &a, const FwdTcPlan &p, uint8_t *ws, StreamSet &ss)
{
    CUtensorMap maps[6];
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!make_map(&maps[0], a.q, BF, 2, 128, a.H, a.T, a.B, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&maps[1], a.k, BF, 2, 128, a.H, a.T, a.B, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&maps[2], a.b, BF, 2, 128, a.H, a.T, a.B, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&maps[3], a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 128, a.H, a.T, a.B, 128,
                  CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&maps[4], a.v, BF, 2, a.dv, a.H, a.T, a.B, a.dv, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&maps[5], a.w, BF, 2, a.dv, a.H, a.T, a.B, a.dv, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const size_t half = p.rec_total + p.sx_total;
    float *carry = p.carry_bytes ? reinterpret_cast<float *>(ws + 2 * half) : nullptr;
    cudaError_t e = cudaEventRecord(ss.start, a.stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss.prep, ss.start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss.chain, ss.start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss.out, ss.start, 0);
    for (int w = 0; w < p.nwindows && e == cudaSuccess; ++w) {
        const int c0 = w * p.wc, slot = w & 3;
        const int ncw = (p.nchunks - c0 < p.wc) ? p.nchunks - c0 : p.wc;
        uint8_t *recs = ws + (w & 1) * half, *sxs = recs + p.rec_total;
        const float *S_in = (w == 0) ? a.S0 : carry;
        float *S_out = (w == p.nwindows - 1) ? a.S_T : carry;
        FwdArgs ap = a, ac = a, ao = a;
        ap.stream = ss.prep;
        ac.stream = ss.chain;
        ao.stream = ss.out;
        if (w >= 2) {
            e = cudaStreamWaitEvent(ss.prep, ss.ev_c[(w - 2) & 3], 0);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(ss.prep, ss.ev_o[(w - 2) & 3], 0);
        }
        // prep and output launches of consecutive windows touch disjoint data, so
        // each may start while the previous one of its stream drains
        if (e == cudaSuccess) e = launch_prep(ap, maps, recs, c0, ncw, p.wc, true);
        if (e == cudaSuccess) e = cudaEventRecord(ss.ev_p[slot], ss.prep);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(ss.chain, ss.ev_p[slot], 0);
        if (e == cudaSuccess) e = launch_chain(ac, p.dvt, recs, sxs, S_in, S_out, ncw, p.wc);
        if (e == cudaSuccess) e = cudaEventRecord(ss.ev_c[slot], ss.chain);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(ss.out, ss.ev_c[slot], 0);
        if (e == cudaSuccess) e = launch_out(ao, recs, sxs, c0, ncw, p.wc, true);
        if (e == cudaSuccess) e = cudaEventRecord(ss.ev_o[slot], ss.out);
    }
    // join: the caller's stream waits for the last chain and the last two outputs
    if (e == cudaSuccess && p.nwindows > 0) {
        const int last = p.nwindows - 1;
        e = cudaStreamWaitEvent(a.stream, ss.ev_c[last & 3], 0);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(a.stream, ss.ev_o[last & 3], 0);
        if (e == cudaSuccess && last >= 1) e = cudaStreamWaitEvent(a.stream, ss.ev_o[(last - 1) & 3], 0);
    }
    return e;
}

}  // namespace

cudaError_t launch_fwd_tc(const FwdArgs &a)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    cudaMemPool_t pool = workspace_pool(dev);
    StreamSet *ss = stream_set(dev);
    if (!pool || !ss) return cudaErrorMemoryAllocation;
    // two window halves of half the budget each
    FwdTcPlan p = plan_fwd_tc(a.B, a.T, a.H, a.dv, kWindowBudgetBytes / 2);
    const size_t bytes = 2 * (p.rec_total + p.sx_total) + p.carry_bytes;
    void *ws = nullptr;
    e = cudaMallocFromPoolAsync(&ws, bytes, pool, a.stream);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> lock(ss->mu);
        e = run_fwd_tc_overlapped(a, p, static_cast<uint8_t *>(ws), *ss);
    }
    const cudaError_t f = cudaFreeAsync(ws, a.stream);
    return e != cudaSuccess ? e : f;
}

}  // namespace gdn2
