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

#include "gdn2.h"
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
}  // namespace

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

bool make_token_map(CUtensorMap *m, const void *base, int d, int H, int T, int B)
{
    return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, H, T, B, 64, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Tensor maps of the TMA-loaded inputs: q, k, b, log_alpha and the output-gate
// logits of the fused layer.  A gate given as one value per (token, head), and
// an absent output gate, are not loaded by TMA; their slots hold q's map, which
// the kernels do not use for them.
bool make_input_maps(const FwdArgs &a, CUtensorMap *maps)
{
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!make_map(&maps[0], a.q, BF, 2, 128, a.H, a.T, a.B, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&maps[1], a.k, BF, 2, 128, a.H, a.T, a.B, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return false;
    maps[2] = maps[3] = maps[4] = maps[0];
    if (!(a.layout & GDN2_ERASE_SCALAR) &&
        !make_map(&maps[2], a.b, BF, 2, 128, a.H, a.T, a.B, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return false;
    if (!(a.layout & GDN2_DECAY_SCALAR) &&
        !make_map(&maps[3], a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 128, a.H, a.T, a.B, 128,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
        return false;
    return !a.g || make_map(&maps[4], a.g, BF, 2, a.dv, a.H, a.T, a.B, 64, CU_TENSOR_MAP_SWIZZLE_128B);
}

FwdTcPlan plan_fwd_tc(int B, int T, int H, int dv, size_t budget, int num_sms)
{
    FwdTcPlan p{};
    const long bh = (long)B * H;
    // The serial chain costs about the same per UMMA instruction for 64 and 128
    // columns; 64-wide tiles halve each thread's epilogue when SMs are plentiful.
    p.dvt = (dv == 64 || bh * 2 <= 148) ? 64 : 128;
    p.nchunks = (T + kChunk - 1) / kChunk;
    p.rec_bytes = (dv == 128) ? Record<128>::BYTES : Record<64>::BYTES;
    p.sx_bytes = (dv == 128) ? SxSlot<128>::BYTES : SxSlot<64>::BYTES;
    // A chain CTA takes a whole SM.  When the chain leaves at least half of the
    // SMs, a window's prep runs beside the previous window's chain (four windows
    // in flight); otherwise prep and chain take turns on the whole GPU (two).
    const long chain_ctas = bh * (dv / p.dvt);
    p.overlap = num_sms > 0 && chain_ctas * 2 <= num_sms;
    p.slots = num_sms > 0 ? (p.overlap ? kWindowSlots : 2) : 1;
    if (num_sms > 0) budget = p.overlap ? kWindowBudgetBytes : kWideWindowBudgetBytes;
    const size_t per_chunk = (size_t)bh * (p.rec_bytes + p.sx_bytes);
    long wc = per_chunk ? (long)(budget / p.slots / per_chunk) : 0;
    // beside the chain, a window whose prep CTAs (two per SM) fit the other SMs in
    // one wave keeps the chain from waiting for a second wave
    if (p.overlap) {
        const long cap = 2 * (num_sms - chain_ctas) / bh;
        if (cap >= 1 && wc > cap) wc = cap;
    }
    if (wc < 1) wc = 1;
    if (wc > p.nchunks) wc = p.nchunks;
    p.wc = (int)wc;
    p.nwindows = p.nchunks ? (p.nchunks + p.wc - 1) / p.wc : 0;
    if (num_sms > 0 && p.nwindows > 0 && p.slots > p.nwindows) p.slots = p.nwindows;  // no idle slots
    p.rec_total = (size_t)p.wc * bh * p.rec_bytes;
    p.sx_total = (size_t)p.wc * bh * p.sx_bytes;
    p.carry_bytes = p.nwindows > 1 ? (size_t)bh * 128 * dv * sizeof(float) : 0;
    p.ws_bytes = p.slots * (p.rec_total + p.sx_total) + p.carry_bytes;
    return p;
}

cudaError_t run_fwd_tc(const FwdArgs &a, const FwdTcPlan &p, uint8_t *ws)
{
    CUtensorMap maps[5];
    if (!make_input_maps(a, maps)) return cudaErrorInvalidValue;
    uint8_t *recs = ws, *sxs = ws + p.rec_total;
    float *carry = p.carry_bytes ? reinterpret_cast<float *>(ws + p.rec_total + p.sx_total) : nullptr;
    for (int w = 0; w < p.nwindows; ++w) {
        const int c0 = w * p.wc;
        const int ncw = (p.nchunks - c0 < p.wc) ? p.nchunks - c0 : p.wc;
        const float *S_in = (w == 0) ? a.S0 : carry;
        float *S_out = (w == p.nwindows - 1) ? a.S_T : carry;
        cudaError_t e = launch_prep(a, maps, recs, c0, ncw, p.wc, false);
        if (e == cudaSuccess) e = launch_chain(a, p.dvt, recs, sxs, S_in, S_out, ncw, p.wc, false);
        if (e == cudaSuccess) e = launch_out(a, &maps[4], recs, sxs, c0, ncw, p.wc, false);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

namespace {

// The output stream and the events of the overlapped schedule, one set per
// device, created on first use and kept for the life of the process.
struct StreamSet {
    std::mutex mu;
    cudaStream_t out = nullptr;
    cudaEvent_t start = nullptr, ev_c[kWindowSlots] = {}, ev_o[kWindowSlots] = {};
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
        // lowest priority: the caller's stream (prep and chain) goes first
        if (cudaStreamCreateWithPriority(&ss.out, cudaStreamNonBlocking, lo) != cudaSuccess ||
            cudaEventCreateWithFlags(&ss.start, cudaEventDisableTiming) != cudaSuccess)
            return nullptr;
        for (int i = 0; i < kWindowSlots; ++i)
            if (cudaEventCreateWithFlags(&ss.ev_c[i], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&ss.ev_o[i], cudaEventDisableTiming) != cudaSuccess)
                return nullptr;
        ss.ready = true;
    }
    return &ss;
}

// Overlapped schedule over p.slots workspace slots (window w uses slot w % p.slots).
// A chain CTA needs a whole SM, so the chain of a window must not queue behind
// prep CTAs of later windows.  The caller's stream therefore carries
//   prep(0), chain(0), prep(1), chain(1), ...
// With p.overlap, prep(w + 1) is a programmatic dependent of chain(w): it starts
// once every chain CTA of window w is resident and fills the other SMs while the
// chain walks window w; chain(w + 1) starts when both are done.  Without it
// (a chain that takes most SMs) prep and chain take turns.  The output kernels
// run on their own stream, each after its window's chain:
//   out stream:    [wait ev_c[w]]  out(w) -> ev_o[w]
// and before chain(w) the caller's stream waits for the output kernel that last
// used the slot prep(w + 1) is about to overwrite.  The output stream forks from
// the caller's stream at the start and joins it at the end.
cudaError_t run_fwd_tc_overlapped(const FwdArgs &a, const FwdTcPlan &p, uint8_t *ws, StreamSet &ss)
{
    CUtensorMap maps[5];
    if (!make_input_maps(a, maps)) return cudaErrorInvalidValue;
    const int nslots = p.slots;
    const size_t slot_bytes = p.rec_total + p.sx_total;
    float *carry = p.carry_bytes ? reinterpret_cast<float *>(ws + nslots * slot_bytes) : nullptr;
    cudaError_t e = cudaEventRecord(ss.start, a.stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss.out, ss.start, 0);
    auto window = [&](int w, int &c0, int &ncw, uint8_t *&recs, uint8_t *&sxs) {
        c0 = w * p.wc;
        ncw = (p.nchunks - c0 < p.wc) ? p.nchunks - c0 : p.wc;
        recs = ws + (w % nslots) * slot_bytes;
        sxs = recs + p.rec_total;
    };
    const FwdArgs &ac = a;
    FwdArgs ao = a;
    ao.stream = ss.out;
    int c0, ncw;
    uint8_t *recs, *sxs;
    if (p.nwindows > 0) {
        window(0, c0, ncw, recs, sxs);
        e = launch_prep(ac, maps, recs, c0, ncw, p.wc, false);
    }
    for (int w = 0; w < p.nwindows && e == cudaSuccess; ++w) {
        const int slot = w % nslots;
        if (w + 1 < p.nwindows && w + 1 >= nslots) e = cudaStreamWaitEvent(a.stream, ss.ev_o[(w + 1) % nslots], 0);
        window(w, c0, ncw, recs, sxs);
        const float *S_in = (w == 0) ? a.S0 : carry;
        float *S_out = (w == p.nwindows - 1) ? a.S_T : carry;
        if (e == cudaSuccess) e = launch_chain(ac, p.dvt, recs, sxs, S_in, S_out, ncw, p.wc, p.overlap);
        if (e == cudaSuccess && w + 1 < p.nwindows) {
            int c1, n1;
            uint8_t *r1, *x1;
            window(w + 1, c1, n1, r1, x1);
            e = launch_prep(ac, maps, r1, c1, n1, p.wc, p.overlap);
        }
        if (e == cudaSuccess) e = cudaEventRecord(ss.ev_c[slot], a.stream);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(ss.out, ss.ev_c[slot], 0);
        // output launches of consecutive windows write disjoint rows
        if (e == cudaSuccess) e = launch_out(ao, &maps[4], recs, sxs, c0, ncw, p.wc, true);
        if (e == cudaSuccess) e = cudaEventRecord(ss.ev_o[slot], ss.out);
    }
    // join: the caller's stream waits for the last output (the output stream runs
    // its windows in order)
    if (e == cudaSuccess && p.nwindows > 0) e = cudaStreamWaitEvent(a.stream, ss.ev_o[(p.nwindows - 1) % nslots], 0);
    return e;
}

// Wide batches, whose chains take most SMs so that prep and chain take turns,
// with plain outputs: per window the prep, then the chain CTAs, which also
// compute the window's outputs (fwd_chain_out.cu).  No output pass, no state
// images in the workspace.
cudaError_t run_fwd_tc_chain_out(const FwdArgs &a, const FwdTcPlan &p, uint8_t *ws)
{
    CUtensorMap maps[5];
    if (!make_input_maps(a, maps)) return cudaErrorInvalidValue;
    const size_t slot_bytes = p.rec_total + p.sx_total;
    float *carry = p.carry_bytes ? reinterpret_cast<float *>(ws + p.slots * slot_bytes) : nullptr;
    cudaError_t e = cudaSuccess;
    for (int w = 0; w < p.nwindows && e == cudaSuccess; ++w) {
        const int c0 = w * p.wc, ncw = (p.nchunks - c0 < p.wc) ? p.nchunks - c0 : p.wc;
        uint8_t *recs = ws + (w % p.slots) * slot_bytes;
        const float *S_in = (w == 0) ? a.S0 : carry;
        float *S_out = (w == p.nwindows - 1) ? a.S_T : carry;
        e = launch_prep(a, maps, recs, c0, ncw, p.wc, false);
        if (e == cudaSuccess) e = launch_chain_out(a, p.dvt, recs, S_in, S_out, c0, ncw, p.wc, false);
    }
    return e;
}

// The persistent launch (fwd_persist.cu) for shapes whose chains leave most
// SMs free; returns false (nothing enqueued) when the device cannot hold the
// cooperative grid, so that the windowed schedule runs instead.
bool try_fwd_persist(const FwdArgs &a, cudaMemPool_t pool, cudaError_t *status)
{
    const PersistPlan p = plan_fwd_persist(a.B, a.T, a.H, a.dv, a.num_sms);
    if (!p.use) return false;
    CUtensorMap maps[5];
    if (!make_input_maps(a, maps)) {
        *status = cudaErrorInvalidValue;
        return true;
    }
    void *ws = nullptr;
    cudaError_t e = cudaMallocFromPoolAsync(&ws, p.ws_bytes, pool, a.stream);
    if (e != cudaSuccess) {
        *status = e;
        return true;
    }
    e = launch_persist(a, maps, static_cast<uint8_t *>(ws), p);
    const cudaError_t f = cudaFreeAsync(ws, a.stream);
    if (e == cudaErrorCooperativeLaunchTooLarge) {
        (void)cudaGetLastError();
        return false;
    }
    *status = e != cudaSuccess ? e : f;
    return true;
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
    if (try_fwd_persist(a, pool, &e)) return e;
    const FwdTcPlan p = plan_fwd_tc(a.B, a.T, a.H, a.dv, 0, a.num_sms);
    const size_t bytes = p.ws_bytes;
    void *ws = nullptr;
    e = cudaMallocFromPoolAsync(&ws, bytes, pool, a.stream);
    if (e != cudaSuccess) return e;
    if (!p.overlap && !a.g) {
        e = run_fwd_tc_chain_out(a, p, static_cast<uint8_t *>(ws));
    } else {
        std::lock_guard<std::mutex> lock(ss->mu);
        e = run_fwd_tc_overlapped(a, p, static_cast<uint8_t *>(ws), *ss);
    }
    const cudaError_t f = cudaFreeAsync(ws, a.stream);
    return e != cudaSuccess ? e : f;
}

}  // namespace gdn2
