// fwd_persist.cu -- the chunkwise forward (bf16 inputs) as one persistent launch.
//
// The three kinds of work of the chunkwise form -- the prep of a chunk
// (prep_body.cuh), the chain of a (batch, head, value tile) over all chunks
// (chain_body.cuh) and the outputs of a chunk (out_body.cuh) -- run in one
// cooperative grid of one CTA per SM, so that every CTA is resident and may
// wait for another:
//   * CTAs [0, nchain) each run one chain (a 64- or 128-wide value tile of one
//     (batch, head)) over the whole sequence;
//   * every other CTA is two independent workers of 256 threads, each with half
//     of the SM's shared and tensor memory, which take items from one counter
//     in a fixed order: the prep of chunk c for all heads, then the outputs of
//     chunk c - kLag for all heads, for c = 0, 1, ...
// Records and state images live in rings of kRing chunks per (batch, head).
// Hand-offs go through flags in global memory (release / acquire at GPU scope):
//   prep(c)   -> rec_gen    : record c is written
//                             (the chain's producer and output(c) wait for it)
//   chain     -> prog = n   : the state images of chunks [0, n) are exported
//                             (output(c) waits for n > c; prep(c + kRing) waits for
//                             n > c + 1, the chain being done with record c then)
//   out(c)    -> out_gen    : the ring slots of chunk c have been read
//                             (prep(c + kRing) waits for it)
// The chain exports the state image of chunk c into its slot once its producer
// has seen record c ready: prep(c) waited for output(c - kRing), the slot's last
// reader.  Every item waits only for items earlier in the order or for chain
// progress that those items make possible, and kLag < kRing, so the order
// cannot deadlock (tests/test_persist_schedule.py replays these rules).  Every wait is bounded: a wait that gives up raises kErrTimeout and
// an abort flag that ends every other wait, and the CTA leaves once its
// copies in flight have landed.
//
// Compared with the windowed schedule (fwd_tc.cu) there are no launch gaps or
// chain restarts between windows, workers are not phase-locked (one loading
// while another computes), and outputs follow the chain chunk by chunk.
#include <cuda.h>

#include "chain_body.cuh"
#include "launch.h"
#include "out_body.cuh"
#include "prep_body.cuh"

namespace gdn2 {
namespace {

using namespace sm100;

constexpr int kPersistThreads = 512;
constexpr uint64_t kFlagWaitNs = 1000000000ull;

// Shared memory of a persistent CTA (from its 1024-aligned base): two worker
// regions, each with its mbarriers and item slot at the end, and the workers'
// tensor-memory address slot after them; or the layout of a chain over a DVT-wide
// value tile, which keeps its own slot.
constexpr int kHalfData = align_up(prep::PrepLayout::DATA, 1024);
constexpr int kHalf = kHalfData + 1024;  // + mbarriers (prep TMA, prep UMMA, output loads, output UMMA), item
constexpr int kTmemSlot = 2 * kHalf;
template <int DV, int DVT>
constexpr int persist_smem()
{
    return chain::ChainLayout<DV, DVT>::BYTES > kTmemSlot + 16 + 1024 ? chain::ChainLayout<DV, DVT>::BYTES
                                                                         : kTmemSlot + 16 + 1024;
}
static_assert(outp::OutLayout<128>::DATA <= kHalfData, "output region");
static_assert(chain::ChainLayout<128, 64>::NS >= 3 && chain::ChainLayout<64, 64>::NS >= 3, "chain ring depth");
static_assert(persist_smem<128, 64>() <= 232448, "shared memory");

struct FlagLayout {
    int bh, nt;
    __host__ __device__ int rec_gen() const { return 0; }
    __host__ __device__ int out_gen() const { return bh * kRing; }
    __host__ __device__ int prog() const { return 2 * bh * kRing; }
    __host__ __device__ int next() const { return align_up(2 * bh * kRing + bh * nt, 32); }
    __host__ __device__ int abort() const { return next() + 32; }
    __host__ __device__ int words() const { return abort() + 32; }
};

// Wait until *p >= target.  Gives up after kFlagWaitNs (raising kErrTimeout
// and the abort flag) or when another wait has raised the abort flag.
__device__ __noinline__ bool wait_flag(const uint32_t *p, uint32_t target, uint32_t *abort, unsigned int *err)
{
    if (ld_acquire_gpu(p) >= target) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t n = 0; n < (1u << 26); ++n) {
        __nanosleep(64);
        if (ld_acquire_gpu(p) >= target) return true;
        if (*reinterpret_cast<volatile uint32_t *>(abort)) return false;
        if ((n & 255) == 255 && global_ns() - t0 > kFlagWaitNs) break;
    }
    atomicOr(err, kErrTimeout);
    atomicExch(abort, 1u);
    return false;
}

// A flag that nothing sets and its abort word, for the bounded-wait self-test.
__device__ uint32_t g_selftest_words[2];

__global__ void selftest_wait_kernel(unsigned int *err)
{
    if (threadIdx.x == 0) wait_flag(&g_selftest_words[0], 1u, &g_selftest_words[1], err);
}

// The chain's view of the rings of one (batch, head) and of its own progress counter.
template <int DV>
struct RingFlow {
    static constexpr bool kPublishes = true;
    const uint8_t *recs;
    uint8_t *sxs;
    const uint32_t *rec_gen, *out_gen;
    uint32_t *prog, *abort;
    unsigned int *err;
    __device__ const uint8_t *record(int c) const { return recs + (long)(c % kRing) * Record<DV>::BYTES; }
    __device__ uint8_t *sx_slot(int c) const { return sxs + (long)(c % kRing) * SxSlot<DV>::BYTES; }
    __device__ bool record_ready(int c) const
    {
        const bool ok = wait_flag(rec_gen + c % kRing, (uint32_t)(c / kRing + 1), abort, err);
        fence_proxy_async_global();
        return ok;
    }
    // bounded wait for the state warps' export count (shared memory)
    __device__ bool wait_count(const uint32_t *cnt, uint32_t target) const
    {
        const uint64_t t0 = global_ns();
        for (uint32_t n = 0; n < (1u << 28); ++n) {
            if (smem_ld_acquire(cnt) >= target) return true;
            if ((n & 63) == 63) {
                if (*reinterpret_cast<volatile uint32_t *>(abort)) return false;
                if (global_ns() - t0 > kFlagWaitNs) break;
            }
        }
        atomicOr(err, kErrTimeout);
        atomicExch(abort, 1u);
        return false;
    }
    // the state images of chunks [0, n) are in the workspace
    __device__ void exported(int n) const { st_release_gpu(prog, (uint32_t)n); }
};

// Item n of the workers' order: kind 0 = prep, 1 = outputs, -1 = none left.
struct Item {
    int kind, c, r;
};

__device__ __forceinline__ Item decode_item(int n, int P, int bh)
{
    if (n < 0) return {-1, 0, 0};  // no item (the abort flag was up)
    const int lag = min(kLag, P);
    const int head = lag * bh;
    if (n < head) return {0, n / bh, n % bh};
    n -= head;
    const int mid = 2 * bh * (P - lag);
    if (n < mid) {
        const int g = lag + n / (2 * bh), k = n % (2 * bh);
        return k < bh ? Item{0, g, k} : Item{1, g - lag, k - bh};
    }
    n -= mid;
    if (n < head) return {1, P - lag + n / bh, n % bh};
    return {-1, 0, 0};
}

// GEN: any gate layout and the fused layer's processing; without it the
// operator's plain form (per-channel gates, plain outputs), whose code is
// compiled without those branches.
template <int DV, int DVT, bool GEN>
__global__ void __launch_bounds__(kPersistThreads, 1)
persist_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_la,
               const __grid_constant__ CUtensorMap tm_g,
               const bf16 *__restrict__ vg, const bf16 *__restrict__ wg, const prep::GateSrc gs_arg,
               const outp::OutEpi epi_arg, bf16 *__restrict__ o, const float *S0,
               float *S_T, uint8_t *__restrict__ recs, uint8_t *__restrict__ sxs, uint32_t *flags, int B, int T,
               int H, int nchain, unsigned int *err)
{
    const prep::GateSrc gs = GEN ? gs_arg : prep::GateSrc{gs_arg.b, gs_arg.la, 0u};
    const outp::OutEpi epi = GEN ? epi_arg : outp::OutEpi{nullptr, nullptr, 0.f};
    using CL = chain::ChainLayout<DV, DVT>;
    constexpr int NT = DV / DVT;  // chain CTAs per head
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int bh = B * H, P = (T + kChunk - 1) / kChunk;
    const bool is_chain = (int)blockIdx.x < nchain;
    const FlagLayout fl{bh, NT};
    uint32_t *rec_gen = flags + fl.rec_gen(), *out_gen = flags + fl.out_gen(), *prog = flags + fl.prog();
    uint32_t *next = flags + fl.next(), *abort = flags + fl.abort();
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + (is_chain ? CL::SLOT : kTmemSlot));
    const uint32_t tcols = is_chain ? CL::TMEM_COLS : 512;

    if (is_chain) {
        if (tid == 0) chain::chain_init<DV, DVT>(sm);
    } else if ((tid & 255) == 0) {
        uint64_t *hb = reinterpret_cast<uint64_t *>(sm + (tid >> 8) * kHalf + kHalfData);
        for (int k = 0; k < 4; ++k) mbar_init(hb + k, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    if (is_chain) {
        if (tid < chain::kChainThreads) {
            const int pair = blockIdx.x / NT, tile = blockIdx.x % NT;
            const RingFlow<DV> f{recs + (long)pair * kRing * Record<DV>::BYTES,
                                 sxs + (long)pair * kRing * SxSlot<DV>::BYTES,
                                 rec_gen + pair * kRing,
                                 out_gen + pair * kRing,
                                 prog + pair * NT + tile,
                                 abort,
                                 err};
            chain::chain_run<DV, DVT>(sm, tmem, tid, f, S0, S_T, pair, tile, P, err);
        }
    } else {
        // ---------------------------------------------------------------- worker
        const int half = tid >> 8, lt = tid & 255, bar_id = 2 + half, bcast_id = 4 + half;
        uint8_t *hs = sm + half * kHalf;
        uint64_t *hb = reinterpret_cast<uint64_t *>(hs + kHalfData);
        volatile int *item_slot = reinterpret_cast<volatile int *>(hs + kHalfData + 64);
        const uint32_t ht = tmem + (uint32_t)(half * 256);
        uint32_t tma_phase = 0, mma_phase = 0, out_phase = 0;
        for (;;) {
            // Warp 1 takes the next item, checks its dependencies (one flag per
            // lane) and issues its loads while warp 0 may still be releasing the
            // last item (a GPU-scope fence); warp 0 joins at the barrier after.
            if (lt == 32) item_slot[0] = *reinterpret_cast<volatile uint32_t *>(abort) ? -1 : (int)atomicAdd(next, 1u);
            if (lt >= 32) named_bar(bcast_id, 224);
            bool ok = true;
            if (lt >= 32 && lt < 64) {
                const Item it = decode_item(item_slot[0], P, bh);
                const int c = it.c, r = it.r, slot = c % kRing, lane = lt - 32;
                const uint32_t *fp = nullptr;
                uint32_t target = 0;
                if (it.kind == 0) {
                    if (c >= kRing && lane == 0) fp = out_gen + r * kRing + slot, target = (uint32_t)(c / kRing);
                    if (c >= kRing && lane >= 1 && lane <= NT) fp = prog + r * NT + lane - 1, target = (uint32_t)(c - kRing + 2);
                } else if (it.kind == 1) {
                    if (lane == 0) fp = rec_gen + r * kRing + slot, target = (uint32_t)(c / kRing + 1);
                    if (lane >= 1 && lane <= NT) fp = prog + r * NT + lane - 1, target = (uint32_t)(c + 1);
                }
                ok = __all_sync(0xffffffffu, fp == nullptr || wait_flag(fp, target, abort, err)) != 0;
                if (lane == 0 && it.kind >= 0) {
                    fence_proxy_async_global();
                    if (ok) {
                        if (it.kind == 0)
                            prep::prep_issue_loads(hs, hb, &tm_q, &tm_k, &tm_b, &tm_la, c * kChunk, r % H, r / H,
                                                 gs.layout);
                        else
                            outp::out_issue_loads<DV>(hs, hb + 2, recs + ((long)r * kRing + slot) * Record<DV>::BYTES,
                                                      sxs + ((long)r * kRing + slot) * SxSlot<DV>::BYTES,
                                                      epi.g ? &tm_g : nullptr, c * kChunk, r % H, r / H);
                    }
                }
            }
            ok = named_bar_and(bar_id, 256, ok);
            const Item it = decode_item(item_slot[0], P, bh);
            if (it.kind < 0 || !ok) break;
            const int c = it.c, r = it.r, h = r % H, bi = r / H, slot = c % kRing;
            uint8_t *rec = recs + ((long)r * kRing + slot) * Record<DV>::BYTES;
            uint64_t *ld_bar = it.kind == 0 ? hb : hb + 2;
            const uint32_t ld_phase = it.kind == 0 ? tma_phase : out_phase;
            if (it.kind == 0) {
                ok = prep::prep_chunk<DV>(hs, ht, lt, bar_id, hb, tma_phase, hb + 1, mma_phase, vg, wg, gs, rec, T,
                                          H, c * kChunk, h, bi, err);
                tma_phase ^= 1;
            } else {
                const int t0 = c * kChunk;
                const long row0 = (((long)bi * T + t0) * H + h) * (long)DV;
                ok = outp::out_chunk<DV, 256>(hs, ht, lt, bar_id, hb + 2, hb + 3, out_phase, o + row0, T - t0,
                                              (long)H * DV, epi, err);
            }
            // publish: every thread's stores, then one release
            fence_proxy_async_global();
            tc_fence_before();
            ok = named_bar_and(bar_id, 256, ok);
            if (lt == 0) {
                if (ok) {
                    st_release_gpu((it.kind == 0 ? rec_gen : out_gen) + r * kRing + slot, (uint32_t)(c / kRing + 1));
                } else {
                    atomicExch(abort, 1u);
                    mbar_wait(ld_bar, ld_phase, err);  // the item's copies land before the CTA may leave
                }
            }
            if (!ok) break;
            tc_fence_after();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, tcols);
    }
}

}  // namespace

cudaError_t launch_selftest_wait(cudaStream_t stream, unsigned int *err)
{
    void *words = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&words, g_selftest_words);
    if (e == cudaSuccess) e = cudaMemsetAsync(words, 0, sizeof(uint32_t) * 2, stream);
    if (e != cudaSuccess) return e;
    selftest_wait_kernel<<<1, 32, 0, stream>>>(err);
    return cudaGetLastError();
}

PersistPlan plan_fwd_persist(int B, int T, int H, int dv, int num_sms)
{
    PersistPlan p{};
    const long bh = (long)B * H;
    // Value tile of a chain CTA: 64 columns.  Its step is shorter than a 128-wide
    // tile's (B1 H16 T4096: 121.6 -> 117.6 us), and at B1 H16 T65536, where the
    // wider tile would leave more SMs to the workers, the two measured 1.50 against
    // 1.75 ms on some devices and 1.48 against 1.46 ms on others.
    p.dvt = 64;
    const int nt = dv / p.dvt;
    p.nchain = (int)(bh * nt);
    // the chain CTAs must leave most SMs to the workers
    p.use = (dv == 64 || dv == 128) && num_sms > 0 && T > 0 && p.nchain * 4 <= num_sms;
    p.grid = num_sms;
    p.rec_total = (size_t)bh * kRing * (dv == 128 ? Record<128>::BYTES : Record<64>::BYTES);
    p.sx_total = (size_t)bh * kRing * (dv == 128 ? SxSlot<128>::BYTES : SxSlot<64>::BYTES);
    p.flag_bytes = (size_t)FlagLayout{(int)bh, nt}.words() * 4;
    p.ws_bytes = p.rec_total + p.sx_total + align_up((int)p.flag_bytes, 256);
    return p;
}

cudaError_t launch_persist(const FwdArgs &a, const CUtensorMap *maps, uint8_t *ws, const PersistPlan &p)
{
    uint8_t *recs = ws, *sxs = ws + p.rec_total;
    uint32_t *flags = reinterpret_cast<uint32_t *>(ws + p.rec_total + p.sx_total);
    cudaError_t e = cudaMemsetAsync(flags, 0, p.flag_bytes, a.stream);
    if (e != cudaSuccess) return e;
    const bool gen = a.layout != 0 || a.g != nullptr;
    auto kern = a.dv == 64 ? (gen ? persist_kernel<64, 64, true> : persist_kernel<64, 64, false>)
                               : (gen ? persist_kernel<128, 64, true> : persist_kernel<128, 64, false>);
    const int smem = a.dv == 64 ? persist_smem<64, 64>() : persist_smem<128, 64>();
    static std::atomic<unsigned long long> smem_set[4] = {};
    e = ensure_smem_limit(kern, smem, smem_set[(a.dv == 64 ? 0 : 1) + (gen ? 2 : 0)]);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(kPersistThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = a.stream;
    // every CTA resident at once: the CTAs wait for one another
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const prep::GateSrc gs{(const bf16 *)a.b, a.log_alpha, a.layout};
    const outp::OutEpi epi{a.g, a.norm_weight, a.eps};
    return cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], maps[3], maps[4], (const bf16 *)a.v,
                              (const bf16 *)a.w,
                              gs, epi, (bf16 *)a.o, a.S0, a.S_T, recs, sxs, flags, a.B, a.T, a.H, p.nchain, a.err);
}

}  // namespace gdn2
