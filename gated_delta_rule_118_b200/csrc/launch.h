// launch.h -- internal (C++) interface between the C ABI layer and the kernels.
// Arguments arrive here already validated by gdn2_api.cu.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

namespace gdn2 {

struct DecodeArgs {
    const void *q, *k, *v, *b, *w;
    const float *log_alpha;
    float *S;
    void *o;
    int B, T, H, dk, dv;  // T tokens per call (1 for a decode step)
    bool bf16;
    unsigned layout;      // gdn2_gate_layout bits
    cudaStream_t stream;
};

struct FwdArgs {
    const void *q, *k, *v, *b, *w;
    const float *log_alpha;
    const float *S0;  // may be null (zero state)
    void *o;
    float *S_T;       // may be null (not written); may alias S0
    int B, T, H, dk, dv;
    bool bf16;
    unsigned layout;    // gdn2_gate_layout bits, and kLayerInputs for the fused layer
    cudaStream_t stream;
    unsigned int *err;  // device error word
    int num_sms;
    // the fused layer's output processing (null g: the operator's plain outputs)
    const void *g;             // [B][T][H][dv] output-gate logits
    const float *norm_weight;  // [dv]
    float eps;
};
// FwdArgs::layout bit: q, k and the gates are the layer's raw inputs (gdn2_layer_fwd)
constexpr unsigned kLayerInputsBit = 8u;
cudaError_t launch_layer_epilogue_rows(const FwdArgs &a);  // y = RMSNorm(o) * weight * sigmoid(g), in place

// Chunkwise backward (bwd_simt.cu): gradients of sum(o * dO) + sum(S_T * dS_T).
struct BwdArgs {
    const void *q, *k, *v, *b, *w;
    const float *log_alpha;
    const float *S0;     // may be null (zero)
    const void *dO;
    const float *dS_T;   // may be null (zero)
    float *ws;           // bwd_workspace_floats(...) fp32 of workspace
    float *gq, *gk, *gv, *gb, *gw, *gla;   // fp32 gradients
    float *dS0;          // may be null (not written)
    int B, T, H, dk, dv;
    bool bf16;
    cudaStream_t stream;
};
size_t bwd_workspace_floats(int B, int T, int H, int dk, int dv);
cudaError_t launch_bwd_simt(const BwdArgs &a);
// The bf16 tensor-core backward (bwd_tc.cu; dk = 128): prep records with T and
// P for every chunk, the forward chain's state images, the adjoint chain's
// images of dS', then the gradients of every chunk in parallel.  `ws` holds
// bwd_tc_workspace_bytes(...) bytes.
size_t bwd_tc_workspace_bytes(int B, int T, int H, int dv);
cudaError_t launch_bwd_tc(const BwdArgs &a, uint8_t *ws, unsigned int *err, int num_sms);
// The library's stream-ordered workspace pool of a device (keeps freed blocks).
cudaMemPool_t workspace_pool(int dev);

bool device_error_word(unsigned int **err);
cudaError_t launch_decode(const DecodeArgs &a);
cudaError_t launch_fwd_simt(const FwdArgs &a);

// bf16 tensor-core forward, per window of WC chunks:
//   prep (per chunk) -> records -> chain (sequential, exports the state image Sx) -> output (per chunk)
struct FwdTcPlan {
    int dvt;            // value-tile width of a chain CTA
    int nchunks;        // chunks in the sequence
    int wc;             // chunks per window
    int nwindows;
    size_t rec_bytes;   // bytes of one prep record
    size_t sx_bytes;  // bytes of one exported state image
    size_t rec_total;   // records of one window
    size_t sx_total;  // state images of one window
    size_t carry_bytes; // state carried between windows
    size_t ws_bytes;    // total workspace
    int slots;          // windows in flight (workspace slots)
    bool overlap;       // a window's prep runs beside the previous window's chain
};
// Workspace of the allocating entry point: kWindowSlots windows in flight when a
// window's prep overlaps the previous chain, else two larger ones.  Wide batches
// (chains on most SMs) gain from few, long windows: each window pays for a prep
// tail and a chain that leaves SMs idle, which costs more than the records'
// round trip through HBM (training batch B8 H16 T4096: 16-chunk windows 742 us,
// 32-chunk 663 us, one window 637 us).
constexpr size_t kWindowBudgetBytes = size_t(128) << 20;
constexpr size_t kWideWindowBudgetBytes = size_t(2048) << 20;
constexpr int kWindowSlots = 4;
// num_sms > 0: plan the overlapped schedule of the allocating entry point on a
// device with num_sms SMs (budget ignored); num_sms == 0: one window slot of
// `budget` bytes (the no-allocation entry point).
FwdTcPlan plan_fwd_tc(int B, int T, int H, int dv, size_t budget, int num_sms);
cudaError_t run_fwd_tc(const FwdArgs &a, const FwdTcPlan &p, uint8_t *ws);
// Tensor maps of the forward's TMA-loaded inputs (q, k, b, log_alpha, output-gate
// logits), and of a bf16 [B][T][H][d] tensor in boxes of 64 channels x 64
// tokens with the 128-byte swizzle.
bool make_input_maps(const FwdArgs &a, CUtensorMap *maps);
bool make_token_map(CUtensorMap *m, const void *base, int d, int H, int T, int B);
cudaError_t launch_fwd_tc(const FwdArgs &a);
// `overlap`: launch as a programmatic dependent of the previous kernel in the
// stream, so that it may start before that kernel ends (only where the two
// touch disjoint data).
// tp: non-null for the backward, which keeps every chunk's T, P and T - bf16(T) there
// (kTpBytes per record).
constexpr int kTpBytes = 3 * 8192;
cudaError_t launch_prep(const FwdArgs &a, const CUtensorMap *maps, uint8_t *ws, int c0, int ncw, int WC,
                        bool overlap, uint8_t *tp = nullptr);
cudaError_t launch_chain(const FwdArgs &a, int dvt, const uint8_t *ws, uint8_t *sx, const float *S_in,
                         float *S_out, int ncw, int WC, bool overlap);
cudaError_t launch_out(const FwdArgs &a, const CUtensorMap *tm_g, const uint8_t *ws, const uint8_t *sx, int c0,
                       int ncw, int WC, bool overlap);
// The chain of a window with the window's (plain) outputs in the same CTAs.
cudaError_t launch_chain_out(const FwdArgs &a, int dvt, const uint8_t *ws, const float *S_in, float *S_out, int c0,
                             int ncw, int WC, bool overlap);
// Persistent forward (fwd_persist.cu): prep, chain and output work in one
// cooperative launch of one CTA per SM, records and state images in rings of
// kRing chunks per (batch, head); the outputs of chunk c are handed out after
// the prep of chunk c + kLag (kLag < kRing).
// A prep takes about as long as a dozen chain steps, so prep runs that far ahead
// of the chain; outputs are handed out kLag chunks behind it, when they can run.
constexpr int kRing = 24;
constexpr int kLag = 16;
struct PersistPlan {
    bool use;           // the shape suits the persistent launch
    int dvt;            // value tile of a chain CTA
    int nchain;         // chain CTAs (the others are workers)
    int grid;           // CTAs (one per SM)
    size_t rec_total;   // record rings
    size_t sx_total;    // state-image rings
    size_t flag_bytes;  // flags and counters (zeroed before the launch)
    size_t ws_bytes;    // total workspace
};
PersistPlan plan_fwd_persist(int B, int T, int H, int dv, int num_sms);
cudaError_t launch_persist(const FwdArgs &a, const CUtensorMap *maps, uint8_t *ws, const PersistPlan &p);
// One-warp kernel whose flag wait (the persistent forward's) runs out: kErrTimeout after one second.
cudaError_t launch_selftest_wait(cudaStream_t stream, unsigned int *err);
// Raise a kernel's dynamic shared-memory limit on the current device, once per
// device (bit d of `done` records device d).
template <typename Kernel>
cudaError_t ensure_smem_limit(Kernel kern, int bytes, std::atomic<unsigned long long> &done)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_release);
    return e;
}

// Launch configuration with the programmatic-dependent-launch attribute set when `overlap`.
struct LaunchCfg {
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    LaunchCfg(dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool overlap)
    {
        cfg.gridDim = grid;
        cfg.blockDim = block;
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = overlap ? 1 : 0;
    }
};

}  // namespace gdn2
