// prep_body.cuh -- the prep of one chunk, shared by the windowed prep kernel
// (fwd_prep.cu) and the persistent forward (fwd_persist.cu).
//
// One group of 256 threads per (batch, head, chunk) computes every quantity of the chunkwise WY
// form that does not depend on the state carried in from earlier chunks
// ("Gated DeltaNet-2", iplexlaw.co.kr, section "Procesamiento del token y
// entrenamiento paralelo"; gist.science, section 3: the cumulative per-channel
// decay is folded into asymmetric erase/key factors and a lower triangular
// system (I + T)^{-1} is solved per chunk).  With Gamma the chunk-local
// cumulative log-decay (fp32) and r the chunk midpoint:
//   Ehat = e^{Gamma-Gamma_r} b k    Qhat = e^{Gamma-Gamma_r} q
//   Khat = e^{Gamma_r-Gamma} k      Z = w v
//   A = strict_lower(Ehat Khat^T)   P = lower(Qhat Khat^T)   T = (I + A)^{-1}
//   Y = e^{Gamma_C-Gamma_r} Khat^T T  (= Ktil^T T with Ktil = e^{Gamma_C-Gamma} k)
//   PT = P T    G = Y Ehat    Q' = Qhat - PT Ehat
// and the record keeps NG = -G Diag(e^{Gamma_r}), QS = Q' Diag(e^{Gamma_r}),
// Y, PT, Z and e^{Gamma_C}, so that for the incoming state S
//   S_next = e^{Gamma_C} S + NG S + Y Z        O = QS S + PT Z.
// Nothing here depends on the values except Z, which is a plain product.
//
// Layout of the work on one SM: a group fits in half of the shared memory,
// tensor memory and register file (two CTAs of the windowed prep kernel, or
// the two worker halves of a persistent CTA), so two chunks are in flight per
// SM and one hides the other's load and UMMA latencies.  q, k, b and log_alpha arrive by
// TMA straight into the operand buffers and the factors are formed in place;
// v and w are read with plain vector loads and Z goes straight to the record.
// Products are tcgen05 UMMAs with fp32 accumulators in tensor memory, three
// round trips in all (Gram; Y and PT; G and P T Ehat); the solve is fp32
// (16x16 diagonal blocks by substitution on CUDA cores, then two levels of
// block merging whose small products run as warp-level tf32 MMAs).  Record
// pieces go straight from the tensor-memory readouts to the record, each warp
// store covering 512 contiguous bytes.
#pragma once

#include <cuda.h>

#include "tc_common.cuh"

namespace gdn2 {
namespace prep {

using namespace sm100;

constexpr int kPrepThreads = 256;
constexpr int kDK = 128;

struct PrepLayout {
    static constexpr int EQ = 0;          // [Ehat;Qhat]: b, q arrive here
    static constexpr int KH = 32768;      // solve scratch -> Y (no swizzle)
    static constexpr int KT = 49152;      // k arrives here -> Khat -> PT (no swizzle)
    static constexpr int LA = 65536;      // log_alpha -> fp32 A | fp32 T -> bf16 T over A
    static constexpr int PO = 98304;      // Gamma quarter totals -> P
    static constexpr int DEC = 106496;    // e^{Gamma_C-Gamma_r}[128], e^{Gamma_r}[128]
    static constexpr int QP = 107520;     // bounded path: product of alpha per token quarter [4][128]
    static constexpr int DATA = 109568;   // end of the buffers above
    static constexpr int BAR = DATA;      // the windowed kernel's mbarriers and TMEM slot
    static constexpr int SLOT = BAR + 16;
    static constexpr int BYTES = SLOT + 16 + 1024;
    static constexpr int TX = 3 * 16384 + 32768;  // q, k, b, log_alpha
    static constexpr int AF = LA, TF = LA + 16384, TB = LA, XS = KH, TOT = PO;
    // tensor memory: Gram in [0, 64); then Y in [0, 64), PT in [64, 128); then G in [0, 128), P T Ehat in [128, 256)
    static constexpr uint32_t TM_GRAM = 0, TM_Y = 0, TM_PT = 64, TM_G = 0, TM_PW = 128, TMEM_COLS = 256;
};
static_assert(PrepLayout::BYTES * 2 + 2048 <= 233472, "two CTAs per SM");

// Gate inputs that hold one value per (token, head) (gdn2_gate_layout bits in
// `layout`); per-channel ones arrive by TMA.  Scalar b and log_alpha are
// broadcast over the channels of their rows in shared memory, so everything
// after the loads is the same for every layout.
//
// With kLayerInputs (gdn2_layer_fwd) the loaded tiles are the layer's raw
// inputs -- q and k before their L2 normalisation, and the logits of the erase
// gate, the write gate and the decay -- and the prep turns them into the
// operator's inputs in place ("Gated DeltaNet-2", iplexlaw.co.kr, section
// "Procesamiento del token y entrenamiento paralelo": L2-normalised queries and
// keys, sigmoid gates): q / sqrt(|q|^2 + 1e-6), k likewise, b = sigmoid(.),
// w = sigmoid(.), log_alpha = log sigmoid(.).
struct GateSrc {
    const bf16 *b;     // [B][T][H] with GDN2_ERASE_SCALAR
    const float *la;   // [B][T][H] with GDN2_DECAY_SCALAR
    unsigned layout;
};
constexpr unsigned kEraseScalar = 1u, kWriteScalar = 2u, kDecayScalar = 4u;  // gdn2_gate_layout bits
constexpr unsigned kLayerInputs = 8u;  // raw q, k and gate logits (the fused layer entry point)
constexpr float kL2Eps = 1e-6f;
// T entries off the identity by more than this mark an ill-conditioned chunk for
// the backward (random keys stay below 0.35 on every workload; nearly collinear
// keys with erase gates near 2 reach 0.4 to 1.8)
constexpr float kIllT = 0.5f;

// sigmoid(x) = (1 + tanh(x / 2)) / 2, one MUFU operation (tanh.approx.f32,
// relative error about 2^-11: below the bf16 rounding of the gates)
__device__ __forceinline__ float sigmoid_f(float x)
{
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
}
// log(sigmoid(x)) = min(x, 0) - log(1 + y), y = e^{-|x|} in (0, 1], finite for
// every finite x.  For y < 2^-10 the log is its series y - y^2/2 (the next term,
// y^3/3, is below 4e-7 of the result): a decay near 1 keeps its small log,
// which a rounded 1 + y would lose.
__device__ __forceinline__ float log_sigmoid_f(float x)
{
    const float y = __expf(-fabsf(x));
    const float l = y < 0.0009765625f ? y * (1.f - 0.5f * y) : __logf(1.f + y);
    return fminf(x, 0.f) - l;
}

__device__ __forceinline__ void tmem_ld32_wait(uint32_t taddr, float (&r)[32])
{
    tmem_ld32(taddr, r);
    tmem_ld_wait();
}

// The TMA loads of one chunk's q, b, k and log_alpha into a prep region,
// completing on `bar_tma` (issued by one thread).
// (b and log_alpha only where they are per channel).
__device__ __forceinline__ void prep_issue_loads(uint8_t *sm, uint64_t *bar_tma, const CUtensorMap *tm_q,
                                                 const CUtensorMap *tm_k, const CUtensorMap *tm_b,
                                                 const CUtensorMap *tm_la, int t0, int h, int bi, unsigned layout)
{
    using L = PrepLayout;
    const bool b_tma = !(layout & kEraseScalar), la_tma = !(layout & kDecayScalar);
    mbar_arrive_expect_tx(bar_tma, (uint32_t)(L::TX - (b_tma ? 0 : 16384) - (la_tma ? 0 : 32768)));
    for (int kb = 0; kb < 2; ++kb) {
        tma_load_4d(sm + L::EQ + kb * 16384 + 8192, tm_q, bar_tma, kb * 64, h, t0, bi);
        if (b_tma) tma_load_4d(sm + L::EQ + kb * 16384, tm_b, bar_tma, kb * 64, h, t0, bi);
        tma_load_4d(sm + L::KT + kb * 8192, tm_k, bar_tma, kb * 64, h, t0, bi);
    }
    if (la_tma) tma_load_4d(sm + L::LA, tm_la, bar_tma, 0, h, t0, bi);
}

// The layer's input processing (gdn2_layer_fwd) on a chunk's loaded tiles, in
// place: L2 norm of each q and k row, sigmoid of the erase-gate logits, log
// sigmoid of the decay logits (zero past the sequence end).  Out of line: the
// operator's own path compiles as without it.
static __device__ __noinline__ void prep_layer_inputs(uint8_t *sm, int tid, int bar_id, int Lc, unsigned layout)
{
    using L = PrepLayout;
    // ---------------------------------------------------------- the layer's input processing
    {   // L2 norm of each q and k row: two threads per row, one 64-channel half each
        const int r = tid >> 1, half = tid & 1, t = r & 63;
        uint8_t *row = (r < 64) ? sm + L::EQ + half * 16384 + 8192 + t * 128 : sm + L::KT + half * 8192 + t * 128;
        // the row's 16-byte pieces in an order rotated by the row, so that the
        // lanes of a warp (16 rows) spread over the banks
        float ss = 0.f;
#pragma unroll 2
        for (int c = 0; c < 8; ++c) {
            float x[8];
            unpack8(*reinterpret_cast<const uint4 *>(row + 16 * ((c + t) & 7)), x);
#pragma unroll
            for (int u = 0; u < 8; ++u) ss = fmaf(x[u], x[u], ss);
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        const float inv = rsqrtf(ss + kL2Eps);
#pragma unroll 2
        for (int c = 0; c < 8; ++c) {
            float x[8];
            uint4 *pp = reinterpret_cast<uint4 *>(row + 16 * ((c + t) & 7));
            unpack8(*pp, x);
#pragma unroll
            for (int u = 0; u < 8; ++u) x[u] *= inv;
            *pp = pack8(x);
        }
    }
    if (!(layout & kEraseScalar) || !(layout & kDecayScalar)) {
        const int t = tid >> 2, part = tid & 3;  // token, quarter of its channels
        if (!(layout & kEraseScalar)) {   // erase gate from its logits (row t of both half tiles)
#pragma unroll 1
            for (int m = 0; m < 4; ++m) {
                const int c = part * 4 + ((m + t) & 3);  // rotated by the row: bank spread
                uint4 *pp = reinterpret_cast<uint4 *>(sm + L::EQ + (c >> 3) * 16384 + t * 128 + (c & 7) * 16);
                float f[8];
                unpack8(*pp, f);
#pragma unroll
                for (int u = 0; u < 8; ++u) f[u] = sigmoid_f(f[u]);
                *pp = pack8(f);
            }
        }
        if (!(layout & kDecayScalar)) {   // log-decay from its logits; none past the sequence end
#pragma unroll 2
            for (int m = 0; m < 8; ++m) {
                float4 *pp = reinterpret_cast<float4 *>(sm + L::LA + t * 512 + part * 128 + ((m + t) & 7) * 16);
                const float4 x = *pp;
                *pp = t < Lc ? make_float4(log_sigmoid_f(x.x), log_sigmoid_f(x.y), log_sigmoid_f(x.z),
                                           log_sigmoid_f(x.w))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }
    named_bar(bar_id, kPrepThreads);
}

// The bounded form of a chunk's Gram (its decay too strong for the midpoint
// split), by the prep's threads once the chunk's inputs are in `sm` (raw b, q, k
// tiles and log_alpha): every factor is a decay over a stretch of the chunk,
// never the inverse of one, so nothing can overflow and what underflows is
// negligible:
//   A_ts = sum_j b_tj k_tj k_sj f_tsj,  P_ts = sum_j q_tj k_sj f_tsj,
//   f_tsj = e^{Gamma_tj - Gamma_sj} = prod_{s < u <= t} alpha_uj (running products),
//   Ebar = e^{Gamma} b k, Qbar = e^{Gamma} q (decayed from the chunk start),
//   Ktil = e^{Gamma_C - Gamma} k (decayed to the chunk end),
// and the record's scalings by e^{Gamma_C - Gamma_r} and e^{Gamma_r} become 1.
// Leaves A and a zero T in their fp32 places and P in its bf16 tile, like the
// midpoint form's Gram readout.  Out of line: the fast path's code stays as it is.
static __device__ __noinline__ void prep_bounded(uint8_t *sm, int tid, int bar_id)
{
    using L = PrepLayout;
    const int warp = tid >> 5;
    const int p = tid & 63, qr = tid >> 6;
    float *la = reinterpret_cast<float *>(sm + L::LA);
    float *Af = reinterpret_cast<float *>(sm + L::AF);
    float *Tf = reinterpret_cast<float *>(sm + L::TF);
    float *dec = reinterpret_cast<float *>(sm + L::DEC);
    float *qprod = reinterpret_cast<float *>(sm + L::QP);
    // ------------------------------------------------------ bounded path
    float *Ak = reinterpret_cast<float *>(sm + L::KH);  // A, fp32 (the solve's scratch is free)
    if (qr == 0) {
        dec[2 * p] = 1.f;
        dec[2 * p + 1] = 1.f;
        dec[kDK + 2 * p] = 1.f;
        dec[kDK + 2 * p + 1] = 1.f;
    }
    // alpha over log_alpha, and each quarter's product of alpha per channel
    {
        float q0 = 1.f, q1 = 1.f;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            float2 *lp = reinterpret_cast<float2 *>(la + (qr * 16 + u) * kDK + 2 * p);
            const float2 l = *lp;
            const float2 a = make_float2(ex2_approx(l.x * kLog2e), ex2_approx(l.y * kLog2e));
            *lp = a;
            q0 *= a.x; q1 *= a.y;
        }
        *reinterpret_cast<float2 *>(qprod + qr * kDK + 2 * p) = make_float2(q0, q1);
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) reinterpret_cast<float4 *>(Ak)[tid + m * kPrepThreads] = make_float4(0.f, 0.f, 0.f, 0.f);
    reinterpret_cast<float4 *>(sm + L::PO)[tid] = make_float4(0.f, 0.f, 0.f, 0.f);
    reinterpret_cast<float4 *>(sm + L::PO)[tid + kPrepThreads] = make_float4(0.f, 0.f, 0.f, 0.f);
    named_bar(bar_id, kPrepThreads);
    {
        // thread: token pair (pr, 63 - pr), 16 channels; the 8 lanes of a token reduce by shuffles
        const int pr = tid >> 3, cg = tid & 7, hb = cg >> 2, cb = (cg & 3) * 32;
        const uint8_t *bt = sm + L::EQ + hb * 16384, *qt = bt + 8192, *kt = sm + L::KT + hb * 8192;
        const float *al = la + 16 * cg;
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
            // the lanes of a warp hold 4 tokens; the loop runs to the warp's
            // largest token so that every lane takes part in the shuffles
            const int t = pass ? 63 - pr : pr, tmax = pass ? 63 - 4 * warp : 4 * warp + 3;
            float qv[16], ev[16], f[16];
            unpack8(*reinterpret_cast<const uint4 *>(qt + swz_off(t, cb, 128)), qv);
            unpack8(*reinterpret_cast<const uint4 *>(qt + swz_off(t, cb + 16, 128)), qv + 8);
            unpack8(*reinterpret_cast<const uint4 *>(bt + swz_off(t, cb, 128)), ev);
            unpack8(*reinterpret_cast<const uint4 *>(bt + swz_off(t, cb + 16, 128)), ev + 8);
            unpack8(*reinterpret_cast<const uint4 *>(kt + swz_off(t, cb, 128)), f);
            unpack8(*reinterpret_cast<const uint4 *>(kt + swz_off(t, cb + 16, 128)), f + 8);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                ev[j] *= f[j];
                f[j] = 1.f;
            }
#pragma unroll 1
            for (int s = tmax; s >= 0; --s) {
                const bool on = s <= t;
                float pa = 0.f, aa = 0.f;
                if (on) {
                    float kv[16];
                    unpack8(*reinterpret_cast<const uint4 *>(kt + swz_off(s, cb, 128)), kv);
                    unpack8(*reinterpret_cast<const uint4 *>(kt + swz_off(s, cb + 16, 128)), kv + 8);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float a = f[j] * kv[j];
                        pa = fmaf(qv[j], a, pa);
                        aa = fmaf(ev[j], a, aa);
                    }
#pragma unroll
                    for (int j = 0; j < 16; j += 4) {
                        const float4 a4 = *reinterpret_cast<const float4 *>(al + s * kDK + j);
                        f[j] *= a4.x; f[j + 1] *= a4.y; f[j + 2] *= a4.z; f[j + 3] *= a4.w;
                    }
                }
#pragma unroll
                for (int o = 1; o < 8; o <<= 1) {
                    pa += __shfl_xor_sync(0xffffffffu, pa, o);
                    aa += __shfl_xor_sync(0xffffffffu, aa, o);
                }
                if (cg == 0 && on) {
                    *reinterpret_cast<bf16 *>(sm + L::PO + swz_off(t, 2 * s, 128)) = __float2bfloat16_rn(pa);
                    if (s < t) Ak[af_off(t, s)] = aa;
                }
            }
        }
    }
    named_bar(bar_id, kPrepThreads);
    // the bounded factors over the raw tiles (two channels of 16 tokens per
    // thread), from running products of alpha: e^{Gamma_t} = prod_{u <= t} alpha_u,
    // e^{Gamma_C - Gamma_t} = prod_{u > t} alpha_u
    {
        float pre0 = 1.f, pre1 = 1.f, post0 = 1.f, post1 = 1.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 a = *reinterpret_cast<const float2 *>(qprod + q * kDK + 2 * p);
            if (q < qr) { pre0 *= a.x; pre1 *= a.y; }
            if (q > qr) { post0 *= a.x; post1 *= a.y; }
        }
        float2 sf[16];
#pragma unroll
        for (int u = 15; u >= 0; --u) {
            sf[u] = make_float2(post0, post1);
            const float2 a = *reinterpret_cast<const float2 *>(la + (qr * 16 + u) * kDK + 2 * p);
            post0 *= a.x; post1 *= a.y;
        }
        const int hb = p >> 5;
        const int cbyte = (2 * p & 63) * 2;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int t = qr * 16 + u;
            const float2 a = *reinterpret_cast<const float2 *>(la + t * kDK + 2 * p);
            pre0 *= a.x; pre1 *= a.y;
            const uint32_t off = swz_off(t, cbyte, 128);
            __nv_bfloat162 *ep = reinterpret_cast<__nv_bfloat162 *>(sm + L::EQ + hb * 16384 + off);
            __nv_bfloat162 *qp = reinterpret_cast<__nv_bfloat162 *>(sm + L::EQ + hb * 16384 + 8192 + off);
            __nv_bfloat162 *kp = reinterpret_cast<__nv_bfloat162 *>(sm + L::KT + hb * 8192 + off);
            const float2 bv = __bfloat1622float2(*ep), qv = __bfloat1622float2(*qp), kv = __bfloat1622float2(*kp);
            *ep = __floats2bfloat162_rn(pre0 * bv.x * kv.x, pre1 * bv.y * kv.y);
            *qp = __floats2bfloat162_rn(pre0 * qv.x, pre1 * qv.y);
            *kp = __floats2bfloat162_rn(sf[u].x * kv.x, sf[u].y * kv.y);
        }
    }
    named_bar(bar_id, kPrepThreads);  // every thread has read alpha
    // A into the solve's place, T starts as zero
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int idx = tid + m * kPrepThreads;
        reinterpret_cast<float4 *>(Af)[idx] = reinterpret_cast<const float4 *>(Ak)[idx];
        reinterpret_cast<float4 *>(Tf)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    named_bar(bar_id, kPrepThreads);
}

// The prep of one chunk (tokens [t0, t0 + 64) of head h, batch bi) by the
// kPrepThreads threads tid = 0.. that share named barrier `bar_id`, once
// prep_issue_loads has been issued for it: `sm` is their PrepLayout region
// (1024-byte aligned), `tmem` the first of their 256 tensor-memory columns,
// `bar_mma` an mbarrier for UMMA completion whose phase parity `mma_phase`
// tracks, and `rec` the chunk's record.  With TP (the backward) the chunk's T
// and P also go to `tp`: bf16 [64][64] tiles T and P, rows of 128 bytes with the
// 128-byte swizzle, as they sit in shared memory.  A chunk whose T has an entry
// off the identity by more than kIllT (nearly collinear keys with erase gates
// near 2: its products with T are alternating sums) also gets a third tile,
// T - bf16(T), and a nonzero word at byte 512 of the record's decay area.  Returns false
// (every thread alike) when a wait timed out.
template <int DV, bool TP = false>
__device__ __forceinline__ bool prep_chunk(uint8_t *sm, uint32_t tmem, int tid, int bar_id, uint64_t *bar_tma,
                                           uint32_t tma_phase, uint64_t *bar_mma, uint32_t &mma_phase,
                                           const bf16 *__restrict__ vg, const bf16 *__restrict__ wg,
                                           const GateSrc &gs, uint8_t *__restrict__ rec, int Tlen, int H, int t0,
                                           int h, int bi, unsigned int *err, uint8_t *__restrict__ tp = nullptr)
{
    using L = PrepLayout;
    using R = Record<DV>;
    const int warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wh = warp >> 2;  // TMEM lane quarter, column half
    const int Lc = min(kChunk, Tlen - t0);
    float *la = reinterpret_cast<float *>(sm + L::LA);  // [64][128] fp32
    float *Af = reinterpret_cast<float *>(sm + L::AF);
    float *Tf = reinterpret_cast<float *>(sm + L::TF);
    float *Xs = reinterpret_cast<float *>(sm + L::XS);
    float *dec = reinterpret_cast<float *>(sm + L::DEC);
    float *tot = reinterpret_cast<float *>(sm + L::TOT);
    float *qprod = reinterpret_cast<float *>(sm + L::QP);
    const uint32_t sbase = smem_u32(sm);
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    // v and w for Z = w v: plain vector loads, issued before anything waits
    // (tokens past the sequence end give zero rows of Z)
    constexpr int ZV = 64 * DV / 8 / kPrepThreads;  // 16-byte vectors per thread
    uint4 vv[ZV], wv[ZV];
    auto load_vw = [&]() {
#pragma unroll
        for (int m = 0; m < ZV; ++m) {
            const int idx = tid + m * kPrepThreads;
            const int t = idx / (DV / 8), j = (idx % (DV / 8)) * 8;
            vv[m] = make_uint4(0, 0, 0, 0);
            wv[m] = make_uint4(0, 0, 0, 0);
            if (t < Lc) {
                const long tok = ((long)bi * Tlen + t0 + t) * H + h, off = tok * DV + j;
                vv[m] = __ldg(reinterpret_cast<const uint4 *>(vg + off));
                if (gs.layout & kWriteScalar) {  // (a logit, with kLayerInputs: turned into a gate below)
                    const uint32_t two = (uint32_t)__bfloat16_as_ushort(wg[tok]) * 0x10001u;
                    wv[m] = make_uint4(two, two, two, two);
                } else {
                    wv[m] = __ldg(reinterpret_cast<const uint4 *>(wg + off));
                }
                if (gs.layout & kLayerInputs) {  // write gate from its logits
                    float f[8];
                    unpack8(wv[m], f);
#pragma unroll
                    for (int u = 0; u < 8; ++u) f[u] = sigmoid_f(f[u]);
                    wv[m] = pack8(f);
                }
            }
        }
    };
    load_vw();
    // scalar b / log_alpha: row t of the b tile (both 64-channel halves) and of
    // log_alpha filled with the token's value (zero past the sequence end), into
    // buffers the TMA leaves alone in these layouts
    if (gs.layout & (kEraseScalar | kDecayScalar)) {
        const int t = tid >> 2, part = tid & 3;
        const long tok = ((long)bi * Tlen + t0 + t) * H + h;
        if (gs.layout & kEraseScalar) {
            bf16 bt = t < Lc ? gs.b[tok] : __float2bfloat16_rn(0.f);
            if (gs.layout & kLayerInputs) bt = __float2bfloat16_rn(sigmoid_f(__bfloat162float(bt)));
            const uint32_t two = (uint32_t)__bfloat16_as_ushort(bt) * 0x10001u;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int c = part * 4 + ((m + t) & 3);  // 16-byte piece of the token's 256 bytes (rotated)
                *reinterpret_cast<uint4 *>(sm + L::EQ + (c >> 3) * 16384 + t * 128 + (c & 7) * 16) =
                    make_uint4(two, two, two, two);
            }
        }
        if (gs.layout & kDecayScalar) {
            const float lt = t < Lc ? ((gs.layout & kLayerInputs) ? log_sigmoid_f(gs.la[tok]) : gs.la[tok]) : 0.f;
#pragma unroll
            for (int m = 0; m < 8; ++m)
                *reinterpret_cast<float4 *>(sm + L::LA + t * 512 + part * 128 + ((m + t) & 7) * 16) =
                    make_float4(lt, lt, lt, lt);
        }
    }
    // One thread polls each mbarrier; the others park on the group's barrier,
    // which leaves the issue slots to the co-resident group.  tcgen05.fence::after
    // orders the tensor-memory reads after that barrier.
    auto mma_done = [&]() {
        const bool mine = (tid == 0) ? mbar_wait(bar_mma, mma_phase, err) : true;
        mma_phase ^= 1;
        const bool all = named_bar_and(bar_id, kPrepThreads, mine) != 0;
        tc_fence_after();
        return all;
    };
    bool ok = named_bar_and(bar_id, kPrepThreads, (tid == 0) ? mbar_wait(bar_tma, tma_phase, err) : true) != 0;

    if (ok && (gs.layout & kLayerInputs)) prep_layer_inputs(sm, tid, bar_id, Lc, gs.layout);

    // Z = w v, straight into the record (MN-major operand blocks of 64 value
    // columns; each warp fills whole 128-byte rows)
    auto write_z = [&]() {
#pragma unroll
        for (int m = 0; m < ZV; ++m) {
            const int idx = tid + m * kPrepThreads;
            const int t = idx / (DV / 8), j = (idx % (DV / 8)) * 8;
            float fv[8], fw[8], fz[8];
            unpack8(vv[m], fv);
            unpack8(wv[m], fw);
#pragma unroll
            for (int u = 0; u < 8; ++u) fz[u] = fv[u] * fw[u];
            *reinterpret_cast<uint4 *>(rec + R::Z + (j >> 6) * 8192 + swz_off(t, (j & 63) * 2, 128)) = pack8(fz);
        }
    };
    bool exact = false;  // this chunk's decay is too strong for the midpoint reference

    if (ok) {
        // ---------------------------------------------------------- Gamma
        const int p = tid & 63, qr = tid >> 6;           // channel pair, token quarter
        float2 lv[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) lv[u] = *reinterpret_cast<const float2 *>(la + (qr * 16 + u) * kDK + 2 * p);
        float g0 = 0.f, g1 = 0.f;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            g0 += lv[u].x; g1 += lv[u].y;
            lv[u] = make_float2(g0, g1);
        }
        tot[qr * kDK + 2 * p] = g0;
        tot[qr * kDK + 2 * p + 1] = g1;
        // The split factors e^{+x} and e^{-x}, x = Gamma_t - Gamma_r around the
        // chunk midpoint, stay finite fp32/bf16 numbers for |x| <= 80.  Gamma only
        // decreases, so |x| is at most the decay of a half chunk, which is at most
        // e^{-80} when each quarter's is at most e^{-40}: the midpoint form then.
        // Otherwise (or not a number: log_alpha = -inf) the chunk takes the bounded form.
        exact = !named_bar_and(bar_id, kPrepThreads, (g0 >= -0.5f * kMidpointLogDecayRange) &&
                                                         (g1 >= -0.5f * kMidpointLogDecayRange));
        float pre0 = 0.f, pre1 = 0.f, gc0 = 0.f, gc1 = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float a0 = tot[q * kDK + 2 * p], a1 = tot[q * kDK + 2 * p + 1];
            if (q < qr) { pre0 += a0; pre1 += a1; }
            gc0 += a0; gc1 += a1;
        }
        // midpoint reference: Gamma after 32 tokens (tokens past T carry log_alpha = 0)
        const float gr0 = tot[2 * p] + tot[kDK + 2 * p], gr1 = tot[2 * p + 1] + tot[kDK + 2 * p + 1];
        const float sh0 = pre0 - gr0, sh1 = pre1 - gr1;  // x = lv + sh
        if (qr == 0)
            *reinterpret_cast<float2 *>(rec + R::DEC + 8 * p) = make_float2(expf(gc0), expf(gc1));

        if (!exact) {
            // ------------------------------------------------------ midpoint factors (in place)
            if (qr == 0) {
                dec[2 * p] = expf(gc0 - gr0);
                dec[2 * p + 1] = expf(gc1 - gr1);
                dec[kDK + 2 * p] = expf(gr0);
                dec[kDK + 2 * p + 1] = expf(gr1);
            }
#pragma unroll
            for (int u = 0; u < 16; ++u)
                *reinterpret_cast<float2 *>(la + (qr * 16 + u) * kDK + 2 * p) =
                    make_float2(lv[u].x + sh0, lv[u].y + sh1);
            named_bar(bar_id, kPrepThreads);
            // one 16-byte piece (8 channels of one token) of each swizzled tile per
            // step: Ehat over b, Qhat over q, Khat over k
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int idx = tid + m * kPrepThreads;
                const int t = idx >> 4, g = idx & 15, hb = g >> 3;  // token, channel group, 64-channel half tile
                const uint32_t off = swz_off(t, (g & 7) * 16, 128);
                uint8_t *ep = sm + L::EQ + hb * 16384 + off, *qp = ep + 8192, *kp = sm + L::KT + hb * 8192 + off;
                const float4 xa = *reinterpret_cast<const float4 *>(la + t * kDK + 8 * g);
                const float4 xb = *reinterpret_cast<const float4 *>(la + t * kDK + 8 * g + 4);
                const float x[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
                float kv[8], bv[8], qv[8], fe[8], fq[8], fk[8];
                unpack8(*reinterpret_cast<const uint4 *>(kp), kv);
                unpack8(*reinterpret_cast<const uint4 *>(ep), bv);
                unpack8(*reinterpret_cast<const uint4 *>(qp), qv);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float up = ex2_approx(x[u] * kLog2e), dn = ex2_approx(-x[u] * kLog2e);
                    fe[u] = up * bv[u] * kv[u];
                    fq[u] = up * qv[u];
                    fk[u] = dn * kv[u];
                }
                *reinterpret_cast<uint4 *>(ep) = pack8(fe);
                *reinterpret_cast<uint4 *>(qp) = pack8(fq);
                *reinterpret_cast<uint4 *>(kp) = pack8(fk);
            }
            fence_proxy_async_smem();
            named_bar(bar_id, kPrepThreads);

            // ------------------------------------------------------ Gram: [Ehat;Qhat] Khat^T
            if (tid == 0) {
                tc_fence_after();
                const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
                for (int ks = 0; ks < kDK / 16; ++ks) {
                    const uint32_t kofs = (ks & 3) * 32;
                    umma_bf16(tmem + L::TM_G, smem_desc(sbase + L::EQ + (ks >> 2) * 16384 + kofs, 16, 1024, kSw128),
                              smem_desc(sbase + L::KT + (ks >> 2) * 8192 + kofs, 16, 1024, kSw128), id, ks > 0);
                }
                umma_commit(bar_mma);
            }
            write_z();  // while the Gram runs
            ok = mma_done();
        } else {
            // ------------------------------------------------------ bounded form
            write_z();
            prep_bounded(sm, tid, bar_id);
        }
    }

    if (ok) {
        if (!exact) {
            // ------------------------------------------------------ A (fp32) and P (bf16) from the Gram
            const int r = wq * 32 + lane;
            float v[32];
            tmem_ld32_wait(tmem + lane_base + L::TM_GRAM + wh * 32, v);
            if (r < 64) {
                const int t = r;
#pragma unroll
                for (int s4 = 0; s4 < 32; s4 += 4) {
                    const int s = wh * 32 + s4;
                    float4 a4;
                    a4.x = (s + 0 < t) ? v[s4 + 0] : 0.f;
                    a4.y = (s + 1 < t) ? v[s4 + 1] : 0.f;
                    a4.z = (s + 2 < t) ? v[s4 + 2] : 0.f;
                    a4.w = (s + 3 < t) ? v[s4 + 3] : 0.f;
                    *reinterpret_cast<float4 *>(Af + af_off(t, s)) = a4;
                }
            } else {
                const int t = r - 64;
#pragma unroll
                for (int s8 = 0; s8 < 32; s8 += 8) {
                    float f[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) f[u] = (wh * 32 + s8 + u <= t) ? v[s8 + u] : 0.f;
                    *reinterpret_cast<uint4 *>(sm + L::PO + swz_off(t, (wh * 32 + s8) * 2, 128)) = pack8(f);
                }
            }
            // T starts as zero (log_alpha, consumed by the Gamma scan, gives its room to A and T)
#pragma unroll
            for (int m = 0; m < 4; ++m)
                reinterpret_cast<float4 *>(Tf)[tid + m * kPrepThreads] = make_float4(0.f, 0.f, 0.f, 0.f);
            tc_fence_before();
            named_bar(bar_id, kPrepThreads);
        }

        bool ill = false;  // (the backward) T far from the identity
        // ---------------------------------------------------------- T = (I + A)^{-1}
        // (a) diagonal 16x16 blocks: one column per thread, rows of A read as float4
        if (tid < 64) {
            const int b0 = (tid >> 4) * 16, j = tid & 15;
            float x[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                float a[16];
#pragma unroll
                for (int s4 = 0; s4 < 16; s4 += 4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(Af + af_off(b0 + t, b0 + s4));
                    a[s4] = a4.x; a[s4 + 1] = a4.y; a[s4 + 2] = a4.z; a[s4 + 3] = a4.w;
                }
                float acc0 = (t == j) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
                for (int s = 0; s < t; ++s) {
                    if (s & 1) acc1 -= a[s] * x[s];
                    else acc0 -= a[s] * x[s];
                }
                x[t] = acc0 + acc1;
                Tf[af_off(b0 + t, b0 + j)] = x[t];
            }
        }
        named_bar(bar_id, kPrepThreads);
        // (b), (c): the merges are small products inside a dependency chain; they
        // run as warp-level tf32 MMAs (m16n8k8) on the fp32 blocks.  g, c: fragment
        // coordinates of this lane.
        const int fg = lane >> 2, fc = lane & 3;
        // (b) T_{b+1,b} = -D_{b+1} (A_{b+1,b} D_b) for the pairs (0,1), (2,3).
        //     Warp w < 4: pair w >> 1, 8-column tile w & 1 of the 16x16 block.
        if (warp < 4) {
            const int which = warp >> 1, n0 = (warp & 1) * 8;
            const int R0 = 16 + 32 * which, C0 = 32 * which;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k0 = 0; k0 < 16; k0 += 8) {
                mma_tf32(d, to_tf32(Af[af_off(R0 + fg, C0 + k0 + fc)]), to_tf32(Af[af_off(R0 + fg + 8, C0 + k0 + fc)]),
                         to_tf32(Af[af_off(R0 + fg, C0 + k0 + fc + 4)]), to_tf32(Af[af_off(R0 + fg + 8, C0 + k0 + fc + 4)]),
                         to_tf32(Tf[af_off(C0 + k0 + fc, C0 + n0 + fg)]), to_tf32(Tf[af_off(C0 + k0 + fc + 4, C0 + n0 + fg)]));
            }
            float *x = Xs + which * 256;  // X[16][16]
            x[fg * 16 + n0 + 2 * fc] = d[0];
            x[fg * 16 + n0 + 2 * fc + 1] = d[1];
            x[(fg + 8) * 16 + n0 + 2 * fc] = d[2];
            x[(fg + 8) * 16 + n0 + 2 * fc + 1] = d[3];
        }
        named_bar(bar_id, kPrepThreads);
        if (warp < 4) {
            const int which = warp >> 1, n0 = (warp & 1) * 8;
            const int R0 = 16 + 32 * which, C0 = 32 * which;
            const float *x = Xs + which * 256;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k0 = 0; k0 < 16; k0 += 8) {
                mma_tf32(d, to_tf32(Tf[af_off(R0 + fg, R0 + k0 + fc)]), to_tf32(Tf[af_off(R0 + fg + 8, R0 + k0 + fc)]),
                         to_tf32(Tf[af_off(R0 + fg, R0 + k0 + fc + 4)]), to_tf32(Tf[af_off(R0 + fg + 8, R0 + k0 + fc + 4)]),
                         to_tf32(x[(k0 + fc) * 16 + n0 + fg]), to_tf32(x[(k0 + fc + 4) * 16 + n0 + fg]));
            }
            Tf[af_off(R0 + fg, C0 + n0 + 2 * fc)] = -d[0];
            Tf[af_off(R0 + fg, C0 + n0 + 2 * fc + 1)] = -d[1];
            Tf[af_off(R0 + fg + 8, C0 + n0 + 2 * fc)] = -d[2];
            Tf[af_off(R0 + fg + 8, C0 + n0 + 2 * fc + 1)] = -d[3];
        }
        named_bar(bar_id, kPrepThreads);
        // (c) T[32:64, 0:32] = -T_BB (A[32:64, 0:32] T_AA).  Warp w: 16-row tile w >> 2,
        //     8-column tile w & 3 of the 32x32 block; T_AA and T_BB are lower triangular.
        {
            const int m0 = (warp >> 2) * 16, n0 = (warp & 3) * 8;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k0 = 0; k0 < 32; k0 += 8) {
                if (k0 + 8 <= n0) continue;  // rows k of T_AA above column n0 are zero
                mma_tf32(d, to_tf32(Af[af_off(32 + m0 + fg, k0 + fc)]), to_tf32(Af[af_off(32 + m0 + fg + 8, k0 + fc)]),
                         to_tf32(Af[af_off(32 + m0 + fg, k0 + fc + 4)]), to_tf32(Af[af_off(32 + m0 + fg + 8, k0 + fc + 4)]),
                         to_tf32(Tf[af_off(k0 + fc, n0 + fg)]), to_tf32(Tf[af_off(k0 + fc + 4, n0 + fg)]));
            }
            Xs[(m0 + fg) * 32 + n0 + 2 * fc] = d[0];
            Xs[(m0 + fg) * 32 + n0 + 2 * fc + 1] = d[1];
            Xs[(m0 + fg + 8) * 32 + n0 + 2 * fc] = d[2];
            Xs[(m0 + fg + 8) * 32 + n0 + 2 * fc + 1] = d[3];
        }
        named_bar(bar_id, kPrepThreads);
        {
            const int m0 = (warp >> 2) * 16, n0 = (warp & 3) * 8;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k0 = 0; k0 < 32; k0 += 8) {
                if (k0 >= m0 + 16) continue;  // columns k of T_BB right of row m0 + 15 are zero
                mma_tf32(d, to_tf32(Tf[af_off(32 + m0 + fg, 32 + k0 + fc)]),
                         to_tf32(Tf[af_off(32 + m0 + fg + 8, 32 + k0 + fc)]),
                         to_tf32(Tf[af_off(32 + m0 + fg, 32 + k0 + fc + 4)]),
                         to_tf32(Tf[af_off(32 + m0 + fg + 8, 32 + k0 + fc + 4)]),
                         to_tf32(Xs[(k0 + fc) * 32 + n0 + fg]), to_tf32(Xs[(k0 + fc + 4) * 32 + n0 + fg]));
            }
            Tf[af_off(32 + m0 + fg, n0 + 2 * fc)] = -d[0];
            Tf[af_off(32 + m0 + fg, n0 + 2 * fc + 1)] = -d[1];
            Tf[af_off(32 + m0 + fg + 8, n0 + 2 * fc)] = -d[2];
            Tf[af_off(32 + m0 + fg + 8, n0 + 2 * fc + 1)] = -d[3];
        }
        named_bar(bar_id, kPrepThreads);
        // (d) T -> bf16 operand over A (which has served its purpose)
        {
            const int t = tid >> 2, g = (tid & 3) * 16;
            float f[16];
#pragma unroll
            for (int u = 0; u < 16; u += 4) {
                const float4 v4 = *reinterpret_cast<const float4 *>(Tf + af_off(t, g + u));
                f[u] = v4.x; f[u + 1] = v4.y; f[u + 2] = v4.z; f[u + 3] = v4.w;
            }
            *reinterpret_cast<uint4 *>(sm + L::TB + swz_off(t, g * 2, 128)) = pack8(f);
            *reinterpret_cast<uint4 *>(sm + L::TB + swz_off(t, g * 2 + 16, 128)) = pack8(f + 8);
            if (TP) {
#pragma unroll
                for (int u = 0; u < 16; ++u) ill = ill || fabsf(f[u] - (g + u == t ? 1.f : 0.f)) > kIllT;
            }
        }
        fence_proxy_async_smem();
        if (TP)
            ill = !named_bar_and(bar_id, kPrepThreads, !ill);
        else
            named_bar(bar_id, kPrepThreads);
        if (TP && ill) {  // what the bf16 image of T drops (the fp32 T is still in place)
            const int t = tid >> 2, g = (tid & 3) * 16;
            float f[16];
#pragma unroll
            for (int u = 0; u < 16; u += 4) {
                const float4 v4 = *reinterpret_cast<const float4 *>(Tf + af_off(t, g + u));
                f[u] = v4.x; f[u + 1] = v4.y; f[u + 2] = v4.z; f[u + 3] = v4.w;
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) f[u] -= __bfloat162float(__float2bfloat16_rn(f[u]));
            *reinterpret_cast<uint4 *>(tp + 16384 + swz_off(t, g * 2, 128)) = pack8(f);
            *reinterpret_cast<uint4 *>(tp + 16384 + swz_off(t, g * 2 + 16, 128)) = pack8(f + 8);
        }
        if (TP && tid == 0) *reinterpret_cast<uint32_t *>(rec + R::DEC + 512) = ill ? 1u : 0u;
        if (TP) {  // T and P, final from here on, for the backward
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int idx = tid + m * kPrepThreads;
                reinterpret_cast<uint4 *>(tp)[idx] = reinterpret_cast<const uint4 *>(sm + L::TB)[idx];
                reinterpret_cast<uint4 *>(tp + 8192)[idx] = reinterpret_cast<const uint4 *>(sm + L::PO)[idx];
            }
        }

        // ---------------------------------------------------------- Khat^T T (M = 128),  PT = P T (M = 64)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idy = idesc_bf16(128, 64, 1, 1), idp = idesc_bf16(64, 64, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t bt = smem_desc(sbase + L::TB + ks * 2048, 8192, 1024, kSw128);
                umma_bf16(tmem + L::TM_Y, smem_desc(sbase + L::KT + ks * 2048, 8192, 1024, kSw128), bt, idy, ks > 0);
                umma_bf16(tmem + L::TM_PT, smem_desc(sbase + L::PO + ks * 32, 16, 1024, kSw128), bt, idp, ks > 0);
            }
            umma_commit(bar_mma);
        }
        ok = mma_done();
    }

    if (ok) {
        {   // Y row i, K chunks [4*wh, +4) -> KH and the record;  PT (M = 64: row 16*wq + l
            // in TMEM lane 32*wq + l) -> KT and the record.  No-swizzle K-major tiles.
            float v[32], p[32];
            tmem_ld32(tmem + lane_base + L::TM_Y + wh * 32, v);
            tmem_ld32(tmem + lane_base + L::TM_PT + wh * 32, p);
            tmem_ld_wait();
            const int i = wq * 32 + lane, t = wq * 16 + lane;
            const float ecr = dec[i];
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] *= ecr;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int c = wh * 4 + q;
                const uint4 y = pack8(v + 8 * q);
                *reinterpret_cast<uint4 *>(sm + L::KH + kchunk_off(c, i, 128)) = y;
                *reinterpret_cast<uint4 *>(rec + R::Y + kchunk_off(c, i, 128)) = y;
                if (lane < 16) {
                    const uint4 pt = pack8(p + 8 * q);
                    *reinterpret_cast<uint4 *>(sm + L::KT + kchunk_off(c, t, 64)) = pt;
                    *reinterpret_cast<uint4 *>(rec + R::PT + kchunk_off(c, t, 64)) = pt;
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        named_bar(bar_id, kPrepThreads);

        // ---------------------------------------------------------- G = Y Ehat (M = 128),  PW = PT Ehat (M = 64)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idg = idesc_bf16(128, kDK, 0, 1), idw = idesc_bf16(64, kDK, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t be = smem_desc(sbase + L::EQ + ks * 2048, 16384, 1024, kSw128);
                umma_bf16(tmem + L::TM_G, smem_desc(sbase + L::KH + ks * 4096, 2048, 128, kSwNone), be, idg, ks > 0);
                umma_bf16(tmem + L::TM_PW, smem_desc(sbase + L::KT + ks * 2048, 1024, 128, kSwNone), be, idw, ks > 0);
            }
            umma_commit(bar_mma);
        }
        ok = mma_done();
    }

    if (ok) {
        const float *er = dec + kDK;
        {   // NG = -G Diag(e^{Gamma_r}): row i, K chunks [8*wh, +8) -> the record
            const int i = wq * 32 + lane;
            float v[64];
            tmem_ld32(tmem + lane_base + L::TM_G + wh * 64, *reinterpret_cast<float(*)[32]>(v));
            tmem_ld32(tmem + lane_base + L::TM_G + wh * 64 + 32, *reinterpret_cast<float(*)[32]>(v + 32));
            tmem_ld_wait();
#pragma unroll
            for (int s8 = 0; s8 < 64; s8 += 8) {
                const int j = wh * 64 + s8;
                const float4 e0 = *reinterpret_cast<const float4 *>(er + j);
                const float4 e1 = *reinterpret_cast<const float4 *>(er + j + 4);
                float f[8] = {-v[s8] * e0.x,     -v[s8 + 1] * e0.y, -v[s8 + 2] * e0.z, -v[s8 + 3] * e0.w,
                              -v[s8 + 4] * e1.x, -v[s8 + 5] * e1.y, -v[s8 + 6] * e1.z, -v[s8 + 7] * e1.w};
                *reinterpret_cast<uint4 *>(rec + R::NG + kchunk_off(j >> 3, i, 128)) = pack8(f);
            }
        }
        {   // QS = (Qhat - PT Ehat) Diag(e^{Gamma_r}) -> the record (M = 64 accumulator)
            const int t = wq * 16 + lane;
#pragma unroll
            for (int part = 0; part < 64; part += 32) {
                float v[32];
                tmem_ld32_wait(tmem + lane_base + L::TM_PW + wh * 64 + part, v);
                if (lane < 16) {
#pragma unroll
                    for (int s8 = 0; s8 < 32; s8 += 8) {
                        const int j = wh * 64 + part + s8;
                        const uint4 *qp = reinterpret_cast<const uint4 *>(sm + L::EQ + wh * 16384 + 8192 +
                                                                          swz_off(t, (part + s8) * 2, 128));
                        float qh[8], f[8];
                        unpack8(*qp, qh);
                        const float4 e0 = *reinterpret_cast<const float4 *>(er + j);
                        const float4 e1 = *reinterpret_cast<const float4 *>(er + j + 4);
                        const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
#pragma unroll
                        for (int u = 0; u < 8; ++u) f[u] = (qh[u] - v[s8 + u]) * ev[u];
                        *reinterpret_cast<uint4 *>(rec + R::QS + kchunk_off(j >> 3, t, 64)) = pack8(f);
                    }
                }
            }
        }
    }
    return ok;
}

}  // namespace prep
}  // namespace gdn2
