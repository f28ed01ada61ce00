// decode.cu -- recurrent updates with the fp32 state resident in HBM: one token
// (gdn2_decode_step) or a short run of tokens (gdn2_decode_tokens).
//
// Per token, the gated delta rule with decoupled erase/write gates
// ("Gated DeltaNet-2", iplexlaw.co.kr, section "Decisiones independientes en dos
// ejes"): Sbar = Diag(alpha) S, r = Sbar^T (b*k), S = Sbar + k (w*v - r)^T,
// o = S^T q.  Decoding keeps this fixed-size state instead of a growing cache
// (gist.science, "Problem Statement").
//
// The pass is bound by HBM: each (batch, head) state is read once and written
// once per call, whatever the number of tokens.  One CTA owns one state.  Its
// threads own float4 column strips (lanes run along the contiguous value axis,
// so every warp access is a full 512-byte row), each thread holding DK/RPP rows
// of its strip in registers for the whole call.  Both reductions of a token
// run over the key axis: inside each thread, then across the row groups
// through shared memory.
//
// One token (gdn2_decode_step): the erase read r and the output o in turn.
// A run of tokens (gdn2_decode_tokens): both reductions read the same state,
// o_t = S_t^T q_t and the next token's erase read
// r_{t+1} = (Diag(alpha_{t+1}) S_t)^T e_{t+1} = S_t^T (alpha_{t+1} * e_{t+1}),
// so each token takes one combined reduction (a double-buffered shared array:
// one barrier per token), plus one for r_1 before the first token.
//
// Gate layouts (gdn2_gate_layout): b, w or log_alpha may hold one value per
// (token, head) instead of one per channel; the loads broadcast it.
#include "common.cuh"
#include "gdn2.h"
#include "launch.h"

namespace gdn2 {
namespace {

constexpr int kDecodeThreads = 256;
constexpr int kTokBatch = 8;  // tokens whose inputs are staged in shared memory at a time

// One token (T = 1): the two reductions in turn, with the state's loads issued
// before anything else.
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kDecodeThreads, 2)
decode_step_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
              const T *__restrict__ b, const T *__restrict__ w, const float *__restrict__ log_alpha,
              float *__restrict__ S, T *__restrict__ o, unsigned layout)
{
    constexpr int TPR = DV / 4;                  // threads per state row (one float4 each)
    constexpr int RPP = kDecodeThreads / TPR;    // row groups
    constexpr int RPT = DK / RPP;                // rows held by each thread
    static_assert(DK % RPP == 0, "row split");

    __shared__ float s_k[DK], s_e[DK], s_a[DK], s_q[DK];
    __shared__ float4 s_red[RPP][TPR];

    const long bh = blockIdx.x;
    const int tid = threadIdx.x;
    const int c4 = tid % TPR;
    const int rg = tid / TPR;
    float *Sp = S + bh * (long)DK * DV;

    // Issue every state load of this thread first: they are the long-latency part.
    float4 s[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int i = rg * RPT + m;
        s[m] = __ldcs(reinterpret_cast<const float4 *>(Sp + (long)i * DV) + c4);
    }

    // Per-key-channel scalars: decay, erase key, write key and query (a gate
    // given per (batch, head) is broadcast over the channels).
    for (int i = tid; i < DK; i += kDecodeThreads) {
        const long off = bh * DK + i;
        const float kv = to_f32(k[off]);
        s_k[i] = kv;
        s_e[i] = to_f32(b[(layout & GDN2_ERASE_SCALAR) ? bh : off]) * kv;
        s_a[i] = expf(log_alpha[(layout & GDN2_DECAY_SCALAR) ? bh : off]);
        s_q[i] = to_f32(q[off]);
    }
    const float4 vv = load4(v + bh * DV + 4 * c4);
    float4 ww;
    if (layout & GDN2_WRITE_SCALAR) {
        const float ws = to_f32(w[bh]);
        ww = make_float4(ws, ws, ws, ws);
    } else {
        ww = load4(w + bh * DV + 4 * c4);
    }
    const float4 z = make_float4(ww.x * vv.x, ww.y * vv.y, ww.z * vv.z, ww.w * vv.w);
    __syncthreads();

    // Sbar = Diag(alpha) S; partial r = Sbar^T e over this thread's rows.
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int i = rg * RPT + m;
        const float a = s_a[i], e = s_e[i];
        s[m].x *= a; s[m].y *= a; s[m].z *= a; s[m].w *= a;
        r.x += e * s[m].x; r.y += e * s[m].y; r.z += e * s[m].z; r.w += e * s[m].w;
    }
    s_red[rg][c4] = r;
    __syncthreads();
    r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int g = 0; g < RPP; ++g) {
        const float4 p = s_red[g][c4];
        r.x += p.x; r.y += p.y; r.z += p.z; r.w += p.w;
    }
    const float4 u = make_float4(z.x - r.x, z.y - r.y, z.z - r.z, z.w - r.w);

    // S = Sbar + k u^T, stored in place; partial o = S^T q.
    float4 oo = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int i = rg * RPT + m;
        const float kk = s_k[i], qq = s_q[i];
        s[m].x += kk * u.x; s[m].y += kk * u.y; s[m].z += kk * u.z; s[m].w += kk * u.w;
        oo.x += qq * s[m].x; oo.y += qq * s[m].y; oo.z += qq * s[m].z; oo.w += qq * s[m].w;
        __stcs(reinterpret_cast<float4 *>(Sp + (long)i * DV) + c4, s[m]);
    }
    __syncthreads();  // every thread has read s_red
    s_red[rg][c4] = oo;
    __syncthreads();
    if (rg == 0) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int g = 0; g < RPP; ++g) {
            const float4 p = s_red[g][c4];
            acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
        }
        store4(o + bh * DV + 4 * c4, acc);
    }
}

// A run of T tokens: one combined reduction per token.
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kDecodeThreads, 2)
decode_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
              const T *__restrict__ b, const T *__restrict__ w, const float *__restrict__ log_alpha,
              float *__restrict__ S, T *__restrict__ o, int Tn, int H, unsigned layout)
{
    constexpr int TPR = DV / 4;                  // threads per state row (one float4 each)
    constexpr int RPP = kDecodeThreads / TPR;    // row groups
    constexpr int RPT = DK / RPP;                // rows held by each thread
    constexpr int NB = kTokBatch + 1;            // a batch plus the next token (look-ahead)
    static_assert(DK % RPP == 0, "row split");

    // per staged token: alpha, k, q, alpha * e (e = b * k), z = w * v
    __shared__ __align__(16) float s_a[NB][DK], s_k[NB][DK], s_q[NB][DK], s_ae[NB][DK];
    static_assert(RPT % 4 == 0, "rows per thread in float4 groups");
    __shared__ float4 s_z[NB][TPR];
    __shared__ float4 s_red[2][2][RPP][TPR];     // [buffer][r | o][row group][column strip]

    const long bh = blockIdx.x;
    const long bi = bh / H, h = bh % H;
    const int tid = threadIdx.x;
    const int c4 = tid % TPR;
    const int rg = tid / TPR;
    float *Sp = S + bh * (long)DK * DV;
    const bool b_scalar = layout & GDN2_ERASE_SCALAR, w_scalar = layout & GDN2_WRITE_SCALAR,
               a_scalar = layout & GDN2_DECAY_SCALAR;

    // Issue every state load of this thread first: they are the long-latency part.
    float4 s[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int i = rg * RPT + m;
        s[m] = __ldcs(reinterpret_cast<const float4 *>(Sp + (long)i * DV) + c4);
    }

    // Stage the inputs of tokens [t0, min(t0 + NB, Tn)) into slots 0.. (the
    // last slot of a batch is the first token of the next).
    auto stage = [&](int t0) {
        const int n = min(NB, Tn - t0);
        for (int idx = tid; idx < n * DK; idx += kDecodeThreads) {
            const int j = idx / DK, i = idx % DK;
            const long tok = (bi * Tn + t0 + j) * H + h;  // (batch, token, head)
            const long off = tok * DK + i;
            const float kv = to_f32(k[off]);
            const float a = expf(log_alpha[a_scalar ? tok : off]);
            s_a[j][i] = a;
            s_k[j][i] = kv;
            s_q[j][i] = to_f32(q[off]);
            s_ae[j][i] = a * to_f32(b[b_scalar ? tok : off]) * kv;
        }
        for (int idx = tid; idx < n * TPR; idx += kDecodeThreads) {
            const int j = idx / TPR, c = idx % TPR;
            const long tok = (bi * Tn + t0 + j) * H + h;
            const float4 vv = load4(v + tok * DV + 4 * c);
            float4 ww;
            if (w_scalar) {
                const float ws = to_f32(w[tok]);
                ww = make_float4(ws, ws, ws, ws);
            } else {
                ww = load4(w + tok * DV + 4 * c);
            }
            s_z[j][c] = make_float4(ww.x * vv.x, ww.y * vv.y, ww.z * vv.z, ww.w * vv.w);
        }
    };
    // Sum over the row groups of one partial (every thread, its column strip).
    auto gather = [&](int buf, int which) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int g = 0; g < RPP; ++g) {
            const float4 p = s_red[buf][which][g][c4];
            acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
        }
        return acc;
    };

    stage(0);
    __syncthreads();
    // r_1 = S_0^T (alpha_1 * e_1)
    {
        float4 pr = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const float ae = s_ae[0][rg * RPT + m];
            pr.x += ae * s[m].x; pr.y += ae * s[m].y; pr.z += ae * s[m].z; pr.w += ae * s[m].w;
        }
        s_red[1][0][rg][c4] = pr;
    }
    __syncthreads();
    float4 r = gather(1, 0);

    int slot = 0;
    for (int t = 0; t < Tn; ++t, ++slot) {
        if (slot == kTokBatch) {  // the next batch: this token moves to slot 0
            __syncthreads();      // every thread is done with the staged inputs
            stage(t);
            __syncthreads();
            slot = 0;
        }
        const int buf = t & 1;
        const bool next = t + 1 < Tn;
        const float4 z = s_z[slot][c4];
        const float4 u = make_float4(z.x - r.x, z.y - r.y, z.z - r.z, z.w - r.w);
        // S_t = Diag(alpha_t) S_{t-1} + k_t u^T; partial o_t and r_{t+1}
        float4 po = make_float4(0.f, 0.f, 0.f, 0.f), pr = make_float4(0.f, 0.f, 0.f, 0.f);
        // the per-row scalars of this thread's rows, four rows per shared load
        // (every lane of a warp reads the same rows: broadcasts)
#pragma unroll
        for (int m4 = 0; m4 < RPT; m4 += 4) {
            const int i0 = rg * RPT + m4;
            const float4 a4 = *reinterpret_cast<const float4 *>(&s_a[slot][i0]);
            const float4 k4 = *reinterpret_cast<const float4 *>(&s_k[slot][i0]);
            const float4 q4 = *reinterpret_cast<const float4 *>(&s_q[slot][i0]);
            const float4 e4 = next ? *reinterpret_cast<const float4 *>(&s_ae[slot + 1][i0])
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
            const float av[4] = {a4.x, a4.y, a4.z, a4.w}, kv[4] = {k4.x, k4.y, k4.z, k4.w};
            const float qv[4] = {q4.x, q4.y, q4.z, q4.w}, ev[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float4 &x = s[m4 + j];
                const float a = av[j], kk = kv[j], qq = qv[j], ae = ev[j];
                x.x = a * x.x + kk * u.x; x.y = a * x.y + kk * u.y;
                x.z = a * x.z + kk * u.z; x.w = a * x.w + kk * u.w;
                po.x += qq * x.x; po.y += qq * x.y; po.z += qq * x.z; po.w += qq * x.w;
                pr.x += ae * x.x; pr.y += ae * x.y; pr.z += ae * x.z; pr.w += ae * x.w;
            }
        }
        if (!next) {
#pragma unroll
            for (int m = 0; m < RPT; ++m)
                __stcs(reinterpret_cast<float4 *>(Sp + (long)(rg * RPT + m) * DV) + c4, s[m]);
        }
        s_red[buf][0][rg][c4] = pr;
        s_red[buf][1][rg][c4] = po;
        __syncthreads();
        if (next) r = gather(buf, 0);
        if (rg == 0) store4(o + ((bi * Tn + t) * H + h) * DV + 4 * c4, gather(buf, 1));
    }
}

template <typename T, int DK, int DV>
cudaError_t launch(const DecodeArgs &a)
{
    const long nbh = (long)a.B * a.H;
    if (a.T == 1) {
        decode_step_kernel<T, DK, DV><<<(unsigned)nbh, kDecodeThreads, 0, a.stream>>>(
            (const T *)a.q, (const T *)a.k, (const T *)a.v, (const T *)a.b, (const T *)a.w,
            a.log_alpha, a.S, (T *)a.o, a.layout);
        return cudaGetLastError();
    }
    decode_kernel<T, DK, DV><<<(unsigned)nbh, kDecodeThreads, 0, a.stream>>>(
        (const T *)a.q, (const T *)a.k, (const T *)a.v, (const T *)a.b, (const T *)a.w,
        a.log_alpha, a.S, (T *)a.o, a.T, a.H, a.layout);
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_dims(const DecodeArgs &a)
{
    if (a.dk == 128 && a.dv == 128) return launch<T, 128, 128>(a);
    if (a.dk == 128 && a.dv == 64) return launch<T, 128, 64>(a);
    if (a.dk == 64 && a.dv == 128) return launch<T, 64, 128>(a);
    return launch<T, 64, 64>(a);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a)
{
    if (a.bf16) return dispatch_dims<__nv_bfloat16>(a);
    return dispatch_dims<float>(a);
}

}  // namespace gdn2
