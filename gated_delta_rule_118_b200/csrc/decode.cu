// decode.cu -- single-token recurrent update with the fp32 state resident in HBM.
//
// One token of the gated delta rule with decoupled erase/write gates
// ("Gated DeltaNet-2", iplexlaw.co.kr, section "Decisiones independientes en dos
// ejes"): Sbar = Diag(alpha) S, r = Sbar^T (b*k), S = Sbar + k (w*v - r)^T,
// o = S^T q.  Decoding keeps this fixed-size state instead of a growing cache
// (gist.science, "Problem Statement").
//
// The pass is bound by HBM: each (batch, head) state is read once and written
// once.  One CTA owns one state.  Its threads own float4 column strips (lanes
// run along the contiguous value axis, so every warp access is a full
// 512-byte row), each thread holding DK/RPP rows of its strip in registers
// between the two reductions.  Both reductions run over the key axis: first
// inside each thread, then across the row groups through shared memory.
#include "common.cuh"
#include "launch.h"

namespace gdn2 {
namespace {

constexpr int kDecodeThreads = 256;

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kDecodeThreads, 2)
decode_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
              const T *__restrict__ b, const T *__restrict__ w, const float *__restrict__ log_alpha,
              float *__restrict__ S, T *__restrict__ o)
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

    // Per-key-channel scalars: decay, erase key, write key and query.
    for (int i = tid; i < DK; i += kDecodeThreads) {
        const long off = bh * DK + i;
        const float kv = to_f32(k[off]);
        s_k[i] = kv;
        s_e[i] = to_f32(b[off]) * kv;
        s_a[i] = expf(log_alpha[off]);
        s_q[i] = to_f32(q[off]);
    }
    const float4 vv = load4(v + bh * DV + 4 * c4);
    const float4 ww = load4(w + bh * DV + 4 * c4);
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

template <typename T, int DK, int DV>
cudaError_t launch(const DecodeArgs &a)
{
    const long nbh = (long)a.B * a.H;
    decode_kernel<T, DK, DV><<<(unsigned)nbh, kDecodeThreads, 0, a.stream>>>(
        (const T *)a.q, (const T *)a.k, (const T *)a.v, (const T *)a.b, (const T *)a.w,
        a.log_alpha, a.S, (T *)a.o);
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
