// out_body.cuh -- the outputs of one chunk, shared by the windowed output
// kernel (fwd_out.cu) and the persistent forward (fwd_persist.cu).
//
// The query reads the updated state ("Gated DeltaNet-2", iplexlaw.co.kr,
// section "Decisiones independientes en dos ejes"); in the chunkwise form the
// outputs of a chunk are
//   O = P T Z + (Qhat - P T Ehat) Diag(e^{Gamma_r}) S = PT Z + QS Sx,
// with PT, Z and QS from the chunk's prep record and Sx the bf16 image of the
// incoming state exported by the chain.  Nothing here is sequential in the
// chunk index: the two products accumulate in tensor memory (M = 64 tokens,
// N = dv; K = 64 tokens, then K = dk) and the 64 output rows are written.
#pragma once

#include "tc_common.cuh"

namespace gdn2 {
namespace outp {

using namespace sm100;

template <int DV>
struct OutLayout {
    static constexpr int QS = 0;                    // QS [64][128] K-major, no swizzle
    static constexpr int PT = 16384;                // PT [64][64] K-major, no swizzle
    static constexpr int Z = 24576;                 // Z, DV/64 blocks of [64][64] (MN-major)
    static constexpr int SX = Z + 64 * DV * 2;      // Sx [128][DV] (MN-major, no swizzle)
    static constexpr int TX = SX + 128 * DV * 2;    // bytes of one chunk's loads (plain outputs)
    // layer outputs: the chunk's output-gate logits, DV/64 blocks of [64 tokens][64]
    // with the 128-byte swizzle (TMA), and per-row sums of squares [2][64] fp32
    static constexpr int GT = TX;
    static constexpr int TX_LAYER = TX + 64 * DV * 2;
    static constexpr int RED = TX_LAYER;
    static constexpr int DATA = RED + 512;          // end of the buffers
    static_assert(GT % 1024 == 0, "swizzle atoms");
    static constexpr uint32_t TMEM_COLS = DV;
    static_assert(SX % 1024 == 0, "swizzle atoms");
};

// The loads of one chunk's operands (record pieces and state image, and with
// `tm_g` the output-gate logits of tokens [t0, t0 + 64) of head h, batch bi)
// into an OutLayout region, completing on `bar_ld` (issued by one thread).
template <int DV>
__device__ __forceinline__ void out_issue_loads(uint8_t *sm, uint64_t *bar_ld, const uint8_t *rec, const uint8_t *sx,
                                                const CUtensorMap *tm_g = nullptr, int t0 = 0, int h = 0, int bi = 0)
{
    using L = OutLayout<DV>;
    using R = Record<DV>;
    mbar_arrive_expect_tx(bar_ld, (uint32_t)(tm_g ? L::TX_LAYER : L::TX));
    if (tm_g)
        for (int kb = 0; kb < DV / 64; ++kb) tma_load_4d(sm + L::GT + kb * 8192, tm_g, bar_ld, kb * 64, h, t0, bi);
    bulk_load(sm + L::QS, rec + R::QS, 16384, bar_ld);
    bulk_load(sm + L::PT, rec + R::PT, 8192, bar_ld);
    bulk_load(sm + L::Z, rec + R::Z, 64 * DV * 2, bar_ld);
    bulk_load(sm + L::SX, sx, 128 * DV * 2, bar_ld);
}

// The layer's output processing (gdn2_layer_fwd): each output row o (over the
// value axis) becomes y = o / sqrt(mean(o^2) + eps) * weight * sigmoid(g)
// ("Gated DeltaNet-2", iplexlaw.co.kr, section "Procesamiento del token y
// entrenamiento paralelo": RMS normalisation and an independent output gate).
// g == nullptr: the operator's plain outputs.
struct OutEpi {
    const void *g;        // non-null: the output-gate logits were loaded with the chunk (OutLayout::GT)
    const float *weight;  // [DV]
    float eps;
};

// sigmoid(x) = (1 + tanh(x / 2)) / 2, one MUFU operation (tanh.approx.f32: its
// relative error, about 2^-11, is below the rounding of a bf16 output)
__device__ __forceinline__ float sigmoid_tanh(float x)
{
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
}

// The outputs of one chunk by NT (128 or 256) threads tid = 0.. sharing named
// barrier `bar_id`, once out_issue_loads has been issued: `tmem` is the first
// of DV tensor-memory columns, `bar_mma` an mbarrier for UMMA completion, and
// `phase` the parity both mbarriers are at (advanced here).  Rows t < `live`
// of the chunk are written to dst + t * row_stride.  Returns false (every
// thread alike) when a wait timed out.
template <int DV, int NT>
__device__ __forceinline__ bool out_chunk(uint8_t *sm, uint32_t tmem, int tid, int bar_id, uint64_t *bar_ld,
                                          uint64_t *bar_mma, uint32_t &phase, bf16 *__restrict__ dst, int live,
                                          long row_stride, const OutEpi &epi, unsigned int *err)
{
    static_assert(NT == 128 || NT == 256, "one or two warps per TMEM lane quarter");
    using L = OutLayout<DV>;
    constexpr int CW = DV / (NT / 128);  // output columns per warp
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t sbase = smem_u32(sm);

    bool ok = (tid == 0) ? mbar_wait(bar_ld, phase, err) : true;
    if (tid == 0 && ok) {
        tc_fence_after();
        const uint32_t id = idesc_bf16(64, DV, 0, 1);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            umma_bf16(tmem, smem_desc(sbase + L::PT + ks * 2048, 1024, 128, kSwNone),
                      smem_desc(sbase + L::Z + ks * 2048, 8192, 1024, kSw128), id, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            umma_bf16(tmem, smem_desc(sbase + L::QS + ks * 2048, 1024, 128, kSwNone),
                      smem_desc(sbase + L::SX + ks * 256, 128, 2048, kSwNone), id, 1);
        umma_commit(bar_mma);
        ok = mbar_wait(bar_mma, phase, err);
    }
    phase ^= 1;
    ok = named_bar_and(bar_id, NT, ok);
    if (ok) {
        tc_fence_after();
        // M = 64 accumulator: row 16*q + l sits in TMEM lane 32*q + l (l < 16) of lane quarter q
        const int q = warp & 3, c0 = (warp >> 2) * CW;
        const int t = q * 16 + lane;
        const bool on = lane < 16 && t < live;
        bf16 *row = dst + (long)t * row_stride + c0;
        const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16) + c0;
        if (epi.g == nullptr) {
#pragma unroll
            for (int j = 0; j < CW; j += 32) {
                float a[16], b[16];
                tmem_ld16(lane_addr + j, a);
                tmem_ld16(lane_addr + j + 16, b);
                tmem_ld_wait();
                if (on) {
                    *reinterpret_cast<uint4 *>(row + j) = pack8(a);
                    *reinterpret_cast<uint4 *>(row + j + 8) = pack8(a + 8);
                    *reinterpret_cast<uint4 *>(row + j + 16) = pack8(b);
                    *reinterpret_cast<uint4 *>(row + j + 24) = pack8(b + 8);
                }
            }
        } else {
            // the row's sum of squares (fp32, from the accumulator), over the
            // NT / 128 warps that hold its columns
            float ss = 0.f;
#pragma unroll 1
            for (int j = 0; j < CW; j += 16) {
                float a[16];
                tmem_ld16(lane_addr + j, a);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 16; ++u) ss = fmaf(a[u], a[u], ss);
            }
            if (NT == 256) {
                float *red = reinterpret_cast<float *>(sm + L::RED);
                if (lane < 16) red[(warp >> 2) * 64 + t] = ss;
                named_bar(bar_id, NT);
                if (lane < 16) ss = red[t] + red[64 + t];
            }
            const float inv = rsqrtf(ss * (1.f / DV) + epi.eps);
#pragma unroll 1
            for (int j = 0; j < CW; j += 16) {
                float a[16];
                tmem_ld16(lane_addr + j, a);
                tmem_ld_wait();
                if (on) {
#pragma unroll
                    for (int u = 0; u < 16; u += 8) {
                        const int col = c0 + j + u;
                        float gv[8];
                        unpack8(*reinterpret_cast<const uint4 *>(sm + L::GT + (col >> 6) * 8192 +
                                                                 swz_off(t, (col & 63) * 2, 128)), gv);
                        const float4 w0 = __ldg(reinterpret_cast<const float4 *>(epi.weight + col));
                        const float4 w1 = __ldg(reinterpret_cast<const float4 *>(epi.weight + col + 4));
                        const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) y[e] = a[u + e] * inv * wv[e] * sigmoid_tanh(gv[e]);
                        *reinterpret_cast<uint4 *>(row + j + u) = pack8(y);
                    }
                }
            }
        }
    }
    return ok;
}

}  // namespace outp
}  // namespace gdn2
