// chain_body.cuh -- the state-carrying part of the chunkwise forward, shared by
// the windowed chain kernel (fwd_chain.cu) and the persistent forward
// (fwd_persist.cu).
//
// The chunks of a sequence are passed in order, the state of one chunk being
// the input of the next ("Gated DeltaNet-2", iplexlaw.co.kr, section
// "Procesamiento del token y entrenamiento paralelo").  With the prep records
// of prep_body.cuh one chunk is an affine map of the state:
//   S <- e^{Gamma_C} S + D,    D = Y Z + NG Sx,    Sx = bf16(S)
// D is accumulated in tensor memory by two groups of tcgen05 UMMAs: Y Z (4
// instructions, M = dk, K = 64 tokens) does not depend on the state and is
// issued a chunk ahead; NG Sx (8 instructions, K = dk) is the only tensor-core
// work on the serial path.  The state stays fp32 in registers; its bf16 image
// Sx goes to shared memory (operand of the next UMMA) and to the workspace,
// where the outputs are computed from it.
//
// One CTA owns one (batch, head, DVT-wide value tile); a whole 128-column tile
// costs the tensor core about as much per instruction as a narrow one, so wide
// tiles keep the number of SMs on the serial path small.  Warp roles:
//   warps 0-7  state: thread (i, g) owns key row i, columns [g*COLS, +COLS)
//   warp  8    issues NG Sx (one elected lane)
//   warp  9    producer: streams the records through a ring of shared stages
//   warp  10   issues Y Z (one elected lane)
//   warp  11   publisher (flows that publish progress): tells the workspace's
//              other users how far the exported state images go
// The serial path per chunk is: UMMA completion -> tensor-memory load and state
// update -> Sx to shared memory -> one mbarrier arrival per state warp -> UMMA
// issue.  Everything else (the Sx export, stage refills, the next Y Z, the
// progress flags and their fences) runs beside it: after their arrival the
// state warps store Sx(c) to the workspace with plain vector stores (its slot is
// free once the producer has seen record c ready), count the stores in shared
// memory, and the publisher turns the count into a release of a flag in global
// memory every kPublishEvery chunks.
// A stage carries the chunk's NG, Y, Z tile and decays e^{Gamma_C}; it is
// refilled once the UMMAs have read it and every state warp has taken its
// decays.  Issuing a UMMA blocks the issuing thread while the tensor pipe is
// busy, so the two groups of UMMAs come from different warps, ordered by
// mbarriers: NG Sx of chunk c issued -> Y Z of chunk c + 1 (queued right behind
// it, it runs beside the epilogue of chunk c) -> Y Z done -> NG Sx of chunk c + 1.
//
// Where the records come from and where the state images go is the Flow's
// business: a window of records that are all ready before the chain starts
// (WindowFlow), or rings that the chain shares with concurrent prep and output
// work, with flags in global memory (fwd_persist.cu).
//
// The adjoint chain of the backward (ADJ) walks the same records in reverse.
// The gradient dS of the state entering a chunk follows from the gradient dS'
// of the state leaving it and the chunk's output gradients dO by the transpose
// of the chunk's map:
//   dS = e^{Gamma_C} dS' + NG^T dS'x + QS^T dO,    dS'x = bf16(dS')
// NG^T and QS^T are the record's NG and QS read as MN-major operands (the same
// bytes), dO comes by TMA in Z's place, and the exported images are those of
// dS' for every chunk.
#pragma once

#include "tc_common.cuh"

namespace gdn2 {
namespace chain {

using namespace sm100;

constexpr int kStateWarps = 8;
constexpr int kMmaWarp = kStateWarps, kProducerWarp = kStateWarps + 1, kYzWarp = kStateWarps + 2;
constexpr int kPublishWarp = kStateWarps + 3;
constexpr int kChainThreads = 32 * (kStateWarps + 4);
constexpr int kPublishEvery = 2;  // chunks per progress release (each costs a GPU-scope fence)
constexpr int kDK = 128;

// MAX: the dynamic shared memory the CTA has (the ring takes as many stages as fit).
template <int DV, int DVT, int MAX = 232448>
struct ChainLayout {
    static constexpr int NB = DVT / 64;                       // 64-column blocks of Z in the tile
    static constexpr int COLS = DVT / (kStateWarps / 4);      // columns per state thread
    // one stage: NG | Y | Z tile (NB blocks of [64 tokens][64 values]); the
    // decays of the stage's chunk sit in a small array of their own
    static constexpr int S_NG = 0, S_Y = 32768, S_Z = 49152;
    static constexpr int STAGE = S_Z + NB * 8192;
    // Sx buffer: [128][DVT], no swizzle.  One is enough: Sx of chunk c + 1 is
    // written after the UMMA that read Sx of chunk c has completed.
    static constexpr int SRB = DVT * 256;
    static constexpr int DEC_BYTES = kDK * 4;
    static constexpr int bytes(int ns) { return ns * (STAGE + DEC_BYTES) + SRB + 8 * (2 * ns + 5) + 16 + 1024; }
    static constexpr int NS = bytes(4) <= MAX ? 4 : bytes(3) <= MAX ? 3 : 2;
    static constexpr int SR = NS * STAGE;
    static constexpr int DECR = SR + SRB;
    static constexpr int BAR = DECR + NS * DEC_BYTES;
    static constexpr int NBAR = 2 * NS + 5;  // full[NS], empty[NS], s_done, sx_full, yz_done[2], s_issued
    static constexpr int SLOT = BAR + 8 * NBAR;  // TMEM address; export count at SLOT + 8, records seen at + 12
    static constexpr int DATA = SLOT + 16;   // bytes used from the 1024-aligned base
    static constexpr int BYTES = DATA + 1024;
    static constexpr uint32_t TMEM_COLS = 2 * DVT;            // two D buffers
    static_assert(BYTES <= MAX, "shared memory");
    static_assert(COLS % 32 == 0, "state columns per thread: whole 32-column tensor-memory loads");
    static_assert(STAGE % 1024 == 0 && SR % 1024 == 0, "swizzle atoms");
};

// Records of a window, all written before the chain starts; state images in
// the window's slots.  A flow tells the producer when record c may be read
// (record_ready) and, where it publishes progress, waits for the state warps'
// export count (wait_count) and announces that the images of chunks [0, n) are
// in the workspace (exported(n)).  The slot of state image c is free once
// record c is ready: the flow's users release a slot before the record that
// follows it in the ring is written.
template <int DV>
struct WindowFlow {
    static constexpr bool kPublishes = false;
    const uint8_t *recs;
    uint8_t *sxs;
    __device__ const uint8_t *record(int c) const { return recs + (long)c * Record<DV>::BYTES; }
    __device__ uint8_t *sx_slot(int c) const { return sxs + (long)c * SxSlot<DV>::BYTES; }
    __device__ bool record_ready(int) const { return true; }
    __device__ bool wait_count(const uint32_t *, uint32_t) const { return true; }
    __device__ void exported(int) const {}
};

// The adjoint walk: records and dS' image slots of chunks n-1, ..., 0, and the
// output gradients dO of chunk c by TMA (`tm_do`: [B][T][H][DV] bf16, boxes of
// 64 values x 64 tokens with the 128-byte swizzle).
template <int DV>
struct ReverseFlow {
    static constexpr bool kPublishes = false;
    const uint8_t *recs;
    uint8_t *sxs;
    const CUtensorMap *tm_do;
    int n, h, bi;
    __device__ const uint8_t *record(int cw) const { return recs + (long)(n - 1 - cw) * Record<DV>::BYTES; }
    __device__ uint8_t *sx_slot(int cw) const { return sxs + (long)(n - 1 - cw) * SxSlot<DV>::BYTES; }
    __device__ bool record_ready(int) const { return true; }
    __device__ bool wait_count(const uint32_t *, uint32_t) const { return true; }
    __device__ void exported(int) const {}
    __device__ void load_do(uint8_t *dst, uint64_t *bar, int cw, int blk) const
    {
        tma_load_4d(dst, tm_do, bar, blk * 64, h, (n - 1 - cw) * kChunk, bi);
    }
};

// One thread: the mbarriers of a chain CTA.
template <int DV, int DVT>
__device__ __forceinline__ void chain_init(uint8_t *sm)
{
    using L = ChainLayout<DV, DVT>;
    constexpr int NS = L::NS;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BAR);
    for (int s = 0; s < NS; ++s) {
        mbar_init(bars + s, 1);                    // full: the producer's bytes
        mbar_init(bars + NS + s, 1 + kStateWarps); // empty: the UMMAs and every state warp are done with it
    }
    mbar_init(bars + 2 * NS, 1);                   // s_done
    mbar_init(bars + 2 * NS + 1, kStateWarps);     // sx_full
    for (int b = 0; b < 2; ++b) mbar_init(bars + 2 * NS + 2 + b, 1);  // yz_done
    mbar_init(bars + 2 * NS + 4, 1);               // s_issued
    *reinterpret_cast<uint32_t *>(sm + L::SLOT + 8) = 0;   // export count
    *reinterpret_cast<uint32_t *>(sm + L::SLOT + 12) = 0;  // records seen by the producer
    fence_mbar_init();
}

// The chain of one (batch `pair`, value tile `tile`) over chunks [0, ncw), by
// threads tid < kChainThreads of a CTA whose mbarriers chain_init has set up
// and whose `tmem` holds TMEM_COLS columns.  S_in / S_out (either may be null)
// are the [pairs][128][DV] fp32 states before the first and after the last chunk.
template <int DV, int DVT, class Flow, bool ADJ = false>
__device__ __forceinline__ void chain_run(uint8_t *sm, uint32_t tmem, int tid, const Flow &f, const float *S_in,
                                          float *S_out, long pair, int tile, int ncw, unsigned int *err)
{
    using L = ChainLayout<DV, DVT>;
    using R = Record<DV>;
    constexpr int NS = L::NS, COLS = L::COLS, NB = L::NB;
    const int warp = tid >> 5, lane = tid & 31;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BAR);
    uint64_t *full = bars, *empty = bars + NS, *s_done = bars + 2 * NS, *sx_full = bars + 2 * NS + 1;
    uint64_t *yz_done = bars + 2 * NS + 2, *s_issued = bars + 2 * NS + 4;
    uint32_t *exports = reinterpret_cast<uint32_t *>(sm + L::SLOT + 8);
    uint32_t *rec_seen = reinterpret_cast<uint32_t *>(sm + L::SLOT + 12);
    const uint32_t sbase = smem_u32(sm);

    if (warp == kPublishWarp) {
        // ------------------------------------------------------------ publisher
        if (Flow::kPublishes && lane == 0) {
            for (int n = 0; n < ncw;) {
                n = min(n + kPublishEvery, ncw);
                if (!f.wait_count(exports, (uint32_t)(kStateWarps * n))) break;
                f.exported(n);
            }
        }
    } else if (warp == kProducerWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0;
            for (int cw = 0; cw < ncw; ++cw) {
                const int s = cw % NS;
                // the record first: its flag takes a round trip to L2, which
                // overlaps the wait for the stage
                if (!f.record_ready(cw)) break;
                smem_st_release(rec_seen, (uint32_t)(cw + 1));
                if (cw >= NS && !mbar_wait(empty + s, ((cw / NS) - 1) & 1, err)) break;
                uint8_t *st = sm + s * L::STAGE;
                const uint8_t *rec = f.record(cw);
                mbar_arrive_expect_tx(full + s, (uint32_t)(L::STAGE + L::DEC_BYTES));
                bulk_load(st + L::S_NG, rec + R::NG, 32768, full + s);
                if constexpr (ADJ) {
                    bulk_load(st + L::S_Y, rec + R::QS, 16384, full + s);
                    for (int b = 0; b < NB; ++b) f.load_do(st + L::S_Z + b * 8192, full + s, cw, tile * NB + b);
                } else {
                    bulk_load(st + L::S_Y, rec + R::Y, 16384, full + s);
                    bulk_load(st + L::S_Z, rec + R::Z + tile * NB * 8192, NB * 8192, full + s);
                }
                bulk_load(sm + L::DECR + s * L::DEC_BYTES, rec + R::DEC, L::DEC_BYTES, full + s);
                issued = cw + 1;
            }
            // copies in flight land before the CTA may leave
            for (int c = issued > NS ? issued - NS : 0; c < issued; ++c) mbar_wait(full + c % NS, (c / NS) & 1, err);
        }
    } else if (warp == kYzWarp) {
        // ------------------------------------------------------------ Y Z issuer
        if (lane == 0) {
            // Y: K-major, no-swizzle K chunks of 128 rows (16 tokens a step = 4 KB);
            // QS^T (ADJ): MN-major, 8-token K groups of 128 bytes, 8-key M chunks
            // of 1 KB (16 tokens a step = 256 bytes)
            const uint32_t idd = idesc_bf16(128, DVT, ADJ ? 1 : 0, 1);
            const uint64_t y0 = ADJ ? smem_desc(sbase + L::S_Y, 128, 1024, kSwNone)
                                    : smem_desc(sbase + L::S_Y, 2048, 128, kSwNone);
            constexpr int kYStep = ADJ ? 256 : 4096;
            const uint64_t z0 = smem_desc(sbase + L::S_Z, 8192, 1024, kSw128);
            bool ok = true;
            for (int cw = 0; cw < ncw; ++cw) {
                const int s = cw % NS, b = cw & 1;
                ok = ok && mbar_wait(full + s, (cw / NS) & 1, err);
                // right behind NG Sx of chunk cw - 1, whose issue also means that
                // the epilogue of chunk cw - 2 has read D[b]
                if (cw >= 1) ok = ok && mbar_wait(s_issued, (cw - 1) & 1, err);
                tc_fence_after();
                if (ok) {
                    const uint64_t so = (uint64_t)((s * L::STAGE) >> 4);
                    const uint32_t d = tmem + (uint32_t)(b * DVT);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(d, y0 + so + (uint64_t)((ks * kYStep) >> 4), z0 + so + (uint64_t)((ks * 2048) >> 4),
                                  idd, ks > 0);
                }
                umma_commit(yz_done + b);
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ NG Sx issuer
        if (lane == 0) {
            // NG: K-major (16 key channels a step = 4 KB); NG^T (ADJ): MN-major, the
            // same bytes with 8-row K groups of 128 bytes and 8-column M chunks of
            // 2 KB (16 a step = 256 bytes)
            const uint32_t idd = idesc_bf16(128, DVT, ADJ ? 1 : 0, 1);
            // descriptor start addresses are in 16-byte units: byte offsets >> 4 add directly
            const uint64_t ng0 = ADJ ? smem_desc(sbase + L::S_NG, 128, 2048, kSwNone)
                                     : smem_desc(sbase + L::S_NG, 2048, 128, kSwNone);
            constexpr int kNgStep = ADJ ? 256 : 4096;
            const uint64_t sx0 = smem_desc(sbase + L::SR, 128, 2048, kSwNone);   // MN-major, 8-row K groups
            bool ok = true;
            for (int cw = 0; cw < ncw; ++cw) {
                const int s = cw % NS, b = cw & 1;
                // Sx(cw) is in its buffer and D[(cw + 1) & 1] has been read
                ok = ok && mbar_wait(sx_full, cw & 1, err);
                ok = ok && mbar_wait(yz_done + b, (cw >> 1) & 1, err);
                tc_fence_after();
                if (ok) {
                    const uint64_t so = (uint64_t)((s * L::STAGE) >> 4);
                    const uint32_t d = tmem + (uint32_t)(b * DVT);
#pragma unroll
                    for (int ks = 0; ks < kDK / 16; ++ks)
                        umma_bf16(d, ng0 + so + (uint64_t)((ks * kNgStep) >> 4), sx0 + (uint64_t)((ks * 256) >> 4), idd, 1);
                }
                umma_commit(s_done);
                if (cw + NS < ncw) umma_commit(empty + s);
                mbar_arrive(s_issued);
            }
        }
    } else if (warp < kStateWarps) {
        // ------------------------------------------------------------ state
        const int i = tid & 127, grp = tid >> 7;
        const int col0 = grp * COLS;  // first column (within the tile) of this thread
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + col0;
        const float *decr = reinterpret_cast<const float *>(sm + L::DECR);
        float S[COLS];
#pragma unroll
        for (int j = 0; j < COLS; ++j) S[j] = 0.f;
        if (S_in) {
            const float *src = S_in + (pair * kDK + i) * DV + tile * DVT + col0;
#pragma unroll
            for (int j = 0; j < COLS; j += 4) {
                const float4 v4 = *reinterpret_cast<const float4 *>(src + j);
                S[j] = v4.x; S[j + 1] = v4.y; S[j + 2] = v4.z; S[j + 3] = v4.w;
            }
        }
        // Sx(cw) -> the Sx buffer (the next UMMA's operand), signal the MMA warp,
        // then, once the producer has seen record cw ready (the slot is free),
        // the same 16-byte pieces to the slot (every warp store covers 512
        // contiguous bytes) and count the warp's export.
        auto publish_sx = [&](int cw, bool ok) {
            uint8_t *sr = sm + L::SR;
#pragma unroll
            for (int j = 0; j < COLS; j += 8) *reinterpret_cast<uint4 *>(sr + sx_off(i, col0 + j)) = pack8(S + j);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(sx_full);
                for (uint32_t n = 0; ok && smem_ld_acquire(rec_seen) < (uint32_t)(cw + 1); ++n)
                    if (n == (1u << 24)) {
                        atomicOr(err, kErrTimeout);
                        ok = false;
                    }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (ok) {
                uint8_t *dst = f.sx_slot(cw);
#pragma unroll
                for (int j = 0; j < COLS; j += 8)
                    *reinterpret_cast<uint4 *>(dst + sx_off(i, tile * DVT + col0 + j)) =
                        *reinterpret_cast<const uint4 *>(sr + sx_off(i, col0 + j));  // this thread's own pieces
                if (Flow::kPublishes) {
                    __syncwarp();
                    if (lane == 0) smem_add_release(exports, 1);
                }
            }
            return ok;
        };
        bool ok = true;
        if (ncw > 0) ok = publish_sx(0, ok);
        for (int cw = 0; cw < ncw; ++cw) {
            const int s = cw % NS;
            ok = ok && mbar_wait(s_done, cw & 1, err);
            // the stage's decays (its bytes have landed: the UMMAs that just
            // completed read it), then release the stage to the producer
            ok = ok && mbar_wait(full + s, (cw / NS) & 1, err);
            tc_fence_after();
            const float gc = decr[s * kDK + i];
            __syncwarp();
            if (lane == 0 && cw + NS < ncw) mbar_arrive(empty + s);
            // the update in 32-column pieces (one tensor-memory load each)
            const uint32_t da = lane_addr + (uint32_t)((cw & 1) * DVT);
#pragma unroll
            for (int h = 0; h < COLS; h += 32) {
                float d[32];
                tmem_ld32(da + h, d);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 32; ++u) S[h + u] = gc * S[h + u] + d[u];
            }
            if (cw + 1 < ncw) ok = publish_sx(cw + 1, ok);
        }
        if (S_out) {
            float *dst = S_out + (pair * kDK + i) * DV + tile * DVT + col0;
#pragma unroll
            for (int j = 0; j < COLS; j += 4)
                *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }
}

}  // namespace chain
}  // namespace gdn2
