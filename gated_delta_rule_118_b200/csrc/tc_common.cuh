// tc_common.cuh -- helpers shared by the tensor-core forward kernels: bf16
// packing, warp-level tf32 MMAs, and the layout of the workspace records that
// carry a chunk's state-independent quantities from the prep kernel to the
// chain and output kernels.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "sm100.cuh"

namespace gdn2 {

using bf16 = __nv_bfloat16;

constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// One prep record per (batch, head, chunk), read by the chain and output kernels.
// With Ebar = e^{Gamma} b k the erase keys decayed from the chunk start, the
// chunk maps the incoming state S to
//   S_next = Diag(e^{Gamma_C}) S + NG S + Y Z       NG = -Ktil^T T Ebar
//   O      = QS S + PT Z                            QS = (Qhat - P T Ehat) Diag(e^{Gamma_r})
// The A operands (NG, QS, Y, PT) are bf16 K-major without swizzle, stored as
// 16-byte K chunks of all rows in turn: element (row m, k) at byte
// (k / 8) * (16 * ROWS) + m * 16 + (k % 8) * 2, so that a warp writing one
// K chunk of 32 consecutive rows stores 512 contiguous bytes, and the UMMA
// reads the tile with a leading (K) byte offset of 16 * ROWS and a stride
// (8-row) byte offset of 128.
//   NG  [128 rows = key channel i][128 K = key channel j]
//   QS  [64 rows = token][128 K = key channel]
//   Y   [128 rows = key channel][64 K = token]:  Y = Ktil^T T
//   PT  [64 rows = token][64 K = token]:         P T
//   Z   [64 rows = token (K)][DV = value (N)], MN-major B operand with the
//       128-byte swizzle, DV/64 blocks of 8 KB: Z = w v
//   DEC [128] fp32: e^{Gamma_C} per key channel
template <int DV>
struct Record {
    static constexpr int NG = 0;
    static constexpr int QS = 32768;
    static constexpr int Y = 49152;
    static constexpr int PT = 65536;
    static constexpr int Z = 73728;
    static constexpr int DEC = Z + 64 * DV * 2;
    static constexpr int BYTES = DEC + 1024;
};

// Byte offset of K chunk c (8 elements), row m, in a no-swizzle K-major tile of ROWS rows.
__host__ __device__ constexpr uint32_t kchunk_off(int c, int m, int rows) { return (uint32_t)(c * 16 * rows + m * 16); }

// The chain kernel exports the bf16 image Sx of the state entering every chunk
// for the output kernel: [128 key channels (K)][DV values (N)], an MN-major B
// operand without swizzle: element (j, n) at byte (n / 8) * 2048 + j * 16 + (n % 8) * 2.
// A warp holding 8 value columns of 32 consecutive key rows stores 512
// contiguous bytes; the UMMA reads it with a leading (8-row K group) byte
// offset of 128 and a stride (8-column N chunk) byte offset of 2048.
template <int DV>
struct SxSlot {
    static constexpr int BYTES = 128 * DV * 2;
};
__host__ __device__ constexpr uint32_t sx_off(int j, int n) { return (uint32_t)((n >> 3) * 2048 + j * 16 + (n & 7) * 2); }

__device__ __forceinline__ uint4 pack8(const float *f)
{
    uint4 r;
    __nv_bfloat162 h;
    h = __floats2bfloat162_rn(f[0], f[1]); r.x = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2bfloat162_rn(f[2], f[3]); r.y = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2bfloat162_rn(f[4], f[5]); r.z = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2bfloat162_rn(f[6], f[7]); r.w = *reinterpret_cast<uint32_t *>(&h);
    return r;
}

__device__ __forceinline__ void unpack8(uint4 v, float *f)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 p = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
        f[2 * i] = p.x;
        f[2 * i + 1] = p.y;
    }
}


__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Warp-level D += A B on tf32 operands, m16n8k8 (A row-major 16x8, B column-major
// 8x8, fp32 accumulators).  Fragment of lane l (g = l / 4, c = l % 4):
//   a0 = A[g][c], a1 = A[g+8][c], a2 = A[g][c+4], a3 = A[g+8][c+4]
//   b0 = B[c][g], b1 = B[c+4][g]
//   d0 = D[g][2c], d1 = D[g][2c+1], d2 = D[g+8][2c], d3 = D[g+8][2c+1]
__device__ __forceinline__ uint32_t to_tf32(float x)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// fp32 64x64 matrix in shared memory with 16-byte chunks XOR-swizzled by row,
// so that row-per-thread float4 stores and column walks avoid bank conflicts.
__device__ __forceinline__ int af_off(int t, int s) { return t * 64 + ((((s >> 2) ^ (t & 15)) << 2) | (s & 3)); }

}  // namespace gdn2
