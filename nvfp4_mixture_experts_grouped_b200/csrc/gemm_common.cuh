// gemm_common.cuh -- helpers shared by the tcgen05 expert GEMMs: epilogue
// arithmetic (SiLU, NVFP4 requantisation of the SwiGLU output, an in-warp
// transpose of 16-byte chunks) and the weights' block-scale layout.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "formats.cuh"

namespace nvfp4moe {

// SiLU with the hardware exp2 and a fast divide (the layer is checked against the
// float64 oracle with a tolerance; these are not bit-exact steps).
__device__ __forceinline__ float silu_fast(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// NVFP4 requantisation of 16 SwiGLU outputs held by one thread: the block scale
// is decided exactly as the standalone quantiser does ((amax / 6) / gs with IEEE
// divisions, E4M3 round-to-nearest-even), the codes use x * (1 / (value(sf) * gs)).
__device__ __forceinline__ uint32_t requant_block16(const float* x, float gs, uint32_t& w0, uint32_t& w1) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
    const uint32_t sf = f32x2_to_e4m3x2(__fdiv_rn(__fdiv_rn(amax, 6.0f), gs), 0.0f) & 0xFFu;
    const float sfv = e4m3_to_float(sf);
    const float r = sfv != 0.0f ? __frcp_rn(sfv * gs) : 0.0f;
    float q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = x[i] * r;
    w0 = f32x8_to_e2m1x8(q);
    w1 = f32x8_to_e2m1x8(q + 8);
    return sf;
}

// Transposes the 8 x 8 matrix of 16-byte chunks held by each group of 8 lanes
// (pk: a lane's 8 chunks of 4 words), a butterfly over lane bits 1, 2, 4:
// afterwards lane 8G + c holds chunk c of the group's rows 8G + 0..7, so one
// store instruction writes whole 128-byte row segments.
template <typename T>
__device__ __forceinline__ void transpose_chunks8(T* pk, int lane) {
    const int c8 = lane & 7;
#pragma unroll
    for (int b = 0; b < 3; ++b) {
        const int m = 1 << b;
        const bool hi = (c8 & m) != 0;
#pragma unroll
        for (int k0 = 0; k0 < 8; ++k0) {
            if (k0 & m) continue;
            const int k1 = k0 | m;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const T send = hi ? pk[4 * k0 + w] : pk[4 * k1 + w];
                const T recv = __shfl_xor_sync(0xffffffffu, send, m);
                if (hi) pk[4 * k0 + w] = recv;
                else pk[4 * k1 + w] = recv;
            }
        }
    }
}

// Byte offset of weight scale column kb of packed row r in the weights' scale
// layout: the atom layout (128 rows x 4 columns per 512-byte atom), with the
// atoms a K stage of a 256-row N tile needs stored together -- the stage's
// atoms of rows 0..127 of the tile, then those of rows 128..255 -- so one bulk
// copy fetches them.  n_kb: scale columns per row; stage_atoms: atoms per 128
// rows in a full stage (4 for W4A4, 1 for W4A8); a last, partial stage holds
// fewer of each.
__host__ __device__ inline int64_t wsf_offset(int64_t r, int64_t kb, int64_t n_kb, int stage_atoms) {
    const int64_t atoms_per_row = n_kb >> 2, katom = kb >> 2;
    const int64_t ks = katom / stage_atoms;
    const int64_t na = min((int64_t)stage_atoms, atoms_per_row - ks * stage_atoms);
    return ((r >> 8) * atoms_per_row * 2 + ks * stage_atoms * 2 + ((r >> 7) & 1) * na + (katom - ks * stage_atoms)) *
               512 +
           (r & 31) * 16 + ((r >> 5) & 3) * 4 + (kb & 3);
}

}  // namespace nvfp4moe
