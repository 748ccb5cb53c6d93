// compact.cu -- NVFP4 rows -> compact scales (4.125 bits per weight).
//
// "MiMo-V2.6-Flash-MOPD on one RTX PRO 6000", "Speed v6": a lossless compact
// expert encoding stores the same values in 4.125 instead of 4.5 bits per
// weight.  It is possible because ("AxionML / MiMo-V2.6-Flash-MOPD-NVFP4",
// introduction) after the transcode the two E4M3 scales of every 32 codes are
// the same power of two.  Encoding: per row one exponent r (the largest block
// exponent), per 32 codes a 4-bit distance n = r - e (0..14), or 15 for a
// block whose scale is zero over all-zero codes.  Decode-sized GEMMs are
// weight streams, so the 0.4375 bits per weight saved on scales are ~8% of
// their HBM bytes.
//
// The same check with no spread limit (max_spread large) tells whether a row's
// scales have an E8M0 form (one power of two per 32 codes), which the W4A8
// weights need.
//
// One warp per row: pass 1 classifies the row's blocks (lane j takes blocks 2j
// and 2j+1 of every 64 columns, one 32-bit load of their four scale bytes; the
// codes are read only for zero-scale blocks) and reduces max / min exponent and
// a failure flag; pass 2 writes the nibble bytes (one per 64 columns).
#include "common.cuh"
#include "formats.cuh"
#include "moe_internal.cuh"

namespace nvfp4moe {

namespace {

constexpr int CP_WARPS = 8;

// Kind of the 32-code block b of a row (see compact_block_kind), with the
// zero-scale case resolved: 1 only when its codes are all +-0, else 2.
__device__ __forceinline__ int block_kind(const uint8_t* codes_row, uint32_t s0, uint32_t s1, int64_t b, int& e) {
    int kind = compact_block_kind(s0, s1, e);
    if (kind == 1) {
        const uint4 q = *reinterpret_cast<const uint4*>(codes_row + b * 16);
        if (((q.x | q.y | q.z | q.w) & 0x77777777u) != 0u) kind = 2;
    }
    return kind;
}

__global__ void __launch_bounds__(CP_WARPS * 32)
    k_compact_rows(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf, int64_t rows, int64_t K,
                   int8_t* __restrict__ row_exp, uint8_t* __restrict__ nib, int32_t* __restrict__ row_status,
                   int32_t* __restrict__ n_bad, int max_spread) {
    const int64_t r = (int64_t)blockIdx.x * CP_WARPS + warp_id();
    if (r >= rows) return;
    const int lane = lane_id();
    const uint8_t* crow = codes + r * (K / 2);
    const uint32_t* srow = reinterpret_cast<const uint32_t*>(sf + r * (K / 16));  // 4 scale bytes per 64 columns
    const int64_t n64 = K / 64;
    int emax = -128, emin = 127, bad = 0;
    for (int64_t j = lane; j < n64; j += 32) {
        const uint32_t w = srow[j];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            int e = 0;
            const int kind = block_kind(crow, (w >> (16 * h)) & 0xFFu, (w >> (16 * h + 8)) & 0xFFu, 2 * j + h, e);
            if (kind == 0) {
                emax = max(emax, e);
                emin = min(emin, e);
            }
            bad |= kind == 2;
        }
    }
    emax = __reduce_max_sync(0xffffffffu, emax);
    emin = __reduce_min_sync(0xffffffffu, emin);
    const bool ok = !__any_sync(0xffffffffu, bad) && (emax == -128 || emax - emin <= max_spread);
    const int re = (ok && emax != -128) ? emax : 0;
    if (nib) {
        for (int64_t j = lane; j < n64; j += 32) {
            uint32_t byte = 0xFFu;
            if (ok) {
                const uint32_t w = srow[j];
                byte = 0;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    int e = 0;
                    const int kind =
                        block_kind(crow, (w >> (16 * h)) & 0xFFu, (w >> (16 * h + 8)) & 0xFFu, 2 * j + h, e);
                    byte |= (uint32_t)(kind == 0 ? re - e : 15) << (4 * h);
                }
            }
            nib[r * n64 + j] = (uint8_t)byte;
        }
    }
    if (lane == 0) {
        if (row_exp) row_exp[r] = (int8_t)re;
        if (row_status) row_status[r] = ok ? 0 : 1;
        if (!ok && n_bad) atomicAdd(n_bad, 1);
    }
}

}  // namespace

nvfp4moe_status launch_compact_rows(const uint8_t* codes, const uint8_t* sf, int64_t rows, int64_t K,
                                    int8_t* row_exp, uint8_t* nib, int32_t* row_status, int32_t* n_bad,
                                    cudaStream_t stream, int max_spread) {
    if (rows == 0) return NVFP4MOE_OK;
    k_compact_rows<<<(unsigned)ceil_div(rows, CP_WARPS), CP_WARPS * 32, 0, stream>>>(codes, sf, rows, K, row_exp, nib,
                                                                                     row_status, n_bad, max_spread);
    NVFP4MOE_CHECK_LAUNCH("compact scales kernel");
    return NVFP4MOE_OK;
}

}  // namespace nvfp4moe
