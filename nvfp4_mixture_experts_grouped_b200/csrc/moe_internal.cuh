// moe_internal.cuh -- declarations shared by the kernels and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace nvfp4moe {

constexpr int PERM_CHUNK = 256;  // tokens per permutation chunk (one CTA)
constexpr int PERM_WARPS = PERM_CHUNK / 32;
constexpr int MTILE = 128;       // rows of one tcgen05 M-tile (the row padding and tile size of the GEMM paths)

__device__ __forceinline__ int64_t round_up_dev(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// Device pointers (inside the workspace) describing one routing of T tokens.
struct RoutingPlan {
    int32_t* ids;           // [T*k] expert of each pair (pair = t*k + j)
    float* wts;             // [T*k] routing weight of each pair
    int32_t* chunk_counts;  // [n_chunks*E] per-chunk counts, then per-chunk rank bases
    int32_t* counts;        // [E]
    int32_t* offsets;       // [E+1] unpadded row offsets
    int32_t* pad_offsets;   // [E+1] row offsets with every segment padded to `pad`
    int32_t* row_of_pair;   // [T*k]
    int32_t* pair_of_row;   // [rows_max]
    int4* tiles;            // [max_tiles] {expert, first padded row, valid rows (<= tile_rows), tile index in expert}
    int32_t* n_tiles;       // [1]
    int32_t* active;        // [E] experts with at least one row
    int32_t* n_active;      // [1]
    int tile_rows = MTILE;  // rows per tile of the tile list: MTILE or 2 * MTILE (a CTA pair's tile)
};

// transcode.cu
size_t transcode_ws_size(int64_t num_tensors);
nvfp4moe_status launch_transcode(const uint8_t* codes_in, const uint8_t* e8m0_in, int64_t num_tensors, int64_t N,
                                 int64_t K, uint8_t* codes_out, uint8_t* e4m3_out, float* global_out,
                                 int32_t* status_out, void* workspace, cudaStream_t stream);
nvfp4moe_status read_transcode_report(const void* workspace, nvfp4moe_transcode_report* out, cudaStream_t stream);

// route.cu
nvfp4moe_status launch_route(const float* logits, const float* bias, int T, int E, int n_group, int topk_group,
                             int top_k, float rsf, int renorm, int32_t* ids, float* wts, cudaStream_t stream);

// router.cu
size_t router_ws_size(int T);
constexpr int64_t ROUTER_MAX_T = 65535LL * 128;  // the tiled projection's grid (128 tokens per CTA row)
// the projection is the tiled FP32 GEMM (one FMA chain over H per logit) when
// the token count fills at least one wave of its 128 x 64 tiles
bool router_uses_tiled(int64_t T, int E);
nvfp4moe_status launch_router_topk(const uint16_t* x, const float* w, const float* bias, int T, int H, int E,
                                   int n_group, int topk_group, int top_k, float rsf, int renorm, float* logits,
                                   int32_t* ids, float* wts, void* workspace, cudaStream_t stream);

// permute.cu
nvfp4moe_status launch_permute(const int32_t* ids, int T, int k, int E, int pad, RoutingPlan& plan,
                               cudaStream_t stream);
// precomputed routing: copies ids / weights, replacing tokens with an id outside
// [0, E) or a repeated id by experts 0..k-1 with weight 0 (DEV_ERR_BAD_ROUTING)
nvfp4moe_status launch_check_routing(const int32_t* ids_in, const float* wts_in, int64_t T, int k, int E,
                                     int32_t* ids, float* wts, cudaStream_t stream);
// the down projection's input rows of listed pairs in the checkpoint layout
nvfp4moe_status launch_read_intermediate(int mode, const int32_t* pairs, int n_pairs, int64_t P,
                                         const int32_t* row_of_pair, const uint8_t* codes, const uint8_t* scales,
                                         int I, uint8_t* codes_out, uint8_t* scales_out, cudaStream_t stream);
nvfp4moe_status launch_quantize_linear(const uint16_t* x, int64_t M, int64_t K, float gs, uint8_t* codes,
                                       uint8_t* scales, cudaStream_t stream);
// scales in the atom layout of the W4A4 GEMMs (sf_atom_offset)
nvfp4moe_status launch_quantize_scatter(const uint16_t* x, int64_t T, int64_t H, float gs, uint8_t* codes,
                                        uint8_t* scales, const int32_t* row_of_pair, int k, cudaStream_t stream);
// MXFP8 (E4M3 + E8M0 per 32): linear [M, K] codes / [M, K/32] scales, and the
// scatter into permuted rows with atom-layout scales (K % 128 == 0)
nvfp4moe_status launch_quantize_mx8_linear(const uint16_t* x, int64_t M, int64_t K, uint8_t* codes, uint8_t* scales,
                                           cudaStream_t stream);
nvfp4moe_status launch_quantize_mx8_scatter(const uint16_t* x, int64_t T, int64_t H, uint8_t* codes, uint8_t* scales,
                                            const int32_t* row_of_pair, int k, cudaStream_t stream);
// Y staged as FP16 rows with a power-of-two scale per 64 columns (y_scale != nullptr,
// W4A4) or as FP32 rows (y_scale == nullptr, W4A16 and W4A8).
nvfp4moe_status launch_combine(const void* Y, const float* y_scale, const int32_t* row_of_pair, int64_t T, int H,
                               int k, void* out, bool out_f32, cudaStream_t stream);

// compact.cu: compact scales of NVFP4 rows (row_exp [rows], nib [rows, K/64],
// row_status [rows] and the failure counter n_bad, each optional).  K % 64 == 0.
// max_spread: 14 for the compact form; larger only checks that every 32-code
// block's scale is one power of two (the E8M0 form).
constexpr int COMPACT_MAX_SPREAD = 14;
nvfp4moe_status launch_compact_rows(const uint8_t* codes, const uint8_t* sf, int64_t rows, int64_t K,
                                    int8_t* row_exp, uint8_t* nib, int32_t* row_status, int32_t* n_bad,
                                    cudaStream_t stream, int max_spread = COMPACT_MAX_SPREAD);

// w4a16.cu
// compact = the 4.125-bit scale form (mode NVFP4MOE_W4A16C)
size_t w4a16_packed_size(int E, int H, int I, bool compact);
nvfp4moe_status launch_w4a16_pack(const nvfp4moe_expert_weights& w, void* packed, bool compact, cudaStream_t stream);
size_t w4a16_scratch_size(int T, int H, int I, int k);  // FP16 copies of the activations + row scales
nvfp4moe_status launch_w4a16_layer(const uint16_t* x, const void* packed, bool compact, int T, int H, int I,
                                   int E, int k, const RoutingPlan& plan, uint16_t* A2, float* Y, void* scratch,
                                   cudaStream_t stream, cudaEvent_t mid_event);

// tmaps.cu: 2-D tensor maps of the TMA copies.  make_map: uint8 rows
// [rows, row_bytes], a box of 128 bytes x box_rows, 128-byte swizzle; make_map_u4:
// 4-bit codes [rows, k_elems] that the copy unpacks into the padded
// shared-memory form (each 16 codes: 8 bytes, then 8 bytes of gap), a box of 128
// codes x box_rows.  Both set the error string and return false on failure.
bool make_map(CUtensorMap* m, const void* base, int64_t row_bytes, int64_t rows, int box_rows);
bool make_map_u4(CUtensorMap* m, const void* base, int64_t k_elems, int64_t rows, int box_rows);

// w4a4.cu: rows per tile of the tile list the W4A4 / W4A8 GEMMs are cut for at
// this shape (MTILE: single-CTA tiles; 2 * MTILE: CTA-pair tiles)
int w4a4_tile_rows(int64_t T, int k, int E);
// w4a4.cu: the tcgen05 GEMMs; mx8 selects W4A8 (MXFP8 activations x FP4
// weights held in the padded form with E8M0 scales) instead of W4A4
size_t w4a4_packed_size(int E, int H, int I, bool mx8);
nvfp4moe_status launch_w4a4_pack(const nvfp4moe_expert_weights& w, void* packed, bool mx8, cudaStream_t stream);
nvfp4moe_status launch_w4a4_layer(const void* packed, bool mx8, int T, int H, int I, int E, int k,
                                  float act_global_in, float act_global_mid, int64_t rows_max, int max_tiles,
                                  const RoutingPlan& plan, const uint8_t* A1c, const uint8_t* A1s, uint8_t* A2c,
                                  uint8_t* A2s, __half* Y, float* y_scale, cudaStream_t stream, cudaEvent_t mid_event);

}  // namespace nvfp4moe
