// permute.cu -- token permutation (grouping (token, slot) pairs by expert),
// activation quantise-and-scatter, and the weighted un-permute (combine).
//
// Grouped experts: "AxionML / MiMo-V2.6-Flash-MOPD-NVFP4", "Usage" (fused
// grouped MoE backend); "MiMo-V2.6-Flash-MOPD on one RTX PRO 6000", "Speed v4"
// (exact grouped kernel).  Combine: "MiMo-V2.6-Flash -- REAP-50", "Pruning
// Method" 1 (the layer output is the g_{t,j}-weighted sum of the selected
// experts' outputs).
//
// Rows of expert e occupy [pad_off[e], pad_off[e] + count[e]) of the permuted
// buffers, ordered by token then slot (deterministic, no sort).  pad_off rounds
// every expert's segment up to `pad` rows so that GEMM M-tiles never straddle
// two experts (pad = 128 for the tcgen05 path, 1 for the W4A16 path).
#include "common.cuh"
#include "formats.cuh"
#include "moe_internal.cuh"

namespace nvfp4moe {

// ---------------------------------------------------------------------------
// 1. per-chunk expert histogram (chunks of PERM_CHUNK tokens)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(PERM_CHUNK)
    k_count_chunks(const int32_t* __restrict__ ids, int T, int k, int E, int32_t* __restrict__ chunk_counts) {
    extern __shared__ int s_hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
    __syncthreads();
    const int t = blockIdx.x * PERM_CHUNK + threadIdx.x;
    if (t < T)
        for (int j = 0; j < k; ++j) {
            const int e = ids[(int64_t)t * k + j];
            if ((unsigned)e < (unsigned)E) atomicAdd(&s_hist[e], 1);  // ids outside [0, E) are skipped
        }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_counts[(int64_t)blockIdx.x * E + e] = s_hist[e];
}

// ---------------------------------------------------------------------------
// 2. per-expert scan over chunks, expert offsets, tile list (tiles of
//    plan.tile_rows rows: 128 for the single-CTA GEMM form, 256 for the CTA-pair
//    form), active list
// ---------------------------------------------------------------------------
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_tmp, int& total) {
    // blockDim.x == 1024: a shuffle scan inside each warp, then over the 32 warp totals
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_tmp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = s_tmp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_tmp[lane] = w;
    }
    __syncthreads();
    const int before = warp > 0 ? s_tmp[warp - 1] : 0;
    total = s_tmp[31];
    __syncthreads();  // s_tmp is reused by the next scan
    return before + x - v;
}


__global__ void __launch_bounds__(1024)
    k_scan_experts(int n_chunks, int E, int pad, int32_t* __restrict__ chunk_counts, RoutingPlan plan) {
    __shared__ int s_tmp[1024];
    const int e = threadIdx.x;
    int cnt = 0;
    if (e < E) {
        // 16 chunks' loads in flight before their stores: one L2 round trip per 16 chunks
        for (int c0 = 0; c0 < n_chunks; c0 += 16) {
            int v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = c0 + i < n_chunks ? chunk_counts[(int64_t)(c0 + i) * E + e] : 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if (c0 + i < n_chunks) chunk_counts[(int64_t)(c0 + i) * E + e] = cnt;  // the rank base of chunk c0 + i
                cnt += v[i];
            }
        }
    }
    int total;
    const int off = block_exclusive_scan(cnt, s_tmp, total);
    const int padded = e < E ? (int)round_up_dev(cnt, pad) : 0;
    int ptotal;
    const int poff = block_exclusive_scan(padded, s_tmp, ptotal);
    const int tr = plan.tile_rows;
    const int tiles = e < E ? (cnt + tr - 1) / tr : 0;
    int ttotal;
    const int toff = block_exclusive_scan(tiles, s_tmp, ttotal);
    int atotal;
    const int aoff = block_exclusive_scan(e < E && cnt > 0 ? 1 : 0, s_tmp, atotal);
    if (e < E) {
        plan.counts[e] = cnt;
        plan.offsets[e] = off;
        plan.pad_offsets[e] = poff;
        for (int j = 0; j < tiles; ++j)
            plan.tiles[toff + j] = make_int4(e, poff + j * tr, min(tr, cnt - j * tr), j);
        if (cnt > 0) plan.active[aoff] = e;
    }
    if (e == 0) {
        plan.offsets[E] = total;
        plan.pad_offsets[E] = ptotal;
        plan.n_tiles[0] = ttotal;
        plan.n_active[0] = atotal;
    }
}

// ---------------------------------------------------------------------------
// 3. stable scatter: row of every (token, slot) pair
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(PERM_CHUNK)
    k_scatter(const int32_t* __restrict__ ids, int T, int k, int E, const int32_t* __restrict__ chunk_base,
              RoutingPlan plan) {
    extern __shared__ int s_wh[];  // [PERM_WARPS][E] counters, then [E] padded expert offsets
    int* s_poff = s_wh + PERM_WARPS * E;
    const int warp = warp_id(), lane = lane_id();
    for (int i = threadIdx.x; i < PERM_WARPS * E; i += blockDim.x) s_wh[i] = 0;
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_poff[e] = plan.pad_offsets[e];
    __syncthreads();
    const int t0 = blockIdx.x * PERM_CHUNK + warp * 32;
    {
        const int t = t0 + lane;
        if (t < T)
            for (int j = 0; j < k; ++j) {
                const int e = ids[(int64_t)t * k + j];
                if ((unsigned)e < (unsigned)E) atomicAdd(&s_wh[warp * E + e], 1);
            }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = chunk_base[(int64_t)blockIdx.x * E + e];
        for (int w = 0; w < PERM_WARPS; ++w) {
            const int v = s_wh[w * E + e];
            s_wh[w * E + e] = run;
            run += v;
        }
    }
    __syncthreads();
    // tokens of this warp in order; a token's k experts are distinct, so the
    // k lanes never touch the same counter in one step.  Lane j < k holds slot
    // j's expert of all 32 tokens, loaded before the serial part.
    int eid[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) eid[i] = lane < k && t0 + i < T ? ids[(int64_t)(t0 + i) * k + lane] : 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int t = t0 + i;
        if (lane < k && t < T && (unsigned)eid[i] < (unsigned)E) {
            const int64_t p = (int64_t)t * k + lane;
            const int e = eid[i];
            const int r = s_wh[warp * E + e]++;
            const int row = s_poff[e] + r;
            plan.row_of_pair[p] = row;
            plan.pair_of_row[row] = (int32_t)p;
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// 1-3 in one CTA for up to PERM_FUSED_MAX_PAIRS pairs and E <= 256: per-warp
// histograms over contiguous pair chunks, the same scans as k_scan_experts,
// then stable ranks from match_any over 32-pair batches (a warp's chunk in pair
// order, warps in order), so every output equals the three-kernel path's.
// ---------------------------------------------------------------------------
constexpr int PERM_FUSED_MAX_E = 256;
constexpr int PERM_FUSED_MAX_PAIRS = 8192;  // one CTA beats three launches below ~10K pairs

__global__ void __launch_bounds__(1024)
    k_permute_fused(const int32_t* __restrict__ ids, int T, int k, int E, int pad, RoutingPlan plan) {
    __shared__ int s_wc[32 * PERM_FUSED_MAX_E];  // per-warp counts, then per-warp rank bases
    __shared__ int s_tmp[1024];
    __shared__ int s_poff[PERM_FUSED_MAX_E];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int P = T * k;
    const int chunk = (P + 31) / 32;
    const int p0 = min(P, warp * chunk), p1 = min(P, p0 + chunk);
    for (int i = tid; i < 32 * E; i += 1024) s_wc[i] = 0;
    __syncthreads();
    for (int p = p0 + lane; p < p1; p += 32) {
        const int e = ids[p];
        if ((unsigned)e < (unsigned)E) atomicAdd(&s_wc[warp * E + e], 1);
    }
    __syncthreads();
    int cnt = 0;
    if (tid < E) {
        for (int w = 0; w < 32; ++w) {
            const int v = s_wc[w * E + tid];
            s_wc[w * E + tid] = cnt;
            cnt += v;
        }
    }
    int total, ptotal, ttotal, atotal;
    const int off = block_exclusive_scan(cnt, s_tmp, total);
    const int padded = tid < E ? (int)round_up_dev(cnt, pad) : 0;
    const int poff = block_exclusive_scan(padded, s_tmp, ptotal);
    const int tr = plan.tile_rows;
    const int tiles = tid < E ? (cnt + tr - 1) / tr : 0;
    const int toff = block_exclusive_scan(tiles, s_tmp, ttotal);
    const int aoff = block_exclusive_scan(tid < E && cnt > 0 ? 1 : 0, s_tmp, atotal);
    if (tid < E) {
        plan.counts[tid] = cnt;
        plan.offsets[tid] = off;
        plan.pad_offsets[tid] = poff;
        s_poff[tid] = poff;
        for (int j = 0; j < tiles; ++j)
            plan.tiles[toff + j] = make_int4(tid, poff + j * tr, min(tr, cnt - j * tr), j);
        if (cnt > 0) plan.active[aoff] = tid;
    }
    if (tid == 0) {
        plan.offsets[E] = total;
        plan.pad_offsets[E] = ptotal;
        plan.n_tiles[0] = ttotal;
        plan.n_active[0] = atotal;
    }
    __syncthreads();
    for (int b = p0; b < p1; b += 32) {
        const int p = b + lane;
        const int id = p < p1 ? ids[p] : -1;
        const bool valid = (unsigned)id < (unsigned)E;
        const int e = valid ? id : -1 - lane;  // lanes past the chunk or with a bad id: keys of their own
        const unsigned same = __match_any_sync(0xffffffffu, e);
        if (valid) {
            const int row = s_poff[e] + s_wc[warp * E + e] + __popc(same & ((1u << lane) - 1u));
            plan.row_of_pair[p] = row;
            plan.pair_of_row[row] = p;
        }
        __syncwarp();
        if (valid && lane == __ffs(same) - 1) s_wc[warp * E + e] += __popc(same);
        __syncwarp();
    }
}

nvfp4moe_status launch_permute(const int32_t* ids, int T, int k, int E, int pad, RoutingPlan& plan,
                               cudaStream_t stream) {
    if (E <= PERM_FUSED_MAX_E && (int64_t)T * k <= PERM_FUSED_MAX_PAIRS) {
        k_permute_fused<<<1, 1024, 0, stream>>>(ids, T, k, E, pad, plan);
        NVFP4MOE_CHECK_LAUNCH("permute kernel");
        return NVFP4MOE_OK;
    }
    const int n_chunks = (int)ceil_div(T, PERM_CHUNK);
    k_count_chunks<<<n_chunks, PERM_CHUNK, E * sizeof(int), stream>>>(ids, T, k, E, plan.chunk_counts);
    NVFP4MOE_CHECK_LAUNCH("permute count kernel");
    k_scan_experts<<<1, 1024, 0, stream>>>(n_chunks, E, pad, plan.chunk_counts, plan);
    NVFP4MOE_CHECK_LAUNCH("permute scan kernel");
    k_scatter<<<n_chunks, PERM_CHUNK, (PERM_WARPS + 1) * E * sizeof(int), stream>>>(ids, T, k, E, plan.chunk_counts, plan);
    NVFP4MOE_CHECK_LAUNCH("permute scatter kernel");
    return NVFP4MOE_OK;
}

// ---------------------------------------------------------------------------
// Precomputed routing (moe_forward_routed).  The permutation's counters and row
// maps need every id in [0, E) and a token's ids distinct.  A token that breaks
// either rule is replaced by experts 0..k-1 with weight 0 (its output row is 0)
// and DEV_ERR_BAD_ROUTING is set in the device error word; the other tokens are
// copied unchanged.  One thread per token.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    k_check_routing(const int32_t* __restrict__ ids_in, const float* __restrict__ wts_in, int64_t T, int k, int E,
                    int32_t* __restrict__ ids, float* __restrict__ wts, int32_t* err) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    const int32_t* r = ids_in + t * k;
    bool ok = true;
    for (int j = 0; j < k; ++j) {
        const int32_t e = r[j];
        if (e < 0 || e >= E) ok = false;
        for (int i = 0; i < j; ++i)
            if (r[i] == e) ok = false;
    }
    for (int j = 0; j < k; ++j) {
        ids[t * k + j] = ok ? r[j] : j;
        wts[t * k + j] = ok ? wts_in[t * k + j] : 0.0f;
    }
    if (!ok) atomicOr(err, DEV_ERR_BAD_ROUTING);
}

nvfp4moe_status launch_check_routing(const int32_t* ids_in, const float* wts_in, int64_t T, int k, int E,
                                     int32_t* ids, float* wts, cudaStream_t stream) {
    if (T == 0) return NVFP4MOE_OK;
    int32_t* err = device_error_word();
    if (!err) {
        set_error("device error word unavailable");
        return NVFP4MOE_ERR_CUDA;
    }
    k_check_routing<<<(unsigned)ceil_div(T, 256), 256, 0, stream>>>(ids_in, wts_in, T, k, E, ids, wts, err);
    NVFP4MOE_CHECK_LAUNCH("routing check kernel");
    return NVFP4MOE_OK;
}

// ---------------------------------------------------------------------------
// The down projection's input rows of listed pairs, back in the checkpoint layout
// (moe_forward_intermediate).  One CTA per listed pair; a pair index outside
// [0, P) is skipped.  W4A4: NVFP4 codes [I/2] + E4M3 scales [I/16]; W4A8: E4M3
// [I] + E8M0 [I/32], both from the atom layout; W4A16: BF16 rows [I] (no scales).
// ---------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(128)
    k_read_intermediate(const int32_t* __restrict__ pairs, int64_t P, const int32_t* __restrict__ row_of_pair,
                        const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, int I,
                        uint8_t* __restrict__ codes_out, uint8_t* __restrict__ scales_out) {
    const int32_t p = pairs[blockIdx.x];
    if (p < 0 || p >= P) return;
    const int64_t row = row_of_pair[p];
    const int row_bytes = MODE == NVFP4MOE_W4A4 ? I / 2 : MODE == NVFP4MOE_W4A8 ? I : 2 * I;
    for (int i = threadIdx.x; i < row_bytes; i += blockDim.x)
        codes_out[(int64_t)blockIdx.x * row_bytes + i] = codes[row * row_bytes + i];
    if (MODE == NVFP4MOE_W4A4) {
        for (int kb = threadIdx.x; kb < I / 16; kb += blockDim.x)
            scales_out[(int64_t)blockIdx.x * (I / 16) + kb] = scales[sf_atom_offset(row, kb, I / 16)];
    } else if (MODE == NVFP4MOE_W4A8) {
        for (int kb = threadIdx.x; kb < I / 32; kb += blockDim.x)
            scales_out[(int64_t)blockIdx.x * (I / 32) + kb] = scales[sf_atom_offset(row, kb, I / 32)];
    }
}

nvfp4moe_status launch_read_intermediate(int mode, const int32_t* pairs, int n_pairs, int64_t P,
                                         const int32_t* row_of_pair, const uint8_t* codes, const uint8_t* scales,
                                         int I, uint8_t* codes_out, uint8_t* scales_out, cudaStream_t stream) {
    if (n_pairs == 0) return NVFP4MOE_OK;
    if (mode == NVFP4MOE_W4A4)
        k_read_intermediate<NVFP4MOE_W4A4><<<n_pairs, 128, 0, stream>>>(pairs, P, row_of_pair, codes, scales, I,
                                                                        codes_out, scales_out);
    else if (mode == NVFP4MOE_W4A8)
        k_read_intermediate<NVFP4MOE_W4A8><<<n_pairs, 128, 0, stream>>>(pairs, P, row_of_pair, codes, scales, I,
                                                                        codes_out, scales_out);
    else
        k_read_intermediate<NVFP4MOE_W4A16><<<n_pairs, 128, 0, stream>>>(pairs, P, row_of_pair, codes, scales, I,
                                                                         codes_out, scales_out);
    NVFP4MOE_CHECK_LAUNCH("intermediate read-back kernel");
    return NVFP4MOE_OK;
}

// ---------------------------------------------------------------------------
// 4. NVFP4 quantisation (one warp per row, a 16-element block per lane step)
// ---------------------------------------------------------------------------
// Linear layout (quantize_nvfp4): codes [M, K/2], scales [M, K/16].
// Scatter layout (moe_forward W4A4): the token's codes go to the k permuted
// rows of its pairs; scales go to the tcgen05 block-scale atom layout.
template <bool SCATTER, bool BF16_UNIT>
__global__ void __launch_bounds__(256)
    k_quantize(const uint16_t* __restrict__ x, int64_t M, int64_t K, float gs, uint8_t* __restrict__ codes,
               uint8_t* __restrict__ scales, const int32_t* __restrict__ row_of_pair, int k) {
    const int64_t m = (int64_t)blockIdx.x * 8 + warp_id();
    if (m >= M) return;
    const int lane = lane_id();
    const int64_t nb = K / 16;
    const uint16_t* xr = x + m * K;
    // destination rows of this token's k pairs, one per lane (k <= 32), broadcast below
    const int my_row = SCATTER && lane < k ? row_of_pair[m * k + lane] : 0;
    // every lane runs every iteration (the shuffles below need all 32); lanes past
    // the row's last block only skip their loads and stores.  The scatter form
    // needs nb % 4 == 0 (K % 64 == 0) so that a lane quad is all in or all out.
    // the next iteration's loads are issued before this one's arithmetic and stores
    uint4 n0 = make_uint4(0, 0, 0, 0), n1 = n0;
    if (lane < nb) {
        n0 = __ldg(reinterpret_cast<const uint4*>(xr + lane * 16));
        n1 = __ldg(reinterpret_cast<const uint4*>(xr + lane * 16 + 8));
    }
    for (int64_t b0 = 0; b0 < nb; b0 += 32) {
        const int64_t b = b0 + lane;
        const bool active = b < nb;
        const uint4 v0 = n0, v1 = n1;
        if (b + 32 < nb) {
            n0 = __ldg(reinterpret_cast<const uint4*>(xr + (b + 32) * 16));
            n1 = __ldg(reinterpret_cast<const uint4*>(xr + (b + 32) * 16 + 8));
        }
        float f[16];
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            f[2 * i] = bf16_bits_to_float(w[i] & 0xFFFFu);
            f[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
        }
        uint32_t c0, c1;
        const uint32_t sf = quantize_block16<BF16_UNIT>(f, gs, c0, c1);
        if (!SCATTER) {
            if (active) {
                *reinterpret_cast<uint2*>(codes + m * (K / 2) + b * 8) = make_uint2(c0, c1);
                scales[m * nb + b] = (uint8_t)sf;
            }
        } else {
            // lanes 4q..4q+3 hold the scales of blocks b..b+3 (b % 4 == 0 at lane 4q):
            // four consecutive bytes of one atom row, stored as one word by lane 4q
            uint32_t sfw = sf << (8 * (lane & 3));
            sfw |= __shfl_xor_sync(0xffffffffu, sfw, 1);
            sfw |= __shfl_xor_sync(0xffffffffu, sfw, 2);
            for (int j = 0; j < k; ++j) {
                const int64_t row = __shfl_sync(0xffffffffu, my_row, j);
                if (active) {
                    *reinterpret_cast<uint2*>(codes + row * (K / 2) + b * 8) = make_uint2(c0, c1);
                    if ((lane & 3) == 0) *reinterpret_cast<uint32_t*>(scales + sf_atom_offset(row, b, nb)) = sfw;
                }
            }
        }
    }
}

nvfp4moe_status launch_quantize_linear(const uint16_t* x, int64_t M, int64_t K, float gs, uint8_t* codes,
                                       uint8_t* scales, cudaStream_t stream) {
    if (M == 0) return NVFP4MOE_OK;
    // gs == 1 (the unit global scale): the division-free form, same codes
    if (gs == 1.0f)
        k_quantize<false, true><<<(unsigned)ceil_div(M, 8), 256, 0, stream>>>(x, M, K, gs, codes, scales, nullptr, 1);
    else
        k_quantize<false, false><<<(unsigned)ceil_div(M, 8), 256, 0, stream>>>(x, M, K, gs, codes, scales, nullptr, 1);
    NVFP4MOE_CHECK_LAUNCH("quantize kernel");
    return NVFP4MOE_OK;
}

// Scatter form for rows of up to NG * 1024 elements: one warp per token; the
// token's row is quantised once into registers -- lane l takes the two blocks
// 64g + 2l, 64g + 2l + 1 of each 64-block group g (32 elements, all loads issued
// before any arithmetic) -- and then written to each of its k permuted rows with
// one 16-byte store per group (a warp store instruction covers 512 contiguous
// bytes) and one scale word per lane pair (blocks 4q .. 4q + 3 of the atom row,
// assembled by one shuffle).  The same block quantiser as k_quantize: the same
// bytes, with the address arithmetic of a destination row done once per row
// instead of once per block.  Needs K % 64 == 0 (so a lane pair is all in or all
// out of the row).
template <bool BF16_UNIT, int NG>
__global__ void __launch_bounds__(256)
    k_quantize_scatter(const uint16_t* __restrict__ x, int64_t M, int64_t K, float gs, uint8_t* __restrict__ codes,
                       uint8_t* __restrict__ scales, const int32_t* __restrict__ row_of_pair, int k) {
    const int64_t m = (int64_t)blockIdx.x * 8 + warp_id();
    if (m >= M) return;
    const int lane = lane_id();
    const int64_t nb = K / 16;
    const uint16_t* xr = x + m * K;
    const int my_row = lane < k ? row_of_pair[m * k + lane] : 0;
    uint4 v[NG][4];
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        const int64_t b = 64 * g + 2 * lane;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            v[g][i] = b < nb ? __ldg(reinterpret_cast<const uint4*>(xr + b * 16) + i) : make_uint4(0, 0, 0, 0);
    }
    uint4 cw[NG];      // codes of the lane's two blocks of group g
    uint32_t sw[NG];   // even lanes: the scale word of blocks 64g + 2l .. + 3
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        uint32_t c[4], sf[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float f[16];
            const uint32_t w[8] = {v[g][2 * h].x, v[g][2 * h].y, v[g][2 * h].z, v[g][2 * h].w,
                                   v[g][2 * h + 1].x, v[g][2 * h + 1].y, v[g][2 * h + 1].z, v[g][2 * h + 1].w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                f[2 * i] = bf16_bits_to_float(w[i] & 0xFFFFu);
                f[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
            }
            sf[h] = quantize_block16<BF16_UNIT>(f, gs, c[2 * h], c[2 * h + 1]);
        }
        cw[g] = make_uint4(c[0], c[1], c[2], c[3]);
        const uint32_t pair = sf[0] | (sf[1] << 8);
        const uint32_t other = __shfl_xor_sync(0xffffffffu, pair, 1);
        sw[g] = pair | (other << 16);
    }
    for (int j = 0; j < k; ++j) {
        const int64_t row = __shfl_sync(0xffffffffu, my_row, j);
        uint8_t* crow = codes + row * (K / 2);
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const int64_t b = 64 * g + 2 * lane;
            if (b < nb) {
                *reinterpret_cast<uint4*>(crow + b * 8) = cw[g];
                if ((lane & 1) == 0) *reinterpret_cast<uint32_t*>(scales + sf_atom_offset(row, b, nb)) = sw[g];
            }
        }
    }
}

template <bool BF16_UNIT>
static void launch_scatter_ng(int ng, const uint16_t* x, int64_t T, int64_t H, float gs, uint8_t* codes,
                              uint8_t* scales, const int32_t* row_of_pair, int k, cudaStream_t stream) {
    const unsigned grid = (unsigned)ceil_div(T, 8);
    switch (ng) {
        case 1: k_quantize_scatter<BF16_UNIT, 1><<<grid, 256, 0, stream>>>(x, T, H, gs, codes, scales, row_of_pair, k); break;
        case 2: k_quantize_scatter<BF16_UNIT, 2><<<grid, 256, 0, stream>>>(x, T, H, gs, codes, scales, row_of_pair, k); break;
        case 3: k_quantize_scatter<BF16_UNIT, 3><<<grid, 256, 0, stream>>>(x, T, H, gs, codes, scales, row_of_pair, k); break;
        case 4: k_quantize_scatter<BF16_UNIT, 4><<<grid, 256, 0, stream>>>(x, T, H, gs, codes, scales, row_of_pair, k); break;
        case 5: k_quantize_scatter<BF16_UNIT, 5><<<grid, 256, 0, stream>>>(x, T, H, gs, codes, scales, row_of_pair, k); break;
        case 6: k_quantize_scatter<BF16_UNIT, 6><<<grid, 256, 0, stream>>>(x, T, H, gs, codes, scales, row_of_pair, k); break;
        case 7: k_quantize_scatter<BF16_UNIT, 7><<<grid, 256, 0, stream>>>(x, T, H, gs, codes, scales, row_of_pair, k); break;
        default: k_quantize_scatter<BF16_UNIT, 8><<<grid, 256, 0, stream>>>(x, T, H, gs, codes, scales, row_of_pair, k); break;
    }
}

nvfp4moe_status launch_quantize_scatter(const uint16_t* x, int64_t T, int64_t H, float gs, uint8_t* codes,
                                        uint8_t* scales, const int32_t* row_of_pair, int k, cudaStream_t stream) {
    if (T == 0) return NVFP4MOE_OK;
    const int64_t ng = (H / 16 + 63) / 64;  // 64-block groups per row
    if (ng <= 8) {
        // the row held in registers: one pass, 16-byte stores
        if (gs == 1.0f) launch_scatter_ng<true>((int)ng, x, T, H, gs, codes, scales, row_of_pair, k, stream);
        else launch_scatter_ng<false>((int)ng, x, T, H, gs, codes, scales, row_of_pair, k, stream);
    } else if (gs == 1.0f) {
        k_quantize<true, true><<<(unsigned)ceil_div(T, 8), 256, 0, stream>>>(x, T, H, gs, codes, scales, row_of_pair, k);
    } else {
        k_quantize<true, false><<<(unsigned)ceil_div(T, 8), 256, 0, stream>>>(x, T, H, gs, codes, scales, row_of_pair,
                                                                             k);
    }
    NVFP4MOE_CHECK_LAUNCH("quantize-scatter kernel");
    return NVFP4MOE_OK;
}

// MXFP8 of BF16 rows (W4A8 layer input): one warp per row, four lanes per
// 32-element block (8 elements each: one 16-byte load, an amax shuffle within
// the quad, 8 code bytes), so a warp instruction covers 8 blocks = 512 contiguous
// input bytes.  SCATTER writes each token's codes to its k permuted rows and the
// scales in the block-scale atom layout (K % 128 == 0: the four blocks of an
// atom word are in one half-warp); the linear form writes [M, K] codes and
// row-major [M, K/32] scales.
template <bool SCATTER>
__global__ void __launch_bounds__(256)
    k_quantize_mx8(const uint16_t* __restrict__ x, int64_t M, int64_t K, uint8_t* __restrict__ codes,
                   uint8_t* __restrict__ scales, const int32_t* __restrict__ row_of_pair, int k) {
    const int64_t m = (int64_t)blockIdx.x * 8 + warp_id();
    if (m >= M) return;
    const int lane = lane_id();
    const int64_t nb = K / 32;
    const uint16_t* xr = x + m * K;
    const int my_row = SCATTER && lane < k ? row_of_pair[m * k + lane] : 0;
    // loads run two iterations ahead of the arithmetic and stores
    uint4 nx[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int64_t b = 8 * i + (lane >> 2);
        nx[i] = b < nb ? __ldg(reinterpret_cast<const uint4*>(xr + b * 32 + (lane & 3) * 8)) : make_uint4(0, 0, 0, 0);
    }
    for (int64_t b0 = 0; b0 < nb; b0 += 8) {
        const int64_t b = b0 + (lane >> 2);  // this lane's block; it holds elements 8 (lane % 4) .. +7
        const bool active = b < nb;
        const uint4 v = nx[0];
        nx[0] = nx[1];
        nx[1] = b + 16 < nb ? __ldg(reinterpret_cast<const uint4*>(xr + (b + 16) * 32 + (lane & 3) * 8))
                            : make_uint4(0, 0, 0, 0);
        float f[8];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = bf16_bits_to_float(w[i] & 0xFFFFu);
            f[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const int X = mx8_exponent(amax);
        const float r = pow2_f32(-X);
        const uint2 c = make_uint2(f32x4_to_e4m3x4(f[0] * r, f[1] * r, f[2] * r, f[3] * r),
                                   f32x4_to_e4m3x4(f[4] * r, f[5] * r, f[6] * r, f[7] * r));
        const uint32_t sf = (uint32_t)(X + 127);
        if (!SCATTER) {
            if (active) {
                *reinterpret_cast<uint2*>(codes + m * K + b * 32 + (lane & 3) * 8) = c;
                if ((lane & 3) == 0) scales[m * nb + b] = (uint8_t)sf;
            }
        } else {
            // lanes 16h + 4j (j = 0..3) hold the scales of blocks b0 + 4h + j: one
            // atom word, assembled in lane 16h
            uint32_t sfw = sf << (8 * ((lane >> 2) & 3));
            sfw |= __shfl_xor_sync(0xffffffffu, sfw, 4);
            sfw |= __shfl_xor_sync(0xffffffffu, sfw, 8);
            for (int j = 0; j < k; ++j) {
                const int64_t row = __shfl_sync(0xffffffffu, my_row, j);
                if (active) {
                    *reinterpret_cast<uint2*>(codes + row * K + b * 32 + (lane & 3) * 8) = c;
                    if ((lane & 15) == 0) *reinterpret_cast<uint32_t*>(scales + sf_atom_offset(row, b, nb)) = sfw;
                }
            }
        }
    }
}

nvfp4moe_status launch_quantize_mx8_linear(const uint16_t* x, int64_t M, int64_t K, uint8_t* codes, uint8_t* scales,
                                           cudaStream_t stream) {
    if (M == 0) return NVFP4MOE_OK;
    k_quantize_mx8<false><<<(unsigned)ceil_div(M, 8), 256, 0, stream>>>(x, M, K, codes, scales, nullptr, 1);
    NVFP4MOE_CHECK_LAUNCH("mxfp8 quantize kernel");
    return NVFP4MOE_OK;
}

nvfp4moe_status launch_quantize_mx8_scatter(const uint16_t* x, int64_t T, int64_t H, uint8_t* codes, uint8_t* scales,
                                            const int32_t* row_of_pair, int k, cudaStream_t stream) {
    if (T == 0) return NVFP4MOE_OK;
    k_quantize_mx8<true><<<(unsigned)ceil_div(T, 8), 256, 0, stream>>>(x, T, H, codes, scales, row_of_pair, k);
    NVFP4MOE_CHECK_LAUNCH("mxfp8 quantize-scatter kernel");
    return NVFP4MOE_OK;
}

// ---------------------------------------------------------------------------
// 5. weighted un-permute: out[t] = sum_j Y[row_of_pair(t, j)] (routing weights
//    already applied by the down GEMM), FP32 in slot order, one rounding.
//    Y is FP16 with a power-of-two scale per 64 columns (W4A4) or FP32 (W4A16,
//    W4A8).
// ---------------------------------------------------------------------------
template <bool Y_F16, bool OUT_F32>
__global__ void __launch_bounds__(256)
    k_combine(const void* __restrict__ Yv, const float* __restrict__ y_scale, const int32_t* __restrict__ row_of_pair,
              int64_t T, int H, int k, void* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // one 8-element vector
    const int64_t per_row = H / 8;
    if (i >= T * per_row) return;
    const int64_t t = i / per_row;
    const int64_t h8 = (i - t * per_row) * 8;
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
    for (int j = 0; j < k; ++j) {
        const int64_t row = __ldg(row_of_pair + t * k + j);
        if (Y_F16) {
            const float s = __ldg(y_scale + row * (H / 64) + h8 / 64);
            const uint4 v = __ldcs(reinterpret_cast<const uint4*>(static_cast<const __half*>(Yv) + row * H + h8));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[q]));
                acc[2 * q] = __fadd_rn(acc[2 * q], __fmul_rn(f.x, s));
                acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], __fmul_rn(f.y, s));
            }
        } else {
            const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(Yv) + row * H + h8);
            const float4 a = __ldcs(src), b = __ldcs(src + 1);
            const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = __fadd_rn(acc[q], f[q]);
        }
    }
    if (OUT_F32) {
        float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + t * H + h8);
        __stcs(o, make_float4(acc[0], acc[1], acc[2], acc[3]));
        __stcs(o + 1, make_float4(acc[4], acc[5], acc[6], acc[7]));
    } else {
        uint32_t p[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
            p[q] = *reinterpret_cast<uint32_t*>(&b);
        }
        __stcs(reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + t * H + h8), make_uint4(p[0], p[1], p[2], p[3]));
    }
}

nvfp4moe_status launch_combine(const void* Y, const float* y_scale, const int32_t* row_of_pair, int64_t T, int H,
                               int k, void* out, bool out_f32, cudaStream_t stream) {
    if (T == 0) return NVFP4MOE_OK;
    const int64_t n = T * (H / 8);
    const unsigned grid = (unsigned)ceil_div(n, 256);
    if (y_scale) {
        if (out_f32)
            k_combine<true, true><<<grid, 256, 0, stream>>>(Y, y_scale, row_of_pair, T, H, k, out);
        else
            k_combine<true, false><<<grid, 256, 0, stream>>>(Y, y_scale, row_of_pair, T, H, k, out);
    } else {
        if (out_f32)
            k_combine<false, true><<<grid, 256, 0, stream>>>(Y, y_scale, row_of_pair, T, H, k, out);
        else
            k_combine<false, false><<<grid, 256, 0, stream>>>(Y, y_scale, row_of_pair, T, H, k, out);
    }
    NVFP4MOE_CHECK_LAUNCH("combine kernel");
    return NVFP4MOE_OK;
}

}  // namespace nvfp4moe
