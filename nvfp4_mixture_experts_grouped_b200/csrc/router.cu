// router.cu -- the router projection fused with grouped top-k routing.
//
// "MiMo-V2.6-Flash-MOPD on one RTX PRO 6000", "Speed v6" / "What makes it
// fast": one matmul of the layer's router and a fused top-k replace the
// separate kernels (~3 us per layer instead of 27.5 at decode).  Routers are
// kept in F32 ("baekpica MiMo-V2.6-Flash-RL mixed-quant GGUF", tensor precision
// table): logits[t][e] = sum_h x[t][h] * w[e][h], BF16 hidden rows x FP32 router
// rows, FP32 arithmetic.  The routing of the logits is route_token.cuh, the
// same code as moe_route, so ids and weights equal moe_route's on these logits.
//
// One launch.  CTA (bx, by) computes the logits of EPB experts for tokens
// 16by .. 16by+15: warp w < EPB * KS takes expert w % EPB and K slice w / EPB of
// the hidden dimension (KS = 8, 4 or 2 slices as H allows, EPB = 2, 4, 4), each
// lane a 4-column piece per 128 columns; sums run in a fixed order (per-lane FMA
// chain, warp butterfly, then the slices in order), so the logits are
// deterministic.  The CTA has 16 warps so that its routing tail runs one token
// per warp.  After writing them the CTA counts itself done on
// its token tile; the last CTA of a tile (threadfence + atomic counter) routes
// the tile's 16 tokens, reading the logits through L2.  CUDA-core FP32: the
// decode case this targets streams the router (E x H x 4 bytes) once and is
// latency-bound; large token counts re-read the router per 16-token tile.
// Built with -fmad=false; the dot products use explicit FMAs.
#include "moe_internal.cuh"
#include "route_token.cuh"

namespace nvfp4moe {

namespace {

constexpr int RTR_TT = 16;    // tokens per CTA
constexpr int RTR_WARPS = 16;  // dot products: expert (w % EPB) x K slice (w / EPB); routing: one token each
__host__ __device__ constexpr int rtr_epb(int ks) { return ks == 8 ? 2 : 4; }

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int NPL, int SHAPE, int KS>
__global__ void __launch_bounds__(RTR_WARPS * 32)
    k_router_topk(const uint16_t* __restrict__ x, const float* __restrict__ w, const float* __restrict__ bias, int T,
                  int H, int E, int n_group, int topk_group, int top_k, float rsf, int renorm, ExpSpecConsts kc,
                  float* __restrict__ logits, int32_t* __restrict__ ids, float* __restrict__ wts,
                  uint32_t* __restrict__ tile_done) {
    extern __shared__ float rtr_smem[];  // routing scratch: per warp 32 (segments) or RT_MAX_E + 32 floats (general)
    constexpr int EPB = rtr_epb(KS);  // experts per CTA
    __shared__ float s_part[KS][EPB][RTR_TT];
    __shared__ int s_last;
    const int warp = warp_id(), lane = lane_id();
    const int el = warp % EPB, ks = warp / EPB;
    const int e = blockIdx.x * EPB + el;
    const int t0 = blockIdx.y * RTR_TT;
    const int nt = min(RTR_TT, T - t0);
    const int hh = H / KS;
    const float* wr = w + (int64_t)e * H + ks * hh;
    const uint16_t* xr = x + (int64_t)t0 * H + ks * hh;

    float acc[RTR_TT];
#pragma unroll
    for (int j = 0; j < RTR_TT; ++j) acc[j] = 0.0f;
    const int hend = warp < EPB * KS ? hh : 0;  // warps past EPB * KS only route
#pragma unroll 2
    for (int h = lane * 4; h < hend; h += 128) {
        const float4 wv = __ldg(reinterpret_cast<const float4*>(wr + h));
#pragma unroll
        for (int j = 0; j < RTR_TT; ++j) {
            if (j < nt) {
                const uint2 xv = __ldg(reinterpret_cast<const uint2*>(xr + (int64_t)j * H + h));
                float a = acc[j];
                a = __fmaf_rn(bf16lo(xv.x), wv.x, a);
                a = __fmaf_rn(bf16hi(xv.x), wv.y, a);
                a = __fmaf_rn(bf16lo(xv.y), wv.z, a);
                a = __fmaf_rn(bf16hi(xv.y), wv.w, a);
                acc[j] = a;
            }
        }
    }
#pragma unroll
    for (int j = 0; j < RTR_TT; ++j) {
#pragma unroll
        for (int o = 16; o; o >>= 1) acc[j] = __fadd_rn(acc[j], __shfl_xor_sync(0xffffffffu, acc[j], o));
    }
    if (lane == 0 && warp < EPB * KS)
#pragma unroll
        for (int j = 0; j < RTR_TT; ++j) s_part[ks][el][j] = acc[j];
    __syncthreads();
    if (threadIdx.x < EPB * RTR_TT) {
        const int l = threadIdx.x / RTR_TT, j = threadIdx.x % RTR_TT;
        if (j < nt) {
            float v = s_part[0][l][j];
#pragma unroll
            for (int q = 1; q < KS; ++q) v = __fadd_rn(v, s_part[q][l][j]);
            logits[(int64_t)(t0 + j) * E + blockIdx.x * EPB + l] = v;
        }
    }
    // the last CTA to finish this token tile routes it
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&tile_done[blockIdx.y], 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    float* scratch = rtr_smem + warp * (SHAPE == ROUTE_GENERAL ? RT_MAX_E + 32 : 32);
    for (int j = warp; j < nt; j += RTR_WARPS) {
        const int64_t t = t0 + j;
        if (SHAPE == ROUTE_ROWS)
            route_token_rows<NPL, true>(logits + t * E, bias, t, E, n_group, topk_group, top_k, rsf, renorm, kc, ids,
                                        wts);
        else if (SHAPE == ROUTE_SEGMENTS)
            route_token_fast<NPL, true>(logits + t * E, bias, t, E, n_group, topk_group, top_k, rsf, renorm, kc, ids,
                                        wts, scratch);
        else
            route_token_general<NPL, true>(logits + t * E, bias, t, E, n_group, topk_group, top_k, rsf, renorm, kc,
                                           ids, wts, scratch);
    }
    if (threadIdx.x == 0) tile_done[blockIdx.y] = 0u;  // the counters are zero again for the next call
}

}  // namespace

size_t router_ws_size(int T) { return (size_t)ceil_div((int64_t)T, RTR_TT) * sizeof(uint32_t); }

nvfp4moe_status launch_router_topk(const uint16_t* x, const float* w, const float* bias, int T, int H, int E,
                                   int n_group, int topk_group, int top_k, float rsf, int renorm, float* logits,
                                   int32_t* ids, float* wts, void* workspace, cudaStream_t stream) {
    if (T == 0) return NVFP4MOE_OK;
    uint32_t* tile_done = static_cast<uint32_t*>(workspace);
    NVFP4MOE_CUDA(cudaMemsetAsync(tile_done, 0, router_ws_size(T), stream));
    const ExpSpecConsts kc = exp_spec_consts();
    const int ks = H % 1024 == 0 ? 8 : H % 512 == 0 ? 4 : 2;  // K slices per expert
    const dim3 grid((unsigned)(E / rtr_epb(ks)), (unsigned)ceil_div((int64_t)T, RTR_TT));
    const RouteShape shape = route_shape(E, n_group);
    const size_t smem = (size_t)RTR_WARPS * (shape == ROUTE_GENERAL ? RT_MAX_E + 32 : 32) * sizeof(float);
    const int npl = (int)ceil_div(E, 32);
#define RTR_LAUNCH_K(N, F, K)                                                                                     \
    do {                                                                                                          \
        if (smem > 48 * 1024)                                                                                     \
            NVFP4MOE_CUDA(cudaFuncSetAttribute(k_router_topk<N, F, K>,                                           \
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));          \
        k_router_topk<N, F, K><<<grid, RTR_WARPS * 32, smem, stream>>>(x, w, bias, T, H, E, n_group, topk_group, \
                                                                       top_k, rsf, renorm, kc, logits, ids, wts, \
                                                                       tile_done);                                \
    } while (0)
#define RTR_LAUNCH_S(N, S)                \
    do {                                  \
        if (ks == 8)                      \
            RTR_LAUNCH_K(N, S, 8);        \
        else if (ks == 4)                 \
            RTR_LAUNCH_K(N, S, 4);        \
        else                              \
            RTR_LAUNCH_K(N, S, 2);        \
    } while (0)
#define RTR_LAUNCH(N)                                 \
    do {                                              \
        if (shape == ROUTE_ROWS)                      \
            RTR_LAUNCH_S(N, ROUTE_ROWS);              \
        else if (shape == ROUTE_SEGMENTS)             \
            RTR_LAUNCH_S(N, ROUTE_SEGMENTS);          \
        else                                          \
            RTR_LAUNCH_S(N, ROUTE_GENERAL);           \
    } while (0)
    if (npl <= 1)
        RTR_LAUNCH(1);
    else if (npl <= 2)
        RTR_LAUNCH(2);
    else if (npl <= 4)
        RTR_LAUNCH(4);
    else if (npl <= 8)
        RTR_LAUNCH(8);
    else if (npl <= 16)
        RTR_LAUNCH(16);
    else
        RTR_LAUNCH(32);
#undef RTR_LAUNCH
#undef RTR_LAUNCH_S
#undef RTR_LAUNCH_K
    NVFP4MOE_CHECK_LAUNCH("router kernel");
    return NVFP4MOE_OK;
}

}  // namespace nvfp4moe
