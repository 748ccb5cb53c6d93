// route.cu -- grouped sigmoid top-k routing on sm_100a, one warp per token (the
// arithmetic lives in route_token.cuh).
#include "route_token.cuh"

namespace nvfp4moe {

// WPB: warps (tokens) per CTA -- RT_WARPS, or 1 for small token counts, where
// each token's dependent chain then runs alone on its SM sub-partition.
template <int NPL, int WPB>
__global__ void __launch_bounds__(WPB * 32)
    k_route(const float* __restrict__ logits, const float* __restrict__ bias, int T, int E, int n_group, int topk_group,
            int top_k, float rsf, int renorm, ExpSpecConsts kc, int32_t* __restrict__ ids, float* __restrict__ wts) {
    __shared__ float s_c[WPB][RT_MAX_E + 32];
    const int warp = warp_id();
    const int t = blockIdx.x * WPB + warp;
    if (t >= T) return;
    route_token_general<NPL, false>(logits + (int64_t)t * E, bias, t, E, n_group, topk_group, top_k, rsf, renorm, kc,
                                    ids, wts, s_c[warp]);
}

// Up to 256 experts (NPL <= 8) the kernel fits 32 registers, 8 CTAs per SM:
// 8192 tokens then run as one wave of 1024 CTAs instead of 888 + 136.
template <int NPL, int WPB>
__global__ void __launch_bounds__(WPB * 32, NPL <= 8 ? 8 : 1)
    k_route_rows(const float* __restrict__ logits, const float* __restrict__ bias, int T, int E, int n_group,
                 int topk_group, int top_k, float rsf, int renorm, ExpSpecConsts kc, int32_t* __restrict__ ids,
                 float* __restrict__ wts) {
    const int t = blockIdx.x * WPB + warp_id();
    if (t >= T) return;
    route_token_rows<NPL, false>(logits + (int64_t)t * E, bias, t, E, n_group, topk_group, top_k, rsf, renorm, kc, ids,
                                 wts);
}

template <int NPL, int WPB>
__global__ void __launch_bounds__(WPB * 32)
    k_route_fast(const float* __restrict__ logits, const float* __restrict__ bias, int T, int E, int n_group,
                 int topk_group, int top_k, float rsf, int renorm, ExpSpecConsts kc, int32_t* __restrict__ ids,
                 float* __restrict__ wts) {
    __shared__ float s_score[WPB][32];
    const int warp = warp_id();
    const int t = blockIdx.x * WPB + warp;
    if (t >= T) return;
    route_token_fast<NPL, false>(logits + (int64_t)t * E, bias, t, E, n_group, topk_group, top_k, rsf, renorm, kc, ids,
                                 wts, s_score[warp]);
}

nvfp4moe_status launch_route(const float* logits, const float* bias, int T, int E, int n_group, int topk_group,
                             int top_k, float rsf, int renorm, int32_t* ids, float* wts, cudaStream_t stream) {
    if (T == 0) return NVFP4MOE_OK;
    const ExpSpecConsts kc = exp_spec_consts();
    // up to two tokens per SM: one warp per CTA, each token's chain on its own
    // sub-partition; otherwise RT_WARPS tokens per CTA
    const bool lone = T <= 2 * num_sms();
    const dim3 grid((unsigned)(lone ? T : ceil_div(T, RT_WARPS)));
    const int npl = (int)ceil_div(E, 32);
    const RouteShape shape = route_shape(E, n_group);
#define RT_LAUNCH_W(N, W)                                                                                         \
    do {                                                                                                          \
        if (shape == ROUTE_ROWS)                                                                                  \
            k_route_rows<N, W><<<grid, W * 32, 0, stream>>>(logits, bias, T, E, n_group, topk_group, top_k, rsf, \
                                                            renorm, kc, ids, wts);                                \
        else if (shape == ROUTE_SEGMENTS)                                                                         \
            k_route_fast<N, W><<<grid, W * 32, 0, stream>>>(logits, bias, T, E, n_group, topk_group, top_k, rsf, \
                                                            renorm, kc, ids, wts);                                \
        else                                                                                                      \
            k_route<N, W><<<grid, W * 32, 0, stream>>>(logits, bias, T, E, n_group, topk_group, top_k, rsf,      \
                                                       renorm, kc, ids, wts);                                     \
    } while (0)
#define RT_LAUNCH(N)                  \
    do {                              \
        if (lone)                     \
            RT_LAUNCH_W(N, 1);        \
        else                          \
            RT_LAUNCH_W(N, RT_WARPS); \
    } while (0)
    if (npl <= 1)
        RT_LAUNCH(1);
    else if (npl <= 2)
        RT_LAUNCH(2);
    else if (npl <= 4)
        RT_LAUNCH(4);
    else if (npl <= 8)
        RT_LAUNCH(8);
    else if (npl <= 16)
        RT_LAUNCH(16);
    else
        RT_LAUNCH(32);
#undef RT_LAUNCH
#undef RT_LAUNCH_W
    NVFP4MOE_CHECK_LAUNCH("route kernel");
    return NVFP4MOE_OK;
}

}  // namespace nvfp4moe
