// router.cu -- the router projection followed by grouped top-k routing.
//
// "MiMo-V2.6-Flash-MOPD on one RTX PRO 6000", "Speed v6" / "What makes it
// fast": one matmul of the layer's router and a fused top-k replace the
// separate kernels (~3 us per layer instead of 27.5 at decode).  Routers are
// kept in F32 ("baekpica MiMo-V2.6-Flash-RL mixed-quant GGUF", tensor precision
// table): logits[t][e] = sum_h x[t][h] * w[e][h], BF16 hidden rows x FP32 router
// rows, FP32 arithmetic.  The logits are then routed by moe_route's kernel, so
// ids and weights equal moe_route's on these logits.
//
// Two launches.  The projection: CTA (bx, by) computes the logits of EPB experts
// for tokens 16by .. 16by+15; warp w < EPB * KS takes expert w % EPB and K slice
// w / EPB of the hidden dimension (KS = 8, 4 or 2 slices as H allows, EPB = 2,
// 4, 4), each lane a 4-column piece per 128 columns; sums run in a fixed order
// (per-lane FMA chain, warp butterfly, then the slices in order), so the logits
// are deterministic.  At the decode shape the kernel is a latency chain, not a
// bandwidth one (the router is 4 MB): each lane's router slice is loaded into
// registers and the tile's 16 hidden rows are copied into shared memory by the
// whole CTA, all loads issued before any arithmetic, so the kernel waits for one
// memory round trip instead of one per 128 columns.  Then the routing, one warp
// per token (route.cu).  CUDA-core FP32: large token counts re-read the router
// per 16-token tile.  Built with -fmad=false; the dot products use explicit FMAs.
#include "moe_internal.cuh"
#include "route_token.cuh"

namespace nvfp4moe {

namespace {

constexpr int RTR_TT = 16;    // tokens per CTA
constexpr int RTR_WARPS = 16;  // dot products: expert (w % EPB) x K slice (w / EPB)
__host__ __device__ constexpr int rtr_epb(int ks) { return ks == 8 ? 2 : 4; }

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Logits of EPB experts for the tile's tokens.  XS: the tile's hidden rows are
// first copied into shared memory by the whole CTA (16-byte loads, issued
// together), so the FMA loop reads them there; the router slice of each lane is
// loaded into registers before that copy, so both memory round trips overlap.
// Without XS (rows too long for shared memory) the rows are read from global
// memory in the loop.  The summation order is the same either way.
template <int KS, bool XS>
__global__ void __launch_bounds__(RTR_WARPS * 32)
    k_router_logits(const uint16_t* __restrict__ x, const float* __restrict__ w, int T, int H, int E,
                    float* __restrict__ logits) {
    extern __shared__ __align__(16) uint16_t rtr_xs[];  // XS: [nt][H] bf16
    constexpr int EPB = rtr_epb(KS);  // experts per CTA
    constexpr int HMAX4 = 8;          // float4 pieces of the router slice a lane holds (hh <= 1024)
    __shared__ float s_part[KS][EPB][RTR_TT];
    const int warp = warp_id(), lane = lane_id();
    const int el = warp % EPB, ks = warp / EPB;
    const int e = blockIdx.x * EPB + el;
    const int t0 = blockIdx.y * RTR_TT;
    const int nt = min(RTR_TT, T - t0);
    const int hh = H / KS;
    const bool computes = warp < EPB * KS;  // the other warps only help with the copy
    const float* wr = w + (int64_t)e * H + ks * hh;
    const int n4 = hh / 128;  // this lane's float4 pieces of the slice
    float4 wv[XS ? HMAX4 : 1];
    if (XS && computes) {
#pragma unroll
        for (int i = 0; i < HMAX4; ++i)
            if (i < n4) wv[i] = __ldg(reinterpret_cast<const float4*>(wr + lane * 4 + 128 * i));
    }
    if (XS) {
        const uint4* src = reinterpret_cast<const uint4*>(x + (int64_t)t0 * H);
        uint4* dst = reinterpret_cast<uint4*>(rtr_xs);
        const int n16 = nt * H / 8;
#pragma unroll 8
        for (int i = threadIdx.x; i < n16; i += RTR_WARPS * 32) dst[i] = __ldg(src + i);
        __syncthreads();
    }
    float acc[RTR_TT];
#pragma unroll
    for (int j = 0; j < RTR_TT; ++j) acc[j] = 0.0f;
    if (computes) {
        if (XS) {
            const uint16_t* xs = rtr_xs + ks * hh;
#pragma unroll
            for (int i = 0; i < HMAX4; ++i) {
                if (i >= n4) break;
                const int h = lane * 4 + 128 * i;
#pragma unroll
                for (int j = 0; j < RTR_TT; ++j) {
                    if (j < nt) {
                        const uint2 xv = *reinterpret_cast<const uint2*>(xs + j * H + h);
                        float a = acc[j];
                        a = __fmaf_rn(bf16lo(xv.x), wv[i].x, a);
                        a = __fmaf_rn(bf16hi(xv.x), wv[i].y, a);
                        a = __fmaf_rn(bf16lo(xv.y), wv[i].z, a);
                        a = __fmaf_rn(bf16hi(xv.y), wv[i].w, a);
                        acc[j] = a;
                    }
                }
            }
        } else {
            const uint16_t* xr = x + (int64_t)t0 * H + ks * hh;
#pragma unroll 2
            for (int h = lane * 4; h < hh; h += 128) {
                const float4 wq = __ldg(reinterpret_cast<const float4*>(wr + h));
#pragma unroll
                for (int j = 0; j < RTR_TT; ++j) {
                    if (j < nt) {
                        const uint2 xv = __ldg(reinterpret_cast<const uint2*>(xr + (int64_t)j * H + h));
                        float a = acc[j];
                        a = __fmaf_rn(bf16lo(xv.x), wq.x, a);
                        a = __fmaf_rn(bf16hi(xv.x), wq.y, a);
                        a = __fmaf_rn(bf16lo(xv.y), wq.z, a);
                        a = __fmaf_rn(bf16hi(xv.y), wq.w, a);
                        acc[j] = a;
                    }
                }
            }
        }
    }
#pragma unroll
    for (int j = 0; j < RTR_TT; ++j) {
#pragma unroll
        for (int o = 16; o; o >>= 1) acc[j] = __fadd_rn(acc[j], __shfl_xor_sync(0xffffffffu, acc[j], o));
    }
    if (lane == 0 && computes)
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
}

}  // namespace

size_t router_ws_size(int T) { return (size_t)ceil_div((int64_t)T, RTR_TT) * sizeof(uint32_t); }

nvfp4moe_status launch_router_topk(const uint16_t* x, const float* w, const float* bias, int T, int H, int E,
                                   int n_group, int topk_group, int top_k, float rsf, int renorm, float* logits,
                                   int32_t* ids, float* wts, void* workspace, cudaStream_t stream) {
    (void)workspace;  // no scratch: the routing is a second launch on logits
    if (T == 0) return NVFP4MOE_OK;
    const int ks = H % 1024 == 0 ? 8 : H % 512 == 0 ? 4 : 2;  // K slices per expert
    const dim3 grid((unsigned)(E / rtr_epb(ks)), (unsigned)ceil_div((int64_t)T, RTR_TT));
    // the tile's hidden rows in shared memory when they fit and a lane's router
    // slice fits its registers (H / ks <= 1024 columns)
    const size_t xs_bytes = (size_t)RTR_TT * H * sizeof(uint16_t);
    const bool xs = xs_bytes <= 200 * 1024 && H / ks <= 1024;
#define RTR_LAUNCH_K(K)                                                                                           \
    do {                                                                                                          \
        if (xs) {                                                                                                 \
            NVFP4MOE_CUDA(cudaFuncSetAttribute(k_router_logits<K, true>,                                         \
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)xs_bytes));      \
            k_router_logits<K, true><<<grid, RTR_WARPS * 32, xs_bytes, stream>>>(x, w, T, H, E, logits);        \
        } else {                                                                                                  \
            k_router_logits<K, false><<<grid, RTR_WARPS * 32, 0, stream>>>(x, w, T, H, E, logits);              \
        }                                                                                                         \
    } while (0)
    if (ks == 8)
        RTR_LAUNCH_K(8);
    else if (ks == 4)
        RTR_LAUNCH_K(4);
    else
        RTR_LAUNCH_K(2);
#undef RTR_LAUNCH_K
    NVFP4MOE_CHECK_LAUNCH("router projection kernel");
    // the routing of the logits: moe_route's kernel, so ids and weights equal moe_route's
    return launch_route(logits, bias, T, E, n_group, topk_group, top_k, rsf, renorm, ids, wts, stream);
}

}  // namespace nvfp4moe
