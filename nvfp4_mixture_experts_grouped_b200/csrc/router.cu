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
// memory round trip instead of one per 128 columns.  When the token count fills
// at least one wave of 128-token x 64-expert tiles (prefill sizes), the
// projection is instead a register-tiled FP32 GEMM (k_router_logits_tiled), in
// which each hidden row is read once per 64 experts and each router row once per
// 128 tokens.  Then the routing, one warp per token (route.cu).  CUDA-core FP32
// throughout.  Built with -fmad=false; the dot products use explicit FMAs.
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

// Prefill-size projection, a register-tiled FP32 GEMM.  CTA (bx, by) computes
// the logits of experts 64bx .. 64bx+63 for tokens 128by .. 128by+127 with two
// groups of 128 threads: group g takes the chunks of 16 columns of H with
// index = g mod 2, so each SM runs twice the warps for the same tile.  In a
// group, thread (ty, tx) = (l / 8, l % 8) holds 8 tokens {4ty .. 4ty+3,
// 64+4ty .. 64+4ty+3} x 8 experts {4tx .. 4tx+3, 32+4tx .. 32+4tx+3} as 64
// accumulators, so its four shared-memory reads per h (one float4 each) are
// conflict-free across the warp.  Every thread copies one hidden row's 16 BF16
// and half of one router row's 16 FP32 of its group's chunk (four 16-byte
// cp.async, zero fill past T or E) into its own slot of a three-deep staging
// ring, two chunks ahead of the arithmetic; after a chunk's FMAs it waits for
// its own copies of the next one and stores them transposed (h-major, hidden
// values widened to FP32) into the other of its group's two buffers; one
// barrier per pair of chunks.  Each logit is the even-chunk FMA chain plus the
// odd-chunk chain (columns in order within each), added once: deterministic,
// and within gamma_(H/2+1) * sum_h |x_h w_h| of the exact dot product.  Rows
// past T and experts past E are not stored.  E % 4 == 0, H % 32 == 0.
constexpr int RTT_BM = 128;    // tokens per CTA
constexpr int RTT_BN = 64;     // experts per CTA
constexpr int RTT_BK = 16;     // columns of H per chunk
constexpr int RTT_STAGES = 3;  // staging ring depth (copies run two chunks ahead)
constexpr int RTT_GROUP = (RTT_BM / 8) * (RTT_BN / 8);  // threads per K group
constexpr int RTT_KG = 2;                                // K groups
constexpr int RTT_THREADS = RTT_KG * RTT_GROUP;
struct RttSmem {
    float x[RTT_KG][2][RTT_BK][RTT_BM];
    float w[RTT_KG][2][RTT_BK][RTT_BN];
    uint4 stage[RTT_STAGES][RTT_THREADS][4];  // per thread: 32 B hidden, 32 B router
};
static_assert(sizeof(float) * RTT_BM * RTT_BN <= sizeof(RttSmem::x), "the final sum reuses the hidden buffers");

__device__ __forceinline__ void cp_async16_zfill(void* smem, const void* gmem, bool valid) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    const uint32_t n = valid ? 16u : 0u;  // 0: nothing is read, the 16 bytes are zero-filled
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

__global__ void __launch_bounds__(RTT_THREADS, 2)
    k_router_logits_tiled(const uint16_t* __restrict__ x, const float* __restrict__ w, int T, int H, int E,
                          float* __restrict__ logits) {
    extern __shared__ __align__(16) unsigned char rtt_raw[];
    RttSmem& sm = *reinterpret_cast<RttSmem*>(rtt_raw);
    const int tid = threadIdx.x;
    const int g = tid / RTT_GROUP, l = tid % RTT_GROUP;
    const int e0 = blockIdx.x * RTT_BN;
    const int64_t t0 = (int64_t)blockIdx.y * RTT_BM;
    // copy roles within the group: hidden row t0 + l, all 16 columns of a chunk;
    // router row e0 + l % 64, columns 8 (l / 64) .. + 7 of a chunk
    const bool x_ok = t0 + l < T;
    const uint16_t* xrow = x + (x_ok ? t0 + l : 0) * (int64_t)H;
    const int we = l % RTT_BN, wh = (l / RTT_BN) * 8;
    const bool w_ok = e0 + we < E;
    const float* wrow = w + (int64_t)(w_ok ? e0 + we : 0) * H + wh;
    const int nq = H / (RTT_KG * RTT_BK);  // chunks per group
    // the group's chunk q (column chunk KG q + g) into ring slot q % 3, one
    // commit group per chunk (an empty group past the last keeps the count uniform)
    auto issue = [&](int q) {
        if (q < nq) {
            uint4* st = sm.stage[q % RTT_STAGES][tid];
            const int h0 = (RTT_KG * q + g) * RTT_BK;
            cp_async16_zfill(st + 0, xrow + h0, x_ok);
            cp_async16_zfill(st + 1, xrow + h0 + 8, x_ok);
            cp_async16_zfill(st + 2, wrow + h0, w_ok);
            cp_async16_zfill(st + 3, wrow + h0 + 4, w_ok);
        }
        cp_async_commit();
    };
    // this thread's staged chunk q, transposed into its group's buffer buf
    auto transpose = [&](int q, int buf) {
        const uint4* st = sm.stage[q % RTT_STAGES][tid];
        const uint4 x0 = st[0], x1 = st[1], w0 = st[2], w1 = st[3];
        const uint32_t u[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            sm.x[g][buf][2 * i][l] = bf16lo(u[i]);      // column 2i of the chunk
            sm.x[g][buf][2 * i + 1][l] = bf16hi(u[i]);  // column 2i + 1
        }
        const uint32_t f[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) sm.w[g][buf][wh + i][we] = __uint_as_float(f[i]);
    };
    const int ty = l / 8, tx = l % 8;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
    issue(0);
    issue(1);
    cp_async_wait_1();  // chunk 0 has landed (chunk 1 may be in flight)
    transpose(0, 0);
    __syncthreads();
    for (int q = 0; q < nq; ++q) {
        const int buf = q & 1;
        // ring slot (q + 2) % 3 was last read by this thread's transpose of
        // chunk q - 1, before the previous barrier
        issue(q + 2);
#pragma unroll
        for (int kk = 0; kk < RTT_BK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4*>(&sm.x[g][buf][kk][4 * ty]);
            const float4 a1 = *reinterpret_cast<const float4*>(&sm.x[g][buf][kk][64 + 4 * ty]);
            const float4 b0 = *reinterpret_cast<const float4*>(&sm.w[g][buf][kk][4 * tx]);
            const float4 b1 = *reinterpret_cast<const float4*>(&sm.w[g][buf][kk][32 + 4 * tx]);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
        }
        // the other buffer was last read in the previous chunk, before the barrier
        if (q + 1 < nq) {
            cp_async_wait_1();  // chunk q + 1 has landed (chunk q + 2 may be in flight)
            transpose(q + 1, buf ^ 1);
        }
        __syncthreads();
    }
    // the odd-chunk sums through shared memory (the hidden buffers, free after
    // the last barrier), added to the even-chunk sums in that order
    float* red = &sm.x[0][0][0][0];
    if (g == 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) red[(i * 8 + j) * RTT_GROUP + l] = acc[i][j];
    }
    __syncthreads();
    if (g == 1) return;
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = __fadd_rn(acc[i][j], red[(i * 8 + j) * RTT_GROUP + l]);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t t = t0 + (i < 4 ? 4 * ty + i : 64 + 4 * ty + (i - 4));
        if (t >= T) continue;
#pragma unroll
        for (int jh = 0; jh < 2; ++jh) {
            const int e = e0 + 32 * jh + 4 * tx;  // e % 4 == 0 and E % 4 == 0: all four or none
            if (e < E)
                *reinterpret_cast<float4*>(logits + t * E + e) =
                    make_float4(acc[i][4 * jh], acc[i][4 * jh + 1], acc[i][4 * jh + 2], acc[i][4 * jh + 3]);
        }
    }
}

}  // namespace

bool router_uses_tiled(int64_t T, int E) {
    return ceil_div(T, (int64_t)RTT_BM) * ceil_div((int64_t)E, (int64_t)RTT_BN) >= num_sms();
}

size_t router_ws_size(int T) { return (size_t)ceil_div((int64_t)T, RTR_TT) * sizeof(uint32_t); }

nvfp4moe_status launch_router_topk(const uint16_t* x, const float* w, const float* bias, int T, int H, int E,
                                   int n_group, int topk_group, int top_k, float rsf, int renorm, float* logits,
                                   int32_t* ids, float* wts, void* workspace, cudaStream_t stream) {
    (void)workspace;  // no scratch: the routing is a second launch on logits
    if (T == 0) return NVFP4MOE_OK;
    if (router_uses_tiled(T, E)) {
        // at least one wave of 128 x 64 tiles
        const dim3 tgrid((unsigned)ceil_div((int64_t)E, (int64_t)RTT_BN), (unsigned)ceil_div((int64_t)T, (int64_t)RTT_BM));
        NVFP4MOE_CUDA(cudaFuncSetAttribute(k_router_logits_tiled, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)sizeof(RttSmem)));
        k_router_logits_tiled<<<tgrid, RTT_THREADS, sizeof(RttSmem), stream>>>(x, w, T, H, E, logits);
        NVFP4MOE_CHECK_LAUNCH("router projection kernel");
        return launch_route(logits, bias, T, E, n_group, topk_group, top_k, rsf, renorm, ids, wts, stream);
    }
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
