// w4a16.cu -- the W4A16 (BF16 activations x NVFP4 weights) expert GEMMs for
// decode-sized batches on sm_100a.
//
// Mode: "AxionML / MiMo-V2.6-Flash-MOPD-NVFP4", "Usage" (BF16-activation,
// weight-only FP4 mode) and "Accuracy".  Expert MLP: "MiMo-V2.6-Flash --
// REAP-50", "Pruning Method" 1 (down(SiLU(gate h) * up h)).
//
// At decode an expert sees ~1-2 tokens, so the layer is a weight stream: every
// active expert's codes and scales are read from HBM exactly once.  Weights are
// the MMA "A" operand (16 weight rows per mma.sync.m16n8k16), tokens the "B"
// operand (8 per n-tile).  Weights are dequantised in registers to BF16:
//   * one 32-bit word holds the 8 codes a lane needs for one k16 step, with
//     their bits pre-placed by the pack step so that each BF16x2 fragment
//     register is one or two shift/AND operations away: a code (s e1 e0 m)
//     whose 3 magnitude bits land on BF16 bits 8..6 and whose sign lands on bit
//     15 is exactly the E2M1 value times 2^-126 (the 0.5 code becomes the BF16
//     subnormal 2^-127);
//   * the E4M3 block scale becomes the BF16 multiplier scale * 2^118 (through
//     the exact E4M3->F16 conversion and an exponent re-bias), so one BF16x2
//     multiply yields value * scale * 2^-8 exactly (at most 5 significant bits,
//     range [2^-18, 10.5]);
//   * the FP32 accumulator is multiplied by 2^8 * global in the epilogue.
// Gate and up rows of the same 16 intermediates are streamed by the same warp,
// so SwiGLU is applied on the accumulators and only BF16 SwiGLU rows are stored.
// The down GEMM stages its weighted per-pair rows in FP32 (a few MB at decode).
#include <algorithm>

#include "common.cuh"
#include "formats.cuh"
#include "moe_internal.cuh"
#include "tc_ptx.cuh"

namespace nvfp4moe {

namespace {

constexpr int W16_WARPS = 4;
constexpr int W16_MAX_NT = 4;  // n-tiles (of 8 tokens) per pass over the weights

struct W16Layout {
    int64_t gu_codes, gu_scales, d_codes, d_scales, globals, total;
};

__host__ __device__ inline int64_t align256(int64_t v) { return (v + 255) / 256 * 256; }

__host__ __device__ inline W16Layout w16_layout(int E, int H, int I) {
    W16Layout L;
    L.gu_codes = 0;
    L.gu_scales = align256(L.gu_codes + (int64_t)E * I * H);
    L.d_codes = align256(L.gu_scales + (int64_t)E * I * H / 8);
    L.d_scales = align256(L.d_codes + (int64_t)E * H * I / 2);
    L.globals = align256(L.d_scales + (int64_t)E * H * I / 16);
    L.total = align256(L.globals + (int64_t)E * 3 * 4);
    return L;
}

// ---------------------------------------------------------------------------
// pack
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t code_at(const uint8_t* codes, const uint8_t* sf, int64_t r, int64_t k, int64_t K) {
    if (sf[r * (K / 16) + k / 16] == 0) return 0;  // a zero-scale block decodes to 0 whatever its codes
    const uint32_t b = codes[r * (K / 2) + k / 2];
    return (k & 1) ? (b >> 4) : (b & 15u);
}

// Fragment word of lane (g, c) for k16 step at column kb of a 16-row tile at r0.
__device__ uint32_t pack_word(const uint8_t* codes, const uint8_t* sf, int64_t r0, int64_t kb, int g, int c,
                              int64_t K) {
    const int64_t ra = r0 + g, rb = r0 + g + 8;
    const int64_t k0 = kb + 2 * c, k1 = kb + 2 * c + 8;
    const uint32_t q0l = code_at(codes, sf, ra, k0, K), q0h = code_at(codes, sf, ra, k0 + 1, K);
    const uint32_t q1l = code_at(codes, sf, rb, k0, K), q1h = code_at(codes, sf, rb, k0 + 1, K);
    const uint32_t q2l = code_at(codes, sf, ra, k1, K), q2h = code_at(codes, sf, ra, k1 + 1, K);
    const uint32_t q3l = code_at(codes, sf, rb, k1, K), q3h = code_at(codes, sf, rb, k1 + 1, K);
    uint32_t w = 0;
    // register 0: magnitude at 6..8 / 22..24, sign at 15 / 31
    w |= ((q0l & 7u) << 6) | ((q0l >> 3) << 15) | ((q0h & 7u) << 22) | ((q0h >> 3) << 31);
    // register 1: stored 3 bits lower
    w |= ((q1l & 7u) << 3) | ((q1l >> 3) << 12) | ((q1h & 7u) << 19) | ((q1h >> 3) << 28);
    // register 2: stored 6 bits lower
    w |= ((q2l & 7u) << 0) | ((q2l >> 3) << 9) | ((q2h & 7u) << 16) | ((q2h >> 3) << 25);
    // register 3: m -> 10, e0 -> 11, e1 -> 13, sign -> 14 (and +16 for the odd element)
    w |= ((q3l & 1u) << 10) | (((q3l >> 1) & 1u) << 11) | (((q3l >> 2) & 1u) << 13) | ((q3l >> 3) << 14);
    w |= ((q3h & 1u) << 26) | (((q3h >> 1) & 1u) << 27) | (((q3h >> 2) & 1u) << 29) | ((q3h >> 3) << 30);
    return w;
}

// One thread per (tile, k64 chunk, lane): 16 code bytes, plus 8 scale bytes for lanes with c == 0.
__global__ void k_w16_pack(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf, int64_t n_tiles,
                           int64_t K, int interleave_gu, const uint8_t* __restrict__ codes2,
                           const uint8_t* __restrict__ sf2, uint8_t* __restrict__ out_codes,
                           uint8_t* __restrict__ out_scales, int64_t rows_per_expert) {
    const int64_t chunks = K / 64;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= n_tiles * chunks * 32) return;
    const int lane = (int)(idx & 31);
    const int64_t chunk = (idx >> 5) % chunks;
    const int64_t tile = (idx >> 5) / chunks;  // packed tile index
    // source tensor and its first row
    const uint8_t* c = codes;
    const uint8_t* s = sf;
    int64_t r0;
    if (interleave_gu) {
        // packed tile order per expert: (iblock, {gate, up}); rows_per_expert = I
        const int64_t tiles_per_expert = rows_per_expert / 16 * 2;
        const int64_t e = tile / tiles_per_expert;
        const int64_t rem = tile % tiles_per_expert;
        const int64_t ib = rem / 2;
        if (rem & 1) {
            c = codes2;
            s = sf2;
        }
        r0 = e * rows_per_expert + ib * 16;
    } else {
        r0 = tile * 16;
    }
    const int g = lane >> 2, cc = lane & 3;
    uint32_t w[4];
#pragma unroll
    for (int st = 0; st < 4; ++st) w[st] = pack_word(c, s, r0, chunk * 64 + st * 16, g, cc, K);
    *reinterpret_cast<uint4*>(out_codes + (tile * chunks + chunk) * 512 + lane * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    if (cc == 0) {
        uint8_t b[8];
#pragma unroll
        for (int st = 0; st < 4; ++st) {
            const int64_t kb = (chunk * 64 + st * 16) / 16;
            b[2 * st] = s[(r0 + g) * (K / 16) + kb];
            b[2 * st + 1] = s[(r0 + g + 8) * (K / 16) + kb];
        }
        uint2 v;
        v.x = b[0] | (b[1] << 8) | (b[2] << 16) | ((uint32_t)b[3] << 24);
        v.y = b[4] | (b[5] << 8) | (b[6] << 16) | ((uint32_t)b[7] << 24);
        *reinterpret_cast<uint2*>(out_scales + (tile * chunks + chunk) * 64 + g * 8) = v;
    }
}

// ---------------------------------------------------------------------------
// dequantisation helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Two E4M3 scales (bytes lo, hi of `pair`) -> BF16x2 multipliers scale * 2^118.
__device__ __forceinline__ uint32_t scale_mult2(uint32_t pair) {
    uint32_t h;
    asm("{\n\t.reg .b16 t;\n\tmov.b16 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h) : "h"((uint16_t)pair));
    return ((h >> 3) & 0x0FFF0FFFu) + 0x73007300u;
}

// 8 codes of one k16 step -> four BF16x2 A-fragment registers scaled by the
// multipliers of rows g (mg) and g + 8 (mg8).
__device__ __forceinline__ void dequant_step(uint32_t q, uint32_t mg, uint32_t mg8, uint32_t a[4]) {
    const uint32_t P = 0x81C081C0u;
    const uint32_t r0 = q & P;
    const uint32_t r1 = (q << 3) & P;
    const uint32_t r2 = (q << 6) & P;
    const uint32_t r3 = ((q >> 4) & 0x00C000C0u) | ((q >> 5) & 0x01000100u) | ((q << 1) & 0x80008000u);
    const uint32_t dg = __byte_perm(mg, mg, 0x1010), dg8 = __byte_perm(mg, mg, 0x3232);
    (void)mg8;
    a[0] = bf16x2_mul(r0, dg);
    a[1] = bf16x2_mul(r1, dg8);
    a[2] = bf16x2_mul(r2, dg);
    a[3] = bf16x2_mul(r3, dg8);
}

__device__ __forceinline__ void mma_bf16(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

// ---------------------------------------------------------------------------
// Weight streaming: every warp owns a ring of W16_STAGES shared-memory stages;
// lane 0 fills a stage with 1-D bulk copies (cp.async.bulk, completion counted
// on the stage's mbarrier) W16_STAGES groups ahead of the consumer, so each SM
// keeps ~200 KB of the weight stream in flight without holding it in registers.
// A stage holds W16_CH consecutive 64-column chunks of both 16-row tiles.
// ---------------------------------------------------------------------------
constexpr int W16_STAGES = 4;
constexpr int W16_CH = 4;
constexpr int W16_STAGE_CODES = 2 * W16_CH * 512;
constexpr int W16_STAGE_SCALES = 2 * W16_CH * 64;
constexpr int W16_STAGE = W16_STAGE_CODES + W16_STAGE_SCALES;
constexpr int W16_WARP_SMEM = W16_STAGES * W16_STAGE;
constexpr int W16_SMEM = W16_WARPS * (W16_WARP_SMEM + W16_STAGES * 8);

struct Ring {
    uint8_t* buf;   // W16_STAGES stages
    uint64_t* bar;  // W16_STAGES mbarriers
    uint32_t ctr;   // groups consumed so far (stage = ctr % S, parity = ctr / S)
};

__device__ __forceinline__ void ring_issue(Ring& r, int stage, const uint8_t* const codes[2],
                                           const uint8_t* const scales[2], int grp, int ch) {
    uint8_t* st = r.buf + stage * W16_STAGE;
    tc::mbar_arrive_expect_tx(&r.bar[stage], 2 * ch * (512 + 64));
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        tc::bulk_load(st + u * W16_CH * 512, codes[u] + (int64_t)grp * ch * 512, ch * 512, &r.bar[stage]);
        tc::bulk_load(st + W16_STAGE_CODES + u * W16_CH * 64, scales[u] + (int64_t)grp * ch * 64, ch * 64,
                      &r.bar[stage]);
    }
}

// Streams `chunks` 64-column chunks of two 16-row tiles and accumulates their
// products with up to W16_MAX_NT 8-token B tiles.  Returns false on a timeout.
__device__ __forceinline__ bool w16_stream(Ring& r, const uint8_t* const codes[2], const uint8_t* const scales[2],
                                           int chunks, const uint16_t* const bptr[W16_MAX_NT], int nt_count,
                                           float acc[2][W16_MAX_NT][4], int32_t* err) {
    const int lane = lane_id();
    const int g = lane >> 2, c = lane & 3;
    const int ch = (chunks % W16_CH == 0) ? W16_CH : 2;
    const int groups = chunks / ch;
    const uint32_t base = r.ctr;
    if (lane == 0)
        for (int i = 0; i < W16_STAGES && i < groups; ++i) ring_issue(r, (base + i) % W16_STAGES, codes, scales, i, ch);
    __syncwarp();
    for (int grp = 0; grp < groups; ++grp) {
        const uint32_t n = base + grp;
        const int stage = n % W16_STAGES;
        if (!tc::mbar_wait(&r.bar[stage], (n / W16_STAGES) & 1u, err)) return false;
        const uint8_t* st = r.buf + stage * W16_STAGE;
        for (int cc = 0; cc < ch; ++cc) {
            uint4 q[2];
            uint2 sc[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                q[u] = *reinterpret_cast<const uint4*>(st + u * W16_CH * 512 + cc * 512 + lane * 16);
                sc[u] = *reinterpret_cast<const uint2*>(st + W16_STAGE_CODES + u * W16_CH * 64 + cc * 64 + g * 8);
            }
            const int kbase = (grp * ch + cc) * 64;
#pragma unroll
            for (int stp = 0; stp < 4; ++stp) {
                const int kb = kbase + stp * 16;
                uint32_t b0[W16_MAX_NT], b1[W16_MAX_NT];
#pragma unroll
                for (int nt = 0; nt < W16_MAX_NT; ++nt) {
                    b0[nt] = b1[nt] = 0;
                    if (nt < nt_count && bptr[nt]) {
                        b0[nt] = __ldg(reinterpret_cast<const uint32_t*>(bptr[nt] + kb + 2 * c));
                        b1[nt] = __ldg(reinterpret_cast<const uint32_t*>(bptr[nt] + kb + 2 * c + 8));
                    }
                }
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint32_t qw = stp == 0 ? q[u].x : stp == 1 ? q[u].y : stp == 2 ? q[u].z : q[u].w;
                    const uint32_t sw = stp < 2 ? sc[u].x : sc[u].y;
                    const uint32_t m = scale_mult2((stp & 1) ? (sw >> 16) : (sw & 0xFFFFu));
                    uint32_t a[4];
                    dequant_step(qw, m, 0, a);
#pragma unroll
                    for (int nt = 0; nt < W16_MAX_NT; ++nt)
                        if (nt < nt_count) mma_bf16(acc[u][nt], a, b0[nt], b1[nt]);
                }
            }
        }
        __syncwarp();  // every lane has read the stage
        if (lane == 0 && grp + W16_STAGES < groups) {
            tc::fence_proxy_async_smem();
            ring_issue(r, stage, codes, scales, grp + W16_STAGES, ch);
        }
    }
    r.ctr = base + groups;
    return true;
}

__device__ __forceinline__ Ring make_ring(uint8_t* smem) {
    Ring r;
    const int w = warp_id();
    r.buf = smem + w * W16_WARP_SMEM;
    r.bar = reinterpret_cast<uint64_t*>(smem + W16_WARPS * W16_WARP_SMEM) + w * W16_STAGES;
    r.ctr = 0;
    if (lane_id() == 0) {
        for (int i = 0; i < W16_STAGES; ++i) tc::mbar_init(&r.bar[i], 1);
        tc::fence_mbar_init();
    }
    __syncwarp();
    return r;
}

// ---------------------------------------------------------------------------
// gate/up GEMM + SwiGLU: warps loop over (active expert, 16 intermediates)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(W16_WARPS * 32)
    k_w16_gateup(const uint16_t* __restrict__ x, const uint8_t* __restrict__ packed, W16Layout L, int H, int I, int k,
                 RoutingPlan plan, uint16_t* __restrict__ A2, int32_t* err) {
    extern __shared__ __align__(128) uint8_t w16_smem[];
    Ring ring = make_ring(w16_smem);
    const int lane = lane_id();
    const int g = lane >> 2, c = lane & 3;
    const int iblocks = I / 16;
    const int chunks = H / 64;
    const int64_t items = (int64_t)plan.n_active[0] * iblocks;
    const float* glob = reinterpret_cast<const float*>(packed + L.globals);
    for (int64_t item = (int64_t)blockIdx.x * W16_WARPS + warp_id(); item < items;
         item += (int64_t)gridDim.x * W16_WARPS) {
        const int e = plan.active[item / iblocks];
        const int ib = (int)(item % iblocks);
        const int n_e = plan.counts[e];
        const int row0 = plan.offsets[e];
        const float ag = glob[e * 3 + 0] * 256.0f, au = glob[e * 3 + 1] * 256.0f;
        const int64_t tile0 = ((int64_t)e * iblocks + ib) * 2;
        const uint8_t* cb[2];
        const uint8_t* sb[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            cb[u] = packed + L.gu_codes + (tile0 + u) * chunks * 512;
            sb[u] = packed + L.gu_scales + (tile0 + u) * chunks * 64;
        }
        for (int n0 = 0; n0 < n_e; n0 += 8 * W16_MAX_NT) {
            const int nt_count = min(W16_MAX_NT, (n_e - n0 + 7) / 8);
            const uint16_t* bptr[W16_MAX_NT];
#pragma unroll
            for (int nt = 0; nt < W16_MAX_NT; ++nt) {
                const int n = n0 + nt * 8 + g;
                bptr[nt] = (nt < nt_count && n < n_e) ? x + (int64_t)(plan.pair_of_row[row0 + n] / k) * H : nullptr;
            }
            float acc[2][W16_MAX_NT][4] = {};
            if (!w16_stream(ring, cb, sb, chunks, bptr, nt_count, acc, err)) return;
#pragma unroll
            for (int nt = 0; nt < W16_MAX_NT; ++nt) {
                if (nt >= nt_count) break;
#pragma unroll
                for (int h = 0; h < 2; ++h) {      // rows g, g + 8
#pragma unroll
                    for (int j = 0; j < 2; ++j) {  // tokens 2c, 2c + 1
                        const int n = n0 + nt * 8 + 2 * c + j;
                        if (n < n_e) {
                            const float gv = acc[0][nt][2 * h + j] * ag;
                            const float uv = acc[1][nt][2 * h + j] * au;
                            const __nv_bfloat16 v = __float2bfloat16_rn(silu(gv) * uv);
                            A2[(int64_t)(row0 + n) * I + ib * 16 + g + 8 * h] = *reinterpret_cast<const uint16_t*>(&v);
                        }
                    }
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// down GEMM x routing weight: warps loop over (active expert, 32 hidden rows)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(W16_WARPS * 32)
    k_w16_down(const uint8_t* __restrict__ packed, W16Layout L, int H, int I, RoutingPlan plan,
               const uint16_t* __restrict__ A2, float* __restrict__ Y, int32_t* err) {
    extern __shared__ __align__(128) uint8_t w16_smem[];
    Ring ring = make_ring(w16_smem);
    const int lane = lane_id();
    const int g = lane >> 2, c = lane & 3;
    const int hblocks = H / 32;
    const int chunks = I / 64;
    const int64_t items = (int64_t)plan.n_active[0] * hblocks;
    const float* glob = reinterpret_cast<const float*>(packed + L.globals);
    for (int64_t item = (int64_t)blockIdx.x * W16_WARPS + warp_id(); item < items;
         item += (int64_t)gridDim.x * W16_WARPS) {
        const int e = plan.active[item / hblocks];
        const int hb = (int)(item % hblocks);
        const int n_e = plan.counts[e];
        const int row0 = plan.offsets[e];
        const float ad = glob[e * 3 + 2] * 256.0f;
        const int64_t tile0 = (int64_t)e * (H / 16) + hb * 2;
        const uint8_t* cb[2];
        const uint8_t* sb[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            cb[u] = packed + L.d_codes + (tile0 + u) * chunks * 512;
            sb[u] = packed + L.d_scales + (tile0 + u) * chunks * 64;
        }
        for (int n0 = 0; n0 < n_e; n0 += 8 * W16_MAX_NT) {
            const int nt_count = min(W16_MAX_NT, (n_e - n0 + 7) / 8);
            const uint16_t* bptr[W16_MAX_NT];
#pragma unroll
            for (int nt = 0; nt < W16_MAX_NT; ++nt) {
                const int n = n0 + nt * 8 + g;
                bptr[nt] = (nt < nt_count && n < n_e) ? A2 + (int64_t)(row0 + n) * I : nullptr;
            }
            float acc[2][W16_MAX_NT][4] = {};
            if (!w16_stream(ring, cb, sb, chunks, bptr, nt_count, acc, err)) return;
#pragma unroll
            for (int nt = 0; nt < W16_MAX_NT; ++nt) {
                if (nt >= nt_count) break;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int n = n0 + nt * 8 + 2 * c + j;
                    if (n < n_e) {
                        const int row = row0 + n;
                        const float w = plan.wts[plan.pair_of_row[row]] * ad;
#pragma unroll
                        for (int u = 0; u < 2; ++u)
#pragma unroll
                            for (int h = 0; h < 2; ++h)
                                Y[(int64_t)row * H + hb * 32 + u * 16 + g + 8 * h] = acc[u][nt][2 * h + j] * w;
                    }
                }
            }
        }
    }
}

}  // namespace

size_t w4a16_packed_size(int E, int H, int I) { return (size_t)w16_layout(E, H, I).total; }

nvfp4moe_status launch_w4a16_pack(const nvfp4moe_expert_weights& w, void* packed, cudaStream_t stream) {
    const int E = w.E, H = w.H, I = w.I;
    const W16Layout L = w16_layout(E, H, I);
    uint8_t* p = static_cast<uint8_t*>(packed);
    {
        const int64_t n_tiles = (int64_t)E * (I / 16) * 2;
        const int64_t threads = n_tiles * (H / 64) * 32;
        k_w16_pack<<<(unsigned)ceil_div(threads, 256), 256, 0, stream>>>(w.gate_codes, w.gate_sf, n_tiles, H, 1,
                                                                         w.up_codes, w.up_sf, p + L.gu_codes,
                                                                         p + L.gu_scales, I);
        NVFP4MOE_CHECK_LAUNCH("w4a16 pack (gate/up)");
    }
    {
        const int64_t n_tiles = (int64_t)E * (H / 16);
        const int64_t threads = n_tiles * (I / 64) * 32;
        k_w16_pack<<<(unsigned)ceil_div(threads, 256), 256, 0, stream>>>(w.down_codes, w.down_sf, n_tiles, I, 0,
                                                                         nullptr, nullptr, p + L.d_codes,
                                                                         p + L.d_scales, H);
        NVFP4MOE_CHECK_LAUNCH("w4a16 pack (down)");
    }
    NVFP4MOE_CUDA(cudaMemcpyAsync(p + L.globals, w.w_global, (size_t)E * 3 * sizeof(float), cudaMemcpyDeviceToDevice,
                                  stream));
    return NVFP4MOE_OK;
}

nvfp4moe_status launch_w4a16_layer(const uint16_t* x, const void* packed, int T, int H, int I, int E, int k,
                                   const RoutingPlan& plan, uint16_t* A2, float* Y, cudaStream_t stream,
                                   cudaEvent_t mid_event) {
    const W16Layout L = w16_layout(E, H, I);
    const uint8_t* p = static_cast<const uint8_t*>(packed);
    // experts with rows <= min(E, T*k): grids cover that bound; warps loop over
    // the (expert, row block) items the device-side active list holds
    const int64_t max_active = std::min<int64_t>(E, (int64_t)T * k);
    const int64_t max_ctas = (int64_t)num_sms() * 3;
    int32_t* err = device_error_word();
    NVFP4MOE_CUDA(cudaFuncSetAttribute(k_w16_gateup, cudaFuncAttributeMaxDynamicSharedMemorySize, W16_SMEM));
    NVFP4MOE_CUDA(cudaFuncSetAttribute(k_w16_down, cudaFuncAttributeMaxDynamicSharedMemorySize, W16_SMEM));
    {
        const int64_t ctas = std::min<int64_t>(ceil_div(max_active * (I / 16), W16_WARPS), max_ctas);
        k_w16_gateup<<<(unsigned)ctas, W16_WARPS * 32, W16_SMEM, stream>>>(x, p, L, H, I, k, plan, A2, err);
        NVFP4MOE_CHECK_LAUNCH("w4a16 gate/up kernel");
    }
    if (mid_event) cudaEventRecord(mid_event, stream);
    {
        const int64_t ctas = std::min<int64_t>(ceil_div(max_active * (H / 32), W16_WARPS), max_ctas);
        k_w16_down<<<(unsigned)ctas, W16_WARPS * 32, W16_SMEM, stream>>>(p, L, H, I, plan, A2, Y, err);
        NVFP4MOE_CHECK_LAUNCH("w4a16 down kernel");
    }
    return NVFP4MOE_OK;
}

}  // namespace nvfp4moe
