// w4a16.cu -- the W4A16 (16-bit activations x NVFP4 weights) expert GEMMs for
// decode-sized batches on sm_100a.
//
// Mode: "AxionML / MiMo-V2.6-Flash-MOPD-NVFP4", "Usage" (BF16-activation,
// weight-only FP4 mode) and "Accuracy".  Expert MLP: "MiMo-V2.6-Flash --
// REAP-50", "Pruning Method" 1 (down(SiLU(gate h) * up h)).
//
// At decode an expert sees ~1-2 tokens, so the layer is a weight stream: every
// active expert's codes and scales are read from HBM once and dequantised in
// registers, which makes the instruction count per weight the limit.  Weights
// are the mma.sync.m16n8k16 "A" operand (16 weight rows), tokens the "B"
// operand (8 per n-tile), both FP16:
//   * E2M1 codes become exact FP16 values with the hardware e2m1x2->f16x2
//     conversion (one instruction per pair), E4M3 block scales with the
//     e4m3x2->f16x2 conversion, and one FP16x2 multiply gives value * scale
//     exactly (at most 5 significant bits, range [2^-10, 2688]);
//   * the BF16 activations (the layer input, and the SwiGLU output rounded to
//     BF16) are rescaled per row by a power of two 2^s that puts the row's
//     largest magnitude in [2^14, 2^15) and converted to FP16: every element
//     within 2^29 of the row's largest keeps its exact BF16 value, smaller ones
//     round below 2^-40 of the largest; the accumulator is scaled back by 2^-s.
// Weight bytes reach shared memory through per-warp cp.async.bulk rings (see
// w16_stream); gate and up rows of the same 16 intermediates are streamed by
// one warp so SwiGLU is applied on the accumulators.  The down GEMM stages its
// weighted per-pair rows in FP32 (a few MB at decode).
#include <algorithm>

#include "common.cuh"
#include "formats.cuh"
#include "moe_internal.cuh"
#include "tc_ptx.cuh"

namespace nvfp4moe {

namespace {

constexpr int W16_WARPS = 4;
constexpr int W16_MAX_NT = 2;  // n-tiles (of 8 tokens) per pass over the weights

// Scale bytes per 16-row tile and 64-column chunk: 64 E4M3 bytes, or 16 bytes
// of 4-bit compact fields (one byte per row).
__host__ __device__ constexpr int w16_chunk_scale_bytes(bool compact) { return compact ? 16 : 64; }
// 64-column chunks per streamed group: 4 when H and I allow it (fewer, larger
// copies: the copy count, not the bytes, limited the stream with 2), else 2.
inline int w16_ch(int H, int I) { return (H % 256 == 0 && I % 256 == 0) ? 4 : 2; }
// Bytes of one 16-row tile's group of CH chunks: the codes, then the scales,
// contiguous, so that one bulk copy moves both.
__host__ __device__ constexpr int w16_group_bytes(bool compact, int CH) {
    return CH * 512 + CH * w16_chunk_scale_bytes(compact);
}

struct W16Layout {
    int64_t gu, d, globals;                  // gate/up and down tiles (codes + scales per group)
    int64_t rexp_g, rexp_u, rexp_d, status;  // compact form only: row exponents [E, I], [E, I], [E, H]; failures
    int64_t total;
};

__host__ __device__ inline int64_t align256(int64_t v) { return (v + 255) / 256 * 256; }

inline W16Layout w16_layout(int E, int H, int I, bool compact) {
    const int ch = w16_ch(H, I);
    const int64_t gb = w16_group_bytes(compact, ch);
    W16Layout L;
    L.gu = 0;
    L.d = align256(L.gu + (int64_t)E * (2 * I / 16) * (H / (64 * ch)) * gb);
    L.globals = align256(L.d + (int64_t)E * (H / 16) * (I / (64 * ch)) * gb);
    int64_t end = L.globals + (int64_t)E * 3 * 4;
    L.rexp_g = L.rexp_u = L.rexp_d = L.status = -1;
    if (compact) {
        L.rexp_g = align256(end);
        L.rexp_u = align256(L.rexp_g + (int64_t)E * I);
        L.rexp_d = align256(L.rexp_u + (int64_t)E * I);
        L.status = align256(L.rexp_d + (int64_t)E * H);
        end = L.status + 16;
    }
    L.total = align256(end);
    return L;
}

// 2^k as FP32 for k in [-126, 127]
__device__ __forceinline__ float pow2f(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }

// ---------------------------------------------------------------------------
// pack: per 16-row tile and 64-column chunk, 512 bytes in fragment order (lane
// l holds 16 bytes: one 32-bit word per k16 step); inside a word byte j holds
// the two consecutive-column codes of A-fragment register j (low nibble = even
// column): j=0 row g cols 2c,2c+1; j=1 row g+8; j=2 row g cols 2c+8,2c+9; j=3
// row g+8.  Scales: 64 bytes per chunk, 8 per row pair g: [s(g,k16 step t),
// s(g+8,t)] for t = 0..3.  Compact form: 32 bytes per pair of chunks, one word
// per row pair g whose byte p (chunk 2j + p) holds row g's two 4-bit fields
// (the chunk's 32-column blocks, low nibble first) and byte 2 + p row g + 8's,
// so a shift and a mask put row g's field in the low half and row g + 8's in
// the high half; the row exponents stay in row order.  A tile's chunks are
// stored in groups of two, codes then scales, and the groups of a tile pair
// (gate and up of 16 intermediates, or two 16-row down tiles) alternate, so one
// copy moves both tiles' group.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t code_at(const uint8_t* codes, int64_t r, int64_t k, int64_t K) {
    const uint32_t b = codes[r * (K / 2) + k / 2];
    return (k & 1) ? (b >> 4) : (b & 15u);
}

__device__ uint32_t pack_word(const uint8_t* codes, int64_t r0, int64_t kb, int g, int c, int64_t K) {
    const int64_t ra = r0 + g, rb = r0 + g + 8;
    const int64_t k0 = kb + 2 * c, k1 = kb + 2 * c + 8;
    const uint32_t b0 = code_at(codes, ra, k0, K) | (code_at(codes, ra, k0 + 1, K) << 4);
    const uint32_t b1 = code_at(codes, rb, k0, K) | (code_at(codes, rb, k0 + 1, K) << 4);
    const uint32_t b2 = code_at(codes, ra, k1, K) | (code_at(codes, ra, k1 + 1, K) << 4);
    const uint32_t b3 = code_at(codes, rb, k1, K) | (code_at(codes, rb, k1 + 1, K) << 4);
    return b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
}

// One thread per (tile, k64 chunk, lane): 16 code bytes, plus the scale bytes
// of rows g, g + 8 for lanes with c == 0.  rexp/rexp2: row exponents of the
// compact form (COMPACT only).
template <bool COMPACT, int CH>
__global__ void k_w16_pack(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf, int64_t n_tiles,
                           int64_t K, int interleave_gu, const uint8_t* __restrict__ codes2,
                           const uint8_t* __restrict__ sf2, uint8_t* __restrict__ out, int64_t rows_per_expert,
                           const int8_t* __restrict__ rexp, const int8_t* __restrict__ rexp2) {
    const int64_t chunks = K / 64;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= n_tiles * chunks * 32) return;
    const int lane = (int)(idx & 31);
    const int64_t chunk = (idx >> 5) % chunks;
    const int64_t tile = (idx >> 5) / chunks;  // packed tile index
    const uint8_t* c = codes;
    const uint8_t* s = sf;
    const int8_t* rx = rexp;
    int64_t r0;
    if (interleave_gu) {
        // packed tile order per expert: (iblock, {gate, up}); rows_per_expert = I
        const int64_t tiles_per_expert = rows_per_expert / 16 * 2;
        const int64_t e = tile / tiles_per_expert;
        const int64_t rem = tile % tiles_per_expert;
        if (rem & 1) {
            c = codes2;
            s = sf2;
            rx = rexp2;
        }
        r0 = e * rows_per_expert + (rem / 2) * 16;
    } else {
        r0 = tile * 16;
    }
    const int g = lane >> 2, cc = lane & 3;
    uint32_t w[4];
#pragma unroll
    for (int st = 0; st < 4; ++st) w[st] = pack_word(c, r0, chunk * 64 + st * 16, g, cc, K);
    // this chunk's place: tiles are stored in pairs (the two a warp streams together),
    // group by group, the pair's two groups adjacent; in a group the codes at
    // (chunk % CH) * 512, the scales after the codes
    constexpr int GB = w16_group_bytes(COMPACT, CH);
    uint8_t* grp = out + ((tile >> 1) * (chunks / CH) + chunk / CH) * 2 * GB + (tile & 1) * GB;
    const int sub = (int)(chunk % CH);
    *reinterpret_cast<uint4*>(grp + sub * 512 + lane * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    if (COMPACT && cc == 0) {
        uint32_t v = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t row = r0 + g + 8 * h;
            const int re = rx[row];
            uint32_t byte = 0;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int64_t b = chunk * 2 + half;  // 32-column block
                int e = 0;
                const int kind = compact_block_kind(s[row * (K / 16) + 2 * b], s[row * (K / 16) + 2 * b + 1], e);
                byte |= (uint32_t)((kind == 0 ? re - e : 15) & 15) << (4 * half);
            }
            v |= byte << (8 * h);
        }
        // one 32-bit word per row pair g and chunk pair: byte (sub & 1) for row g, byte
        // 2 + (sub & 1) for row g + 8
        uint8_t* wd = grp + CH * 512 + (sub >> 1) * 32 + g * 4 + (sub & 1);
        wd[0] = (uint8_t)(v & 0xFFu);
        wd[2] = (uint8_t)(v >> 8);
    } else if (!COMPACT && cc == 0) {
        uint32_t b[8];
#pragma unroll
        for (int st = 0; st < 4; ++st) {
            const int64_t kb = chunk * 4 + st;
            b[2 * st] = s[(r0 + g) * (K / 16) + kb];
            b[2 * st + 1] = s[(r0 + g + 8) * (K / 16) + kb];
        }
        uint2 v;
        v.x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
        v.y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
        *reinterpret_cast<uint2*>(grp + CH * 512 + sub * 64 + g * 8) = v;
    }
}

// ---------------------------------------------------------------------------
// BF16 rows -> FP16 rows with a per-row power-of-two scale (one warp per row),
// written in MMA B-fragment order: inside every 64-column chunk, lane quad c's
// sixteen values (k = 16 t + 2c, 2c+1, 2c+8, 2c+9 for the chunk's four k16 steps
// t) are 32 consecutive bytes, so a lane fetches a step's B fragment (b0, b1)
// with one 8-byte load.
// ---------------------------------------------------------------------------
// NCH > 0: rows of K = 256 * NCH elements, each lane's NCH 16-byte pieces loaded
// once and held in registers (one memory round trip per row instead of two
// passes of dependent loads); NCH == 0: any K (a multiple of 8), two passes.
template <int NCH>
__global__ void __launch_bounds__(256)
    k_rows_to_f16(const uint16_t* __restrict__ src, int64_t rows, int K, __half* __restrict__ dst,
                  float* __restrict__ inv_scale) {
    const int64_t r = (int64_t)blockIdx.x * 8 + warp_id();
    if (r >= rows) return;
    const int lane = lane_id();
    const uint4* s = reinterpret_cast<const uint4*>(src + r * K);
    // lane's pieces: i = lane + 32 c < K / 8
    const int n_c = NCH > 0 ? NCH : (K / 8 - lane + 31) / 32;
    constexpr int HELD = NCH > 0 ? NCH : 1;
    uint4 held[HELD];
    if (NCH > 0) {
#pragma unroll
        for (int c = 0; c < HELD; ++c) held[c] = s[lane + 32 * c];
    }
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < n_c; ++c) {
        const uint4 v = NCH > 0 ? held[c < HELD ? c : 0] : s[lane + 32 * c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
            amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_float(w[q] & 0xFFFFu)), fabsf(bf16_bits_to_float(w[q] >> 16))));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int sh = 0;
    if (amax > 0.0f && isfinite(amax)) {
        int e;
        frexpf(amax, &e);  // amax in [2^(e-1), 2^e)
        sh = 15 - e;       // amax * 2^sh in [2^14, 2^15)
    }
    uint32_t* d = reinterpret_cast<uint32_t*>(dst + r * K);
#pragma unroll
    for (int c = 0; c < n_c; ++c) {
        const int i = lane + 32 * c;
        const uint4 v = NCH > 0 ? held[c < HELD ? c : 0] : s[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const __half2 h = __floats2half2_rn(ldexpf(bf16_bits_to_float(w[q] & 0xFFFFu), sh),
                                                ldexpf(bf16_bits_to_float(w[q] >> 16), sh));
            o[q] = *reinterpret_cast<const uint32_t*>(&h);
        }
        // elements 8i .. 8i+7: chunk i / 8, k16 step (i / 2) % 4, fragment register i % 2;
        // pair j belongs to lane quad j
        const int64_t wbase = (int64_t)(i >> 3) * 32 + ((i >> 1) & 3) * 2 + (i & 1);
#pragma unroll
        for (int q = 0; q < 4; ++q) d[wbase + q * 8] = o[q];
    }
    if (lane == 0) inv_scale[r] = ldexpf(1.0f, -sh);
}

static void launch_rows_to_f16(const uint16_t* src, int64_t rows, int K, __half* dst, float* inv_scale,
                               cudaStream_t stream) {
    const unsigned grid = (unsigned)ceil_div(rows, 8);
    if (K == 4096)
        k_rows_to_f16<16><<<grid, 256, 0, stream>>>(src, rows, K, dst, inv_scale);
    else if (K == 2048)
        k_rows_to_f16<8><<<grid, 256, 0, stream>>>(src, rows, K, dst, inv_scale);
    else
        k_rows_to_f16<0><<<grid, 256, 0, stream>>>(src, rows, K, dst, inv_scale);
}

// Four E4M3 scales (bytes 0..3 of `w`) -> two FP16x2 (exact): bytes 0, 1 and 2, 3.
__device__ __forceinline__ void scales_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// 8 codes of one k16 step -> the four FP16x2 A-fragment registers, scaled by
// the block scales of rows g and g + 8 (m = FP16x2 {scale g, scale g+8}).
__device__ __forceinline__ void dequant_step(uint32_t q, uint32_t m, uint32_t a[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
        : "r"(q));
    // each scale broadcast to both halves: as half2 operations, which the multiply
    // can take as an operand swizzle instead of a separate byte permute
    __half2 mh;
    memcpy(&mh, &m, 4);
    const __half2 dg = __low2half2(mh), dg8 = __high2half2(mh);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __half2 v;
        memcpy(&v, &a[i], 4);
        v = __hmul2(v, (i & 1) ? dg8 : dg);
        memcpy(&a[i], &v, 4);
    }
}

__device__ __forceinline__ void mma_f16(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

// ---------------------------------------------------------------------------
// Weight streaming: every warp owns a ring of STAGES shared-memory stages;
// lane 0 fills a stage with 1-D bulk copies (cp.async.bulk, completion counted
// on the stage's mbarrier) STAGES groups ahead of the consumer, so the
// weight stream stays in flight without occupying registers.  A stage holds
// CH consecutive 64-column chunks of both 16-row tiles of the warp.
// ---------------------------------------------------------------------------
template <int CH>
struct W16Cfg {
    static constexpr int STAGES = CH == 4 ? 3 : 4;
    static constexpr int MIN_CTAS = CH == 4 ? 4 : 5;       // CTAs per SM the register budget is sized for
    static constexpr int STAGE = 2 * w16_group_bytes(false, CH);  // stage stride (the larger form)
    static constexpr int WARP_SMEM = STAGES * STAGE;
    static constexpr int SMEM = W16_WARPS * (WARP_SMEM + STAGES * 8);
};
static_assert(W16Cfg<4>::SMEM * W16Cfg<4>::MIN_CTAS <= 228 * 1024 && W16Cfg<2>::SMEM * W16Cfg<2>::MIN_CTAS <= 228 * 1024,
              "the rings of the CTAs an SM is sized for must fit its shared memory");

struct Ring {
    uint8_t* buf;   // STAGES stages
    uint64_t* bar;  // STAGES mbarriers
    uint32_t ctr;   // groups consumed so far (stage = ctr % S, parity = ctr / S)
};

template <bool COMPACT, int CH>
__device__ __forceinline__ void ring_issue(Ring& r, int stage, const uint8_t* pair, int grp) {
    constexpr int GB2 = 2 * w16_group_bytes(COMPACT, CH);
    uint8_t* st = r.buf + stage * W16Cfg<CH>::STAGE;
    tc::mbar_arrive_expect_tx(&r.bar[stage], GB2);
    tc::bulk_load(st, pair + (int64_t)grp * GB2, GB2, &r.bar[stage]);
}

// Streams `chunks` 64-column chunks of two 16-row tiles and accumulates their
// products with NT 8-token B tiles (FP16 rows in fragment order; every lane's
// pointer is valid, lanes past the expert's tokens read a real row and their
// results are dropped).  Returns false on a timeout.  COMPACT: the scales are
// 4-bit fields n, one per 32 columns, and each weight is multiplied by 2^(13 - n)
// in FP16 (exact); the row factor 2^(r - 13) is applied by the caller, an exact
// power-of-two move, so the result equals the E4M3-scale form's bit for bit.
template <int NT, bool COMPACT, int CH>
__device__ __forceinline__ bool w16_stream(Ring& r, const uint8_t* pair, int chunks, const __half* const bptr[W16_MAX_NT],
                                           float acc[2][W16_MAX_NT][4], int32_t* err) {
    const int lane = lane_id();
    const int g = lane >> 2, c = lane & 3;
    constexpr int STAGES = W16Cfg<CH>::STAGES;
    constexpr int GB = w16_group_bytes(COMPACT, CH);
    const int groups = chunks / CH;
    const uint32_t base = r.ctr;
    if (lane == 0)
        for (int i = 0; i < STAGES && i < groups; ++i) ring_issue<COMPACT, CH>(r, (base + i) % STAGES, pair, i);
    __syncwarp();
    for (int grp = 0; grp < groups; ++grp) {
        const uint32_t n = base + grp;
        const int stage = n % STAGES;
        if (!tc::mbar_wait(&r.bar[stage], (n / STAGES) & 1u, err)) {
            // error path: the bulk copies already issued into this warp's ring land
            // before the warp leaves
            if (lane == 0)
                for (int i = grp; i < min(grp + STAGES, groups); ++i)
                    tc::mbar_drain(&r.bar[(base + i) % STAGES], ((base + i) / STAGES) & 1u);
            return false;
        }
        const uint8_t* st = r.buf + stage * W16Cfg<CH>::STAGE;
#pragma unroll
        for (int cc = 0; cc < CH; ++cc) {
            // this lane's B fragments of the chunk: (b0, b1) of step t at 8 t bytes
            const uint2* bp[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                bp[nt] = reinterpret_cast<const uint2*>(bptr[nt] + (int64_t)(grp * CH + cc) * 64 + c * 16);
            uint4 q[2];
#pragma unroll
            for (int u = 0; u < 2; ++u)
                q[u] = *reinterpret_cast<const uint4*>(st + u * GB + cc * 512 + lane * 16);
            uint32_t m[2][4];  // FP16x2 {scale g, scale g + 8} of each k16 step
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                if (COMPACT) {
                    // the 4-bit fields n of rows g, g + 8 in the two halves of a word;
                    // multiplier 2^(13 - n) = FP16 bits (28 - n) << 10 (the row factor
                    // 2^(r - 13) is applied in the epilogue)
                    static_assert(CH % 2 == 0, "a compact scale word covers two chunks");
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(st + u * GB + CH * 512 + (cc >> 1) * 32 + g * 4);
                    const uint32_t n0 = (w >> (8 * (cc & 1))) & 0x000F000Fu;
                    const uint32_t n1 = (w >> (8 * (cc & 1) + 4)) & 0x000F000Fu;
                    m[u][0] = m[u][1] = 0x70007000u - n0 * 1024u;
                    m[u][2] = m[u][3] = 0x70007000u - n1 * 1024u;
                } else {
                    const uint2 sc = *reinterpret_cast<const uint2*>(st + u * GB + CH * 512 + cc * 64 + g * 8);
                    scales_f16x2x2(sc.x, m[u][0], m[u][1]);
                    scales_f16x2x2(sc.y, m[u][2], m[u][3]);
                }
            }
#pragma unroll
            for (int stp = 0; stp < 4; ++stp) {
                uint2 bw[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) bw[nt] = __ldg(bp[nt] + stp);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint32_t qw = stp == 0 ? q[u].x : stp == 1 ? q[u].y : stp == 2 ? q[u].z : q[u].w;
                    uint32_t a[4];
                    dequant_step(qw, m[u][stp], a);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_f16(acc[u][nt], a, bw[nt].x, bw[nt].y);
                }
            }
        }
        __syncwarp();  // every lane has read the stage
        if (lane == 0 && grp + STAGES < groups) {
            tc::fence_proxy_async_smem();
            ring_issue<COMPACT, CH>(r, stage, pair, grp + STAGES);
        }
    }
    r.ctr = base + groups;
    return true;
}

template <int CH>
__device__ __forceinline__ Ring make_ring(uint8_t* smem) {
    constexpr int STAGES = W16Cfg<CH>::STAGES;
    Ring r;
    const int w = warp_id();
    r.buf = smem + w * W16Cfg<CH>::WARP_SMEM;
    r.bar = reinterpret_cast<uint64_t*>(smem + W16_WARPS * W16Cfg<CH>::WARP_SMEM) + w * STAGES;
    r.ctr = 0;
    if (lane_id() == 0) {
        for (int i = 0; i < STAGES; ++i) tc::mbar_init(&r.bar[i], 1);
        tc::fence_mbar_init();
    }
    __syncwarp();
    return r;
}

// ---------------------------------------------------------------------------
// gate/up GEMM + SwiGLU: warps loop over (active expert, 16 intermediates)
// ---------------------------------------------------------------------------
template <bool COMPACT, int CH>
__global__ void __launch_bounds__(W16_WARPS * 32, W16Cfg<CH>::MIN_CTAS)
    k_w16_gateup(const __half* __restrict__ x16, const float* __restrict__ x_inv, const uint8_t* __restrict__ packed,
                 W16Layout L, int H, int I, int k, RoutingPlan plan, uint16_t* __restrict__ A2, int32_t* err) {
    extern __shared__ __align__(128) uint8_t w16_smem[];
    Ring ring = make_ring<CH>(w16_smem);
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
        const float ag = glob[e * 3 + 0], au = glob[e * 3 + 1];
        const int64_t pair = (int64_t)e * iblocks + ib;  // tiles 2 pair (gate) and 2 pair + 1 (up)
        const uint8_t* tb = packed + L.gu + pair * (chunks / CH) * 2 * w16_group_bytes(COMPACT, CH);
        for (int n0 = 0; n0 < n_e; n0 += 8 * W16_MAX_NT) {
            const int nt_count = min(W16_MAX_NT, (n_e - n0 + 7) / 8);
            const __half* bptr[W16_MAX_NT];
#pragma unroll
            for (int nt = 0; nt < W16_MAX_NT; ++nt) {
                const int n = n0 + nt * 8 + g;
                bptr[nt] = x16 + (int64_t)(plan.pair_of_row[row0 + (n < n_e ? n : n0)] / k) * H;
            }
            float acc[2][W16_MAX_NT][4] = {};
            const bool ok = nt_count == 1 ? w16_stream<1, COMPACT, CH>(ring, tb, chunks, bptr, acc, err)
                                          : w16_stream<2, COMPACT, CH>(ring, tb, chunks, bptr, acc, err);
            if (!ok) return;
            float ph[2][2] = {{1.0f, 1.0f}, {1.0f, 1.0f}};  // [gate, up][rows g, g + 8]: compact row factors
            if (COMPACT) {
                const int64_t r = (int64_t)e * I + ib * 16 + g;
                const int8_t* rg = reinterpret_cast<const int8_t*>(packed + L.rexp_g);
                const int8_t* ru = reinterpret_cast<const int8_t*>(packed + L.rexp_u);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    ph[0][h] = pow2f(rg[r + 8 * h] - 13);
                    ph[1][h] = pow2f(ru[r + 8 * h] - 13);
                }
            }
#pragma unroll
            for (int nt = 0; nt < W16_MAX_NT; ++nt) {
                if (nt >= nt_count) break;
#pragma unroll
                for (int j = 0; j < 2; ++j) {  // tokens 2c, 2c + 1
                    const int n = n0 + nt * 8 + 2 * c + j;
                    if (n < n_e) {
                        const float inv = x_inv[plan.pair_of_row[row0 + n] / k];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {  // rows g, g + 8
                            const float gv = acc[0][nt][2 * h + j] * inv * (ag * ph[0][h]);
                            const float uv = acc[1][nt][2 * h + j] * inv * (au * ph[1][h]);
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
template <bool COMPACT, int CH>
__global__ void __launch_bounds__(W16_WARPS * 32, W16Cfg<CH>::MIN_CTAS)
    k_w16_down(const uint8_t* __restrict__ packed, W16Layout L, int H, int I, RoutingPlan plan,
               const __half* __restrict__ A16, const float* __restrict__ a_inv, float* __restrict__ Y, int32_t* err) {
    extern __shared__ __align__(128) uint8_t w16_smem[];
    Ring ring = make_ring<CH>(w16_smem);
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
        const float ad = glob[e * 3 + 2];
        const int64_t pair = (int64_t)e * (H / 32) + hb;  // 16-row tiles 2 pair, 2 pair + 1
        const uint8_t* tb = packed + L.d + pair * (chunks / CH) * 2 * w16_group_bytes(COMPACT, CH);
        for (int n0 = 0; n0 < n_e; n0 += 8 * W16_MAX_NT) {
            const int nt_count = min(W16_MAX_NT, (n_e - n0 + 7) / 8);
            const __half* bptr[W16_MAX_NT];
#pragma unroll
            for (int nt = 0; nt < W16_MAX_NT; ++nt) {
                const int n = n0 + nt * 8 + g;
                bptr[nt] = A16 + (int64_t)(row0 + (n < n_e ? n : n0)) * I;
            }
            float acc[2][W16_MAX_NT][4] = {};
            const bool ok = nt_count == 1 ? w16_stream<1, COMPACT, CH>(ring, tb, chunks, bptr, acc, err)
                                          : w16_stream<2, COMPACT, CH>(ring, tb, chunks, bptr, acc, err);
            if (!ok) return;
            float ph[2][2] = {{1.0f, 1.0f}, {1.0f, 1.0f}};  // [tile u][rows g, g + 8]: compact row factors
            if (COMPACT) {
                const int8_t* rd = reinterpret_cast<const int8_t*>(packed + L.rexp_d) + (int64_t)e * H + hb * 32 + g;
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int h = 0; h < 2; ++h) ph[u][h] = pow2f(rd[u * 16 + 8 * h] - 13);
            }
#pragma unroll
            for (int nt = 0; nt < W16_MAX_NT; ++nt) {
                if (nt >= nt_count) break;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int n = n0 + nt * 8 + 2 * c + j;
                    if (n < n_e) {
                        const int row = row0 + n;
                        const float w = plan.wts[plan.pair_of_row[row]] * ad * a_inv[row];
#pragma unroll
                        for (int u = 0; u < 2; ++u)
#pragma unroll
                            for (int h = 0; h < 2; ++h)
                                Y[(int64_t)row * H + hb * 32 + u * 16 + g + 8 * h] =
                                    acc[u][nt][2 * h + j] * (w * ph[u][h]);
                    }
                }
            }
        }
    }
}

}  // namespace

size_t w4a16_packed_size(int E, int H, int I, bool compact) { return (size_t)w16_layout(E, H, I, compact).total; }

size_t w4a16_scratch_size(int T, int H, int I, int k) {
    return (size_t)(align256((int64_t)T * H * 2) + align256((int64_t)T * 4) + align256((int64_t)T * k * I * 2) +
                    align256((int64_t)T * k * 4));
}

template <bool COMPACT, int CH>
static nvfp4moe_status pack_tiles(const nvfp4moe_expert_weights& w, uint8_t* p, const W16Layout& L,
                                  cudaStream_t stream) {
    const int E = w.E, H = w.H, I = w.I;
    const int8_t* rg = COMPACT ? reinterpret_cast<const int8_t*>(p + L.rexp_g) : nullptr;
    const int8_t* ru = COMPACT ? reinterpret_cast<const int8_t*>(p + L.rexp_u) : nullptr;
    const int8_t* rd = COMPACT ? reinterpret_cast<const int8_t*>(p + L.rexp_d) : nullptr;
    {
        const int64_t n_tiles = (int64_t)E * (I / 16) * 2;
        const int64_t threads = n_tiles * (H / 64) * 32;
        k_w16_pack<COMPACT, CH><<<(unsigned)ceil_div(threads, 256), 256, 0, stream>>>(
            w.gate_codes, w.gate_sf, n_tiles, H, 1, w.up_codes, w.up_sf, p + L.gu, I, rg, ru);
        NVFP4MOE_CHECK_LAUNCH("w4a16 pack (gate/up)");
    }
    {
        const int64_t n_tiles = (int64_t)E * (H / 16);
        const int64_t threads = n_tiles * (I / 64) * 32;
        k_w16_pack<COMPACT, CH><<<(unsigned)ceil_div(threads, 256), 256, 0, stream>>>(
            w.down_codes, w.down_sf, n_tiles, I, 0, nullptr, nullptr, p + L.d, H, rd, nullptr);
        NVFP4MOE_CHECK_LAUNCH("w4a16 pack (down)");
    }
    return NVFP4MOE_OK;
}

nvfp4moe_status launch_w4a16_pack(const nvfp4moe_expert_weights& w, void* packed, bool compact, cudaStream_t stream) {
    const int E = w.E, H = w.H, I = w.I;
    const W16Layout L = w16_layout(E, H, I, compact);
    uint8_t* p = static_cast<uint8_t*>(packed);
    if (compact) {
        // row exponents and the count of rows without a compact form, then the tiles
        int32_t* n_bad = reinterpret_cast<int32_t*>(p + L.status);
        NVFP4MOE_CUDA(cudaMemsetAsync(n_bad, 0, sizeof(int32_t), stream));
        int8_t* rg = reinterpret_cast<int8_t*>(p + L.rexp_g);
        int8_t* ru = reinterpret_cast<int8_t*>(p + L.rexp_u);
        int8_t* rd = reinterpret_cast<int8_t*>(p + L.rexp_d);
        const nvfp4moe_status st[3] = {
            launch_compact_rows(w.gate_codes, w.gate_sf, (int64_t)E * I, H, rg, nullptr, nullptr, n_bad, stream),
            launch_compact_rows(w.up_codes, w.up_sf, (int64_t)E * I, H, ru, nullptr, nullptr, n_bad, stream),
            launch_compact_rows(w.down_codes, w.down_sf, (int64_t)E * H, I, rd, nullptr, nullptr, n_bad, stream)};
        for (nvfp4moe_status s : st)
            if (s != NVFP4MOE_OK) return s;
        const nvfp4moe_status s =
            w16_ch(H, I) == 4 ? pack_tiles<true, 4>(w, p, L, stream) : pack_tiles<true, 2>(w, p, L, stream);
        if (s != NVFP4MOE_OK) return s;
    } else {
        const nvfp4moe_status s =
            w16_ch(H, I) == 4 ? pack_tiles<false, 4>(w, p, L, stream) : pack_tiles<false, 2>(w, p, L, stream);
        if (s != NVFP4MOE_OK) return s;
    }
    NVFP4MOE_CUDA(cudaMemcpyAsync(p + L.globals, w.w_global, (size_t)E * 3 * sizeof(float), cudaMemcpyDeviceToDevice,
                                  stream));
    if (compact) {
        int32_t bad = 0;
        NVFP4MOE_CUDA(cudaMemcpyAsync(&bad, p + L.status, sizeof(bad), cudaMemcpyDeviceToHost, stream));
        NVFP4MOE_CUDA(cudaStreamSynchronize(stream));
        if (bad != 0) {
            set_error("moe_pack_weights: %d weight rows have no compact scale form (unequal or non-power-of-two "
                      "scale pairs, a zero scale over non-zero codes, or an exponent spread above 14)",
                      bad);
            return NVFP4MOE_ERR_NOT_REPRESENTABLE;
        }
    }
    return NVFP4MOE_OK;
}

template <bool COMPACT, int CH>
static nvfp4moe_status run_w16(const uint16_t* x, const uint8_t* p, const W16Layout& L, int T, int H, int I, int E,
                               int k, const RoutingPlan& plan, uint16_t* A2, float* Y, uint8_t* sc, cudaStream_t stream,
                               cudaEvent_t mid_event) {
    constexpr int SMEM = W16Cfg<CH>::SMEM;
    __half* x16 = reinterpret_cast<__half*>(sc);
    float* x_inv = reinterpret_cast<float*>(sc + align256((int64_t)T * H * 2));
    __half* a16 = reinterpret_cast<__half*>(sc + align256((int64_t)T * H * 2) + align256((int64_t)T * 4));
    float* a_inv = reinterpret_cast<float*>(sc + align256((int64_t)T * H * 2) + align256((int64_t)T * 4) +
                                            align256((int64_t)T * k * I * 2));
    const int64_t P = (int64_t)T * k;
    // experts with rows <= min(E, T*k): grids cover that bound; warps loop over
    // the (expert, row block) items the device-side active list holds
    const int64_t max_active = std::min<int64_t>(E, P);
    const int64_t max_ctas = (int64_t)num_sms() * W16Cfg<CH>::MIN_CTAS;
    int32_t* err = device_error_word();
    NVFP4MOE_CUDA(cudaFuncSetAttribute(k_w16_gateup<COMPACT, CH>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM));
    NVFP4MOE_CUDA(cudaFuncSetAttribute(k_w16_down<COMPACT, CH>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM));
    launch_rows_to_f16(x, T, H, x16, x_inv, stream);
    NVFP4MOE_CHECK_LAUNCH("w4a16 activation conversion");
    {
        const int64_t ctas = std::min<int64_t>(ceil_div(max_active * (I / 16), W16_WARPS), max_ctas);
        k_w16_gateup<COMPACT, CH><<<(unsigned)ctas, W16_WARPS * 32, SMEM, stream>>>(x16, x_inv, p, L, H, I, k, plan,
                                                                                     A2, err);
        NVFP4MOE_CHECK_LAUNCH("w4a16 gate/up kernel");
    }
    if (mid_event) cudaEventRecord(mid_event, stream);
    launch_rows_to_f16(A2, P, I, a16, a_inv, stream);
    NVFP4MOE_CHECK_LAUNCH("w4a16 intermediate conversion");
    {
        const int64_t ctas = std::min<int64_t>(ceil_div(max_active * (H / 32), W16_WARPS), max_ctas);
        k_w16_down<COMPACT, CH><<<(unsigned)ctas, W16_WARPS * 32, SMEM, stream>>>(p, L, H, I, plan, a16, a_inv, Y, err);
        NVFP4MOE_CHECK_LAUNCH("w4a16 down kernel");
    }
    return NVFP4MOE_OK;
}

nvfp4moe_status launch_w4a16_layer(const uint16_t* x, const void* packed, bool compact, int T, int H, int I,
                                   int E, int k, const RoutingPlan& plan, uint16_t* A2, float* Y, void* scratch,
                                   cudaStream_t stream, cudaEvent_t mid_event) {
    const W16Layout L = w16_layout(E, H, I, compact);
    const uint8_t* p = static_cast<const uint8_t*>(packed);
    uint8_t* sc = static_cast<uint8_t*>(scratch);
    const bool ch4 = w16_ch(H, I) == 4;
    if (compact)
        return ch4 ? run_w16<true, 4>(x, p, L, T, H, I, E, k, plan, A2, Y, sc, stream, mid_event)
                   : run_w16<true, 2>(x, p, L, T, H, I, E, k, plan, A2, Y, sc, stream, mid_event);
    return ch4 ? run_w16<false, 4>(x, p, L, T, H, I, E, k, plan, A2, Y, sc, stream, mid_event)
               : run_w16<false, 2>(x, p, L, T, H, I, E, k, plan, A2, Y, sc, stream, mid_event);
}

}  // namespace nvfp4moe
