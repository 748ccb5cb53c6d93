// w4a4.cu -- W4A4 grouped expert GEMMs on the sm_100a 5th-generation tensor
// cores: NVFP4 activations x NVFP4 weights with tcgen05.mma kind::mxf4nvf4
// (E4M3 block scale per 16 elements, FP32 accumulators in tensor memory).
//
// Mode: "AxionML / MiMo-V2.6-Flash-MOPD-NVFP4", introduction (routed experts as
// W4A4 NVFP4 on native FP4 tensor cores) and "Why a unit activation scale".
// Expert MLP: "MiMo-V2.6-Flash -- REAP-50", "Pruning Method" 1.
//
// One persistent kernel per projection in one of two tile forms, chosen per
// call: one CTA per SM computing 128 x 256 output tiles (128 token rows of one
// expert x 256 weight rows) with the single-CTA MMA (cta_group::1) when the
// experts average fewer than 1024 rows, else CTA pairs computing 256 x 256
// tiles with the pair MMA (cta_group::2), each CTA holding half of the tile's A
// and B rows.  Described here for the single-CTA form; per CTA:
//   warp 0      TMA producer: the tile's A rows and both 128-row halves of its B
//               rows (SWIZZLE_128B tensor maps) and their block-scale atoms (1-D
//               bulk copies) into a 4-stage shared-memory ring guarded by
//               mbarriers;
//   warp 1      MMA issuer: four K=64 block-scaled M=128 x N=256 MMAs per stage
//               into the FP32 TMEM accumulator, nothing else (a tcgen05.cp costs
//               the tensor pipe ~60-80 cycles whatever its size, so twelve scale
//               copies per stage would cost more than the stage's MMAs);
//   warps 18..21 scale warps: tcgen05.st of each stage's scale factors into the
//               stage's TMEM scale columns, one warp per lane quadrant;
//   warps 2..17 epilogue: tcgen05.ld of their 32-lane quadrant, then
//               gate/up: SiLU(gate) * up and NVFP4 requantisation per 16 (the
//                        down GEMM's A operand, written straight into its
//                        block-scale layout);
//               down:    x global scale x routing weight, per-pair rows staged
//                        as FP16 with a power-of-two scale per 64 columns.
// Rows of an expert are padded to 128 by the permutation and cut into 128-row
// tiles, so a tile never straddles two experts; padding rows are computed and
// never stored.  128-row tiles instead of the 256-row pair tiles of the CTA-pair
// form cut the padded MMAs of the 8K prefill from 97,536 to ~82,000 rows, for a
// B operand each CTA loads whole (twice the pair form's B bytes per CTA).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "formats.cuh"
#include "gemm_common.cuh"
#include "moe_internal.cuh"
#include "tc_ptx.cuh"

namespace nvfp4moe {

namespace {

// Two tile forms (CG): a CTA computes a 128 x 256 tile with single-CTA MMAs (CG =
// 1: M = 128 token rows, N = 256 weight rows; it holds the tile's 128 rows of A,
// all 256 rows of B and the scale factors of both), or a CTA pair computes a
// 256 x 256 tile with the pair MMA (CG = 2: each CTA holds 128 rows of A, 128
// rows of B, the scale factors of its A rows and of all 256 B rows).  Two operand
// kinds share the kernel:
//   KIND_NVF4  W4A4: A and B E2M1 with E4M3 scales per 16, kind::mxf4nvf4
//              (scale_vec::4X, K=64 per MMA); a stage is 256 K elements.
//   KIND_MXF8  W4A8: A E4M3 with E8M0 scales per 32 (MXFP8), B E2M1 in the padded
//              shared-memory form with E8M0 scales per 32, kind::mxf8f6f4
//              (scale_vec::1X, K=32 per MMA); a stage is 128 K elements.
// Either way an operand row of a stage is 128 bytes (one SWIZZLE_128B row) and a
// stage holds four MMAs.
constexpr int BM = 128, BN = 256;  // rows of A per CTA; rows of B per tile
enum { KIND_NVF4 = 0, KIND_MXF8 = 1 };

template <int KIND>
struct Cfg;
template <>
struct Cfg<KIND_NVF4> {
    static constexpr int BK = 256;        // K elements per stage
    static constexpr int STAGES_1 = 4, STAGES_2 = 5;  // ring stages of the single-CTA and the pair form
    static constexpr int SF_ELEMS = 16;   // elements per scale
    static constexpr int SFA_ATOMS = 4;   // scale atoms (128 rows x 4 scales) per 128 rows per stage
    static constexpr uint32_t SF_STRIDE = 48;  // TMEM scale columns per ring slot: A 4 x 4, B 4 x 8
    static constexpr uint32_t SFB_COL = 16;    // B's first scale column within a slot
};
template <>
struct Cfg<KIND_MXF8> {
    static constexpr int BK = 128;
    static constexpr int STAGES_1 = 4, STAGES_2 = 6;
    static constexpr int SF_ELEMS = 32;
    static constexpr int SFA_ATOMS = 1;
    static constexpr uint32_t SF_STRIDE = 12;  // A 4, B 8 (one word per row holds the stage's four scales)
    static constexpr uint32_t SFB_COL = 4;
};
constexpr int A_BYTES = BM * 128;         // 128 rows x 128 bytes
template <int CG>  // B rows of a CTA x 128 bytes: all 256 (two 128-row copies), or its half of the pair's
__host__ __device__ constexpr int b_bytes() { return (CG == 1 ? BN : BN / 2) * 128; }
template <int KIND, int CG>
__host__ __device__ constexpr int stages() { return CG == 1 ? Cfg<KIND>::STAGES_1 : Cfg<KIND>::STAGES_2; }
template <int KIND>
__host__ __device__ constexpr int sfa_bytes() { return Cfg<KIND>::SFA_ATOMS * 512; }
template <int KIND>
__host__ __device__ constexpr int sfb_bytes() { return 2 * Cfg<KIND>::SFA_ATOMS * 512; }
template <int KIND, int CG>
__host__ __device__ constexpr int stage_bytes() {  // padded to the 1024-byte alignment of swizzled tiles
    return (A_BYTES + b_bytes<CG>() + sfa_bytes<KIND>() + sfb_bytes<KIND>() + 1023) / 1024 * 1024;
}
template <int KIND, int CG>
__host__ __device__ constexpr int smem_bytes() { return stages<KIND, CG>() * stage_bytes<KIND, CG>() + 1024 + 256; }
static_assert(smem_bytes<KIND_NVF4, 1>() <= 232448 && smem_bytes<KIND_MXF8, 1>() <= 232448 &&
                  smem_bytes<KIND_NVF4, 2>() <= 232448 && smem_bytes<KIND_MXF8, 2>() <= 232448,
              "shared-memory ring above the 227 KB a CTA may use");
static_assert(256 + stages<KIND_NVF4, 1>() * Cfg<KIND_NVF4>::SF_STRIDE <= 512 &&
                  256 + stages<KIND_NVF4, 2>() * Cfg<KIND_NVF4>::SF_STRIDE <= 512 &&
                  256 + stages<KIND_MXF8, 2>() * Cfg<KIND_MXF8>::SF_STRIDE <= 512,
              "accumulator + per-slot scale columns must fit the TMEM allocation");
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_SF = 256;  // scale-factor columns after the 256 accumulator columns
constexpr int EPI_WARPS = 16;  // four warps per TMEM lane quadrant, each on a quarter of the columns
constexpr int SF_WARPS = 4;    // one warp per TMEM lane quadrant writes the scale factors
constexpr int THREADS = (2 + EPI_WARPS + SF_WARPS) * 32;

enum { EPI_GATEUP = 0, EPI_DOWN = 1 };

struct W4Layout {
    int64_t gu_codes, gu_sf, d_codes, d_sf, globals, status, total;
};

inline int64_t a256(int64_t v) { return (v + 255) / 256 * 256; }

// W4A4: codes 4 bits and an E4M3 scale per 16 elements (the checkpoint's bytes).
// W4A8: the same 4-bit codes (the tensor map unpacks them into the padded
// shared-memory form the FP8 x FP4 MMA reads) and an E8M0 scale per 32; a
// status word for the pack.
W4Layout w4_layout(int E, int H, int I, bool mx8 = false) {
    const int64_t n = (int64_t)E * 3 * I * H;  // weights of the layer
    const int64_t gu = (int64_t)E * 2 * I * H;
    W4Layout L;
    L.gu_codes = 0;
    L.gu_sf = a256(L.gu_codes + gu / 2);
    L.d_codes = a256(L.gu_sf + (mx8 ? gu / 32 : gu / 16));
    L.d_sf = a256(L.d_codes + (n - gu) / 2);
    L.globals = a256(L.d_sf + (mx8 ? (n - gu) / 32 : (n - gu) / 16));
    L.status = a256(L.globals + (int64_t)E * 3 * 4);
    L.total = mx8 ? a256(L.status + 16) : L.status;
    return L;
}

struct GemmParams {
    int K;                   // reduction length (elements)
    int n_ntiles;            // N / 256
    int64_t b_rows_per_expert;
    const int4* tiles;       // M-tile list
    const int32_t* n_tiles;  // number of M-tiles (device)
    const uint8_t* sfa;      // A block scales, atom layout
    const uint8_t* sfb;      // B block scales, atom layout
    const float* globals;    // [E, 3]
    float act_global;        // global scale of the A operand's NVFP4 codes
    float out_global;        // gate/up: global scale the intermediate is requantised with
    uint8_t* out_codes;      // gate/up: intermediate codes [rows, I/2]
    uint8_t* out_sf;         // gate/up: intermediate scales, atom layout
    int out_k;               // gate/up: I
    __half* Y;               // down: [rows, H] FP16 staged rows (W4A4)
    float* Yf;               // down: [rows, H] FP32 staged rows (W4A8)
    float* y_scale;          // down: [rows, H / 64] power-of-two scale of each 64 staged columns
    int ldy;                 // down: H
    const float* wts;        // down: routing weight of each pair
    const int32_t* pair_of_row;
    int32_t* err;
};

// One stage's MMA j (of four): K=64 block-scaled FP4 (four E4M3 scales per row
// and MMA, own TMEM columns) or K=32 FP8 x FP4 (one E8M0 scale per row and MMA,
// byte j of the stage's scale word).
template <int KIND, int CG>
__device__ __forceinline__ void stage_mma(uint32_t tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t sf_col, int j, uint32_t accumulate) {
    const uint32_t id8 = idesc | ((uint32_t)j << 29) | ((uint32_t)j << 4);  // W4A8: scale byte j
    if (KIND == KIND_NVF4 && CG == 1)
        tc::mma_mxf4nvf4_1(tmem, adesc + 2 * j, bdesc + 2 * j, idesc, sf_col + 4 * j, sf_col + 16 + 8 * j,
                           accumulate);
    else if (KIND == KIND_NVF4)
        tc::mma_mxf4nvf4_pair(tmem, adesc + 2 * j, bdesc + 2 * j, idesc, sf_col + 4 * j, sf_col + 16 + 8 * j,
                              accumulate);
    else if (CG == 1)
        tc::mma_mxf8f6f4_1(tmem, adesc + 2 * j, bdesc + 2 * j, id8, sf_col, sf_col + Cfg<KIND>::SFB_COL, accumulate);
    else
        tc::mma_mxf8f6f4_pair(tmem, adesc + 2 * j, bdesc + 2 * j, id8, sf_col, sf_col + Cfg<KIND>::SFB_COL,
                              accumulate);
}

template <int EPI, int KIND, int CG>
__global__ void __cluster_dims__(CG, 1, 1) __launch_bounds__(THREADS, 1)
    k_w4a4_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmParams p) {
    constexpr int STAGES = stages<KIND, CG>();
    constexpr int STAGE_BYTES = stage_bytes<KIND, CG>();
    constexpr int B_BYTES = b_bytes<CG>();
    constexpr bool PAIR = CG == 2;  // barriers of the even CTA also see the odd CTA's arrivals
    constexpr int SFA_BYTES = sfa_bytes<KIND>();
    constexpr uint32_t TM_SF_STRIDE = Cfg<KIND>::SF_STRIDE;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    uint64_t* sf_ready = full + STAGES;   // the scale warps (pair: both CTAs', on the even CTA's)
    uint64_t* empty = sf_ready + STAGES;  // the MMA thread's commits
    uint64_t* acc_full = empty + STAGES;  // the MMA thread's commits
    uint64_t* acc_empty = acc_full + 1;   // the epilogue warps (pair: both CTAs', on the even CTA's)
    uint64_t* drain = acc_empty + 1;      // the MMAs of an error path
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

    const uint32_t rank = PAIR ? tc::cluster_ctarank() : 0u;  // 0: issues the MMAs
    const int warp = warp_id(), lane = lane_id();
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&sf_ready[s], CG * SF_WARPS);
            tc::mbar_init(&empty[s], 1);
        }
        tc::mbar_init(acc_full, 1);
        tc::mbar_init(acc_empty, CG * EPI_WARPS);
        tc::mbar_init(drain, 1);
        tc::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tc::prefetch_tmap(&tmA);
        tc::prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        if (PAIR) {
            tc::tmem_alloc_pair(tmem_slot, TMEM_COLS);
            tc::tmem_relinquish_pair();
        } else {
            tc::tmem_alloc_1(tmem_slot, TMEM_COLS);
            tc::tmem_relinquish_1();
        }
    }
    // barriers initialised and TMEM allocated (pair: in both CTAs) before any role uses them
    tc::tc_fence_before();
    if (PAIR) tc::cluster_sync();
    else __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // tile units: a CTA, or a CTA pair
    const int cta = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int n_ctas = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    const int total = p.n_tiles[0] * p.n_ntiles;
    // MMA steps (K=64 FP4 or K=32 FP8) and stages of four; scale atoms per 128 rows
    const int ksub_total = KIND == KIND_NVF4 ? p.K / 64 : p.K / 32;
    const int ks_count = (ksub_total + 3) / 4;
    const int atoms_per_row = p.K / Cfg<KIND>::SF_ELEMS / 4;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // Single CTA: the tile's 128 rows of A, its 256 rows of B (two 128-row
        // copies) and the scale factors of both.  Pair: this CTA's half of the pair
        // tile, A rows [128 rank, +128) and B rows [128 rank, +128), the scale
        // factors of its A rows and of all 256 B rows.
        if (lane == 0) {
            // No L2 prefetch: every TMA instruction costs this thread ~85 cycles of
            // issue (a prefetch ~270), and with five copies per stage the issue
            // time, not the memory system, would bound the MMA rate.
            int it = 0;
            for (int tile = cta; tile < total; tile += n_ctas) {
                const int m = tile / p.n_ntiles, n = tile - m * p.n_ntiles;
                const int4 ti = p.tiles[m];
                // rows of this CTA's half that hold pairs; none in the odd half of an
                // expert's last pair tile when its count leaves it empty (then its A
                // operand is not loaded: those accumulator rows are never stored)
                const bool a_live = ti.z > BM * (int)rank;
                const int a_row = ti.y + BM * (int)rank;
                const int64_t b_tile0 = (int64_t)ti.x * p.b_rows_per_expert + (int64_t)n * BN;
                for (int ks = 0; ks < ks_count; ++ks, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    if (!tc::mbar_wait<PAIR>(&empty[s], ph ^ 1u, p.err)) goto drain_loads;
                    // scale atoms of this stage per 128 rows (a partial last stage: W4A4 only)
                    const int na = KIND == KIND_NVF4 ? min(4, ksub_total - ks * 4) : 1;
                    uint8_t* st = smem + s * STAGE_BYTES;
                    // the unpacking copy of W4A8's B counts the packed bytes it reads (half of
                    // what it writes to shared memory)
                    constexpr int B_TX = KIND == KIND_MXF8 ? B_BYTES / 2 : B_BYTES;
                    tc::mbar_arrive_expect_tx(&full[s], B_TX + 2 * na * 512 + (a_live ? A_BYTES + na * 512 : 0));
                    if (a_live) {
                        tc::tma_load_2d(st, &tmA, ks * 128, a_row, &full[s]);
                        const uint8_t* sfa =
                            p.sfa + ((int64_t)(a_row / 128) * atoms_per_row + ks * Cfg<KIND>::SFA_ATOMS) * 512;
                        tc::bulk_load(st + A_BYTES + B_BYTES, sfa, na * 512, &full[s]);
                    }
                    if (PAIR) {
                        tc::tma_load_2d(st + A_BYTES, &tmB, ks * 128, (int32_t)(b_tile0 + BM * rank), &full[s]);
                    } else {
                        tc::tma_load_2d(st + A_BYTES, &tmB, ks * 128, (int32_t)b_tile0, &full[s]);
                        tc::tma_load_2d(st + A_BYTES + B_BYTES / 2, &tmB, ks * 128, (int32_t)(b_tile0 + BM),
                                        &full[s]);
                    }
                    // the stage's scale atoms of all 256 N rows are stored together: one copy
                    // (placed so that rows 128..255 start na atoms after rows 0..127)
                    const uint8_t* sfb =
                        p.sfb + ((b_tile0 / 256) * atoms_per_row * 2 + ks * Cfg<KIND>::SFA_ATOMS * 2) * 512;
                    tc::bulk_load(st + A_BYTES + B_BYTES + SFA_BYTES, sfb, 2 * na * 512, &full[s]);
                }
            }
            // wait for the MMA's release of every slot still in use, so that no
            // completion signal of the other CTA lands after this CTA has finished
            for (int i = it; i < it + STAGES; ++i)
                if (!tc::mbar_wait<PAIR>(&empty[i % STAGES], ((uint32_t)(i / STAGES) & 1u) ^ 1u, p.err))
                    goto drain_loads;
            goto producer_done;
        drain_loads:
            // error path: the copies of the last STAGES issued stages land before the
            // CTA leaves (a full barrier completes when its bytes have arrived)
            for (int i = max(0, it - STAGES); i < it; ++i) tc::mbar_drain(&full[i % STAGES], (uint32_t)(i / STAGES) & 1u);
        producer_done:;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // One thread (pair: of the even CTA) issues the tile's M=128 (pair: 256) x
        // N=256 MMAs; the scale factors are already in TMEM (the scale warps put
        // them there).
        // The tensor pipe accepts few MMAs ahead of the one it executes (an issue
        // returns ~140 cycles after the previous one), so whatever this thread does
        // between stages is pipe idle time.  The wait for the next stage is
        // therefore made before the current stage's last MMA is issued, and
        // overlaps the MMAs still queued.  The loop carries slot, phase, descriptors
        // and scale column forward instead of recomputing them: its own
        // instructions are pipe idle time too.
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = KIND == KIND_NVF4 ? tc::idesc_mxf4nvf4(CG * BM, BN)
                                                     : tc::idesc_mxf8f6f4_e4m3_e2m1(CG * BM, BN, 0);
            const int n_tiles_mine = cta < total ? (total - cta + n_ctas - 1) / n_ctas : 0;
            const int n_it = n_tiles_mine * ks_count;
            const uint64_t adesc0 = tc::desc_sw128(smem);
            constexpr uint64_t STAGE_DESC = STAGE_BYTES >> 4, B_DESC = A_BYTES >> 4;
            if (n_it > 0) {
                if (!tc::mbar_wait<PAIR>(acc_empty, 1u, p.err)) goto done;
                if (!tc::mbar_wait<PAIR>(&sf_ready[0], 0u, p.err)) goto done;
                tc::tc_fence_after();
            }
            int ks = 0, tl = 0, s = 0;
            uint32_t ph = 0;
            uint64_t adesc = adesc0;
            uint32_t sf_col = tmem + TM_SF;
            for (int it = 0; it < n_it; ++it) {
                const int n64 = ks + 1 < ks_count ? 4 : ksub_total - ks * 4;
                const uint64_t bdesc = adesc + B_DESC;
                const uint32_t acc0 = ks != 0;
                if (n64 == 4) {
                    stage_mma<KIND, CG>(tmem, adesc, bdesc, idesc, sf_col, 0, acc0);
                    stage_mma<KIND, CG>(tmem, adesc, bdesc, idesc, sf_col, 1, 1u);
                    stage_mma<KIND, CG>(tmem, adesc, bdesc, idesc, sf_col, 2, 1u);
                } else {
                    for (int j = 0; j < n64 - 1; ++j)
                        stage_mma<KIND, CG>(tmem, adesc, bdesc, idesc, sf_col, j, (ks | j) != 0);
                }
                const int ns = s + 1 == STAGES ? 0 : s + 1;
                const uint32_t nph = ns == 0 ? ph ^ 1u : ph;
                const bool tile_end = ks + 1 == ks_count;
                const bool more = it + 1 < n_it;
                // next stage of the same tile: its scale factors (and so its operands)
                bool ok = true;
                if (more && !tile_end) ok = tc::mbar_wait<PAIR>(&sf_ready[ns], nph, p.err);
                stage_mma<KIND, CG>(tmem, adesc, bdesc, idesc, sf_col, n64 - 1, (ks | (n64 - 1)) != 0);
                if (PAIR) tc::tc_commit_pair(&empty[s], 0x3);
                else tc::tc_commit_1(&empty[s]);
                if (tile_end) {
                    if (PAIR) tc::tc_commit_pair(acc_full, 0x3);
                    else tc::tc_commit_1(acc_full);
                    ks = 0;
                    ++tl;
                    if (more) {
                        // the single accumulator: the epilogues must have read it
                        ok = ok && tc::mbar_wait<PAIR>(acc_empty, ((uint32_t)tl & 1u) ^ 1u, p.err);
                        ok = ok && tc::mbar_wait<PAIR>(&sf_ready[ns], nph, p.err);
                    }
                } else {
                    ++ks;
                }
                if (!ok) goto drain_mma;
                tc::tc_fence_after();
                s = ns;
                ph = nph;
                adesc = ns == 0 ? adesc0 : adesc + STAGE_DESC;
                sf_col = ns == 0 ? tmem + TM_SF : sf_col + TM_SF_STRIDE;
            }
            goto mma_done;
        drain_mma:
            // error path: the MMAs already issued complete before TMEM is freed
            if (PAIR) tc::tc_commit_pair(drain, 0x1);
            else tc::tc_commit_1(drain);
            tc::mbar_drain(drain, 0u);
        mma_done:;
        }
    } else if (warp >= 2 + EPI_WARPS) {
        // ------------------------------------------------------------ scale warps
        // Warp w writes the scale factors of every stage into TMEM lane quadrant
        // w % 4 with tcgen05.st, in the replicated atom layout the
        // MMA reads: lane (32q + l), column c of an atom's 4 holds word c of the
        // atom's 16-byte row l.  Each ring slot has its own scale columns, rewritten
        // only after the slot's MMAs completed (the slot is refilled only after
        // `empty`).  The MMA thread waits for all four (pair: eight) scale warps.
        const int q = warp & 3;
        const uint32_t t_q = tmem + ((uint32_t)(q * 32) << 16);
        int it = 0;
        for (int tile = cta; tile < total; tile += n_ctas) {
            for (int ks = 0; ks < ks_count; ++ks, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                if (!tc::mbar_wait(&full[s], ph, p.err)) goto done;  // completed by this CTA's copies
                const uint8_t* st = smem + s * STAGE_BYTES + A_BYTES + B_BYTES;
                const uint32_t col = t_q + TM_SF + (uint32_t)s * TM_SF_STRIDE;
                if (KIND == KIND_NVF4) {
                    // B's atoms of N rows 128..255 follow the na atoms of rows 0..127 (na < 4
                    // only in a last, partial stage; atoms past na are not read by the MMAs)
                    const int na = min(4, ksub_total - ks * 4);
                    const uint8_t* sb1 = st + SFA_BYTES + na * 512;
                    uint32_t v[48];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint4 a = *reinterpret_cast<const uint4*>(st + j * 512 + lane * 16);
                        const uint4 b0 = *reinterpret_cast<const uint4*>(st + SFA_BYTES + j * 512 + lane * 16);
                        const uint4 b1 = *reinterpret_cast<const uint4*>(sb1 + j * 512 + lane * 16);
                        v[4 * j + 0] = a.x, v[4 * j + 1] = a.y, v[4 * j + 2] = a.z, v[4 * j + 3] = a.w;
                        v[16 + 8 * j + 0] = b0.x, v[16 + 8 * j + 1] = b0.y, v[16 + 8 * j + 2] = b0.z,
                                       v[16 + 8 * j + 3] = b0.w;
                        v[16 + 8 * j + 4] = b1.x, v[16 + 8 * j + 5] = b1.y, v[16 + 8 * j + 6] = b1.z,
                                       v[16 + 8 * j + 7] = b1.w;
                    }
                    tc::tmem_st16(col, v);
                    tc::tmem_st16(col + 16, v + 16);
                    tc::tmem_st16(col + 32, v + 32);
                } else {
                    // one atom of A (columns 0..3) and the two of B (4..7: N rows 0..127, 8..11: 128..255)
                    const uint4 a = *reinterpret_cast<const uint4*>(st + lane * 16);
                    const uint4 b0 = *reinterpret_cast<const uint4*>(st + SFA_BYTES + lane * 16);
                    const uint4 b1 = *reinterpret_cast<const uint4*>(st + 2 * SFA_BYTES + lane * 16);
                    const uint32_t va[4] = {a.x, a.y, a.z, a.w};
                    const uint32_t vb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                    tc::tmem_st4(col, va);
                    tc::tmem_st8(col + 4, vb);
                }
                tc::tmem_st_wait();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (PAIR) tc::mbar_arrive_remote_relaxed(tc::cluster_addr(&sf_ready[s], 0));
                    else tc::mbar_arrive(&sf_ready[s]);
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // warps 2..17: warp w reads TMEM lane quadrant w % 4 (the hardware rule) and
        // column quarter (w - 2) / 4 of the tile.
        const int q = warp & 3;
        const int quarter = (warp - 2) >> 2;
        const int r_in = q * 32 + lane;
        const uint32_t t_row = tmem + ((uint32_t)(q * 32) << 16);
        const uint32_t acc_empty_leader = PAIR ? tc::cluster_addr(acc_empty, 0) : 0u;
        int tl = 0;
        for (int tile = cta; tile < total; tile += n_ctas, ++tl) {
            const int m = tile / p.n_ntiles, n = tile - m * p.n_ntiles;
            const int4 ti = p.tiles[m];
            // this CTA's 128 rows of the tile
            const int n_valid = ti.z - BM * (int)rank;
            const int64_t row0 = (int64_t)ti.y + BM * (int)rank;
            const bool valid = r_in < n_valid;
            const int64_t row = row0 + r_in;
            if (!tc::mbar_wait<PAIR>(acc_full, (uint32_t)tl & 1u, p.err)) goto done;
            tc::tc_fence_after();
            if (EPI == EPI_GATEUP) {
                // columns [0,128) gate, [128,256) up, for intermediates n*128 .. n*128+127;
                // this warp: 32 intermediates.  All of its accumulator values are read
                // and the accumulator released before the arithmetic, so the MMA warp
                // only waits for the TMEM reads.
                const int i0 = n * (BN / 2) + quarter * 32;
                float gv[32], uv[32];
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    tc::tmem_ld16x2(t_row + quarter * 32 + 16 * c, t_row + 128 + quarter * 32 + 16 * c, gv + 16 * c,
                                    uv + 16 * c);
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (PAIR) tc::mbar_arrive_remote_relaxed(acc_empty_leader);
                    else tc::mbar_arrive(acc_empty);
                }
                if (valid) {
                    const float ag = p.globals[ti.x * 3 + 0] * p.act_global;
                    const float au = p.globals[ti.x * 3 + 1] * p.act_global;
                    if (KIND == KIND_NVF4) {
                        const int nkb = p.out_k / 16;
                        uint32_t codes[4], sfw = 0;
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            float a[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) a[i] = silu_fast(gv[16 * c + i] * ag) * (uv[16 * c + i] * au);
                            const uint32_t sf = requant_block16(a, p.out_global, codes[2 * c], codes[2 * c + 1]);
                            sfw |= sf << (8 * c);
                        }
                        *reinterpret_cast<uint4*>(p.out_codes + row * (p.out_k / 2) + i0 / 2) =
                            make_uint4(codes[0], codes[1], codes[2], codes[3]);
                        // the 2 block scales of this row are 2 consecutive bytes of one atom row
                        *reinterpret_cast<uint16_t*>(p.out_sf + sf_atom_offset(row, i0 / 16, nkb)) = (uint16_t)sfw;
                    } else {
                        // the warp's 32 intermediates are one MXFP8 block of this row
                        float a[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) a[i] = silu_fast(gv[i] * ag) * (uv[i] * au);
                        uint32_t w[8];
                        const uint32_t sf = quantize_block32_mx8(a, w);
                        uint4* dst = reinterpret_cast<uint4*>(p.out_codes + row * p.out_k + i0);
                        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                        p.out_sf[sf_atom_offset(row, i0 / 32, p.out_k / 32)] = (uint8_t)sf;
                    }
                }
            } else {
                // y = acc * global * routing weight.  W4A4: staged as FP16 with one
                // power-of-two scale per (row, 64 columns): the warp's 64 accumulator
                // columns are read and released first; then the max picks the scale and
                // y / scale is converted (exact power-of-two scaling, one FP16 rounding).
                // W4A8: staged as FP32 (its MXFP8 activations carry outliers unclipped,
                // so a row's values can sit far above the layer's rms, where an FP16
                // rounding would exceed the output tolerance).
                float v[64];
                const uint32_t t_col = t_row + quarter * 64;
#pragma unroll
                for (int c = 0; c < 2; ++c) tc::tmem_ld16x2(t_col + 32 * c, t_col + 32 * c + 16, v + 32 * c, v + 32 * c + 16);
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (PAIR) tc::mbar_arrive_remote_relaxed(acc_empty_leader);
                    else tc::mbar_arrive(acc_empty);
                }
                // rows past the tile's valid count hold padding: weight 0, never stored
                const float f = valid ? p.globals[ti.x * 3 + 2] * p.act_global * p.wts[p.pair_of_row[row]] : 0.0f;
                const int c8 = lane & 7, g8 = lane >> 3;
                if (KIND == KIND_MXF8) {
#pragma unroll
                    for (int i = 0; i < 64; ++i) v[i] *= f;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float* pk = v + 32 * h;  // 8 chunks of 4 values, transposed in place
                        transpose_chunks8(pk, lane);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int r_j = q * 32 + g8 * 8 + j;
                            if (r_j < n_valid)
                                *reinterpret_cast<float4*>(p.Yf + (row0 + r_j) * p.ldy + (int64_t)n * BN +
                                                           quarter * 64 + h * 32 + c8 * 4) =
                                    make_float4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                        }
                    }
                } else {
                    float amax = 0.0f;
#pragma unroll
                    for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(v[i]));
                    amax *= fabsf(f);
                    // scale = 2^(e - 14) with amax in [2^e, 2^(e+1)): staged magnitudes stay below 2^15
                    int e = 0;
                    if (amax > 0.0f && isfinite(amax)) e = ((__float_as_uint(amax) >> 23) & 0xFF) - 127;
                    e = max(min(e - 14, 100), -100);
                    const float g = ldexpf(f, -e);
                    // pk: this row's 64 FP16 values as 8 chunks of 16 bytes (4 words each)
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        __half2 b = __floats2half2_rn(v[2 * i] * g, v[2 * i + 1] * g);
                        pk[i] = *reinterpret_cast<uint32_t*>(&b);
                    }
                    if (valid) p.y_scale[row * (p.ldy / 64) + n * 4 + quarter] = ldexpf(1.0f, e);
                    transpose_chunks8(pk, lane);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int r_j = q * 32 + g8 * 8 + j;
                        if (r_j < n_valid)
                            *reinterpret_cast<uint4*>(p.Y + (row0 + r_j) * p.ldy + (int64_t)n * BN + quarter * 64 +
                                                      c8 * 8) = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2],
                                                                           pk[4 * j + 3]);
                    }
                }
            }
        }
    }
done:
    // every role is done with TMEM before it is freed; pair: neither CTA frees its
    // TMEM or exits while the other may still signal it
    if (PAIR) {
        __syncthreads();
        tc::tc_fence_before();
        tc::cluster_sync();
    } else {
        tc::tc_fence_before();
        __syncthreads();
    }
    if (warp == 1) {
        tc::tc_fence_after();
        if (PAIR) tc::tmem_dealloc_pair(tmem, TMEM_COLS);
        else tc::tmem_dealloc_1(tmem, TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// pack: gate/up rows interleaved per 128 (a 256-row N-tile = 128 gate rows then
// the same 128 intermediates' up rows), block scales into the atom layout.
// ---------------------------------------------------------------------------
__global__ void k_w4_pack_codes(const uint8_t* __restrict__ src0, const uint8_t* __restrict__ src1, int64_t rows,
                                int64_t row_bytes, int interleave, int64_t rows_per_expert_src,
                                uint8_t* __restrict__ dst) {
    const int64_t vec_per_row = row_bytes / 16;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= rows * vec_per_row) return;
    const int64_t prow = idx / vec_per_row, v = idx - prow * vec_per_row;
    const uint8_t* src = src0;
    int64_t srow = prow;
    if (interleave) {
        const int64_t per_e = 2 * rows_per_expert_src;
        const int64_t e = prow / per_e, p = prow - e * per_e;
        const int64_t b = p / 256, w = p % 256;
        src = w < 128 ? src0 : src1;
        srow = e * rows_per_expert_src + b * 128 + (w & 127);
    }
    reinterpret_cast<uint4*>(dst)[idx] = reinterpret_cast<const uint4*>(src + srow * row_bytes)[v];
}

__global__ void k_w4_pack_sf(const uint8_t* __restrict__ src0, const uint8_t* __restrict__ src1, int64_t rows,
                             int64_t nkb, int interleave, int64_t rows_per_expert_src, uint8_t* __restrict__ dst) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= rows * nkb) return;
    const int64_t prow = idx / nkb, kb = idx - prow * nkb;
    const uint8_t* src = src0;
    int64_t srow = prow;
    if (interleave) {
        const int64_t per_e = 2 * rows_per_expert_src;
        const int64_t e = prow / per_e, p = prow - e * per_e;
        const int64_t b = p / 256, w = p % 256;
        src = w < 128 ? src0 : src1;
        srow = e * rows_per_expert_src + b * 128 + (w & 127);
    }
    dst[wsf_offset(prow, kb, nkb, Cfg<KIND_NVF4>::SFA_ATOMS)] = src[srow * nkb + kb];
}

// W4A8 weight scales: the E8M0 scale per 32 of each block whose two E4M3 scales
// are one power of two 2^e (byte e + 127); a zero-scale block (all codes +-0)
// takes 2^0.  Rows without that form are counted by the compact-form check
// before this runs.  Atom layout with K/32 columns.
__global__ void k_w8_pack_sf(const uint8_t* __restrict__ src0, const uint8_t* __restrict__ src1, int64_t rows,
                             int64_t nkb32, int interleave, int64_t rows_per_expert_src, uint8_t* __restrict__ dst) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= rows * nkb32) return;
    const int64_t prow = idx / nkb32, kb = idx - prow * nkb32;
    const uint8_t* src = src0;
    int64_t srow = prow;
    if (interleave) {
        const int64_t per_e = 2 * rows_per_expert_src;
        const int64_t e = prow / per_e, p = prow - e * per_e;
        const int64_t b = p / 256, w = p % 256;
        src = w < 128 ? src0 : src1;
        srow = e * rows_per_expert_src + b * 128 + (w & 127);
    }
    const uint8_t* s = src + srow * (2 * nkb32) + 2 * kb;
    int e = 0;
    const int kind = compact_block_kind(s[0], s[1], e);
    dst[wsf_offset(prow, kb, nkb32, Cfg<KIND_MXF8>::SFA_ATOMS)] = (uint8_t)(kind == 0 ? e + 127 : 127);
}

// ---------------------------------------------------------------------------
// host: tensor maps and launches
// ---------------------------------------------------------------------------
// Tile units that fit on the device at once (1 CTA per SM): CTAs, or CTA pairs
// (cluster occupancy), per device, kind and form, cached.
template <int KIND, int CG>
int max_resident_units() {
    constexpr int SMEM_BYTES = smem_bytes<KIND, CG>();
    static std::mutex mu;
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        set_error("w4a4: no usable current CUDA device");
        return 0;
    }
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev] == 0) {
        if (cudaFuncSetAttribute(k_w4a4_gemm<EPI_GATEUP, KIND, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 SMEM_BYTES) != cudaSuccess) {
            set_error("w4a4: cannot raise the shared-memory limit to %d bytes", SMEM_BYTES);
            return 0;
        }
        int n = 0;
        cudaError_t e;
        if (CG == 2) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(2 * 74, 1, 1);
            cfg.blockDim = dim3(THREADS, 1, 1);
            cfg.dynamicSmemBytes = SMEM_BYTES;
            e = cudaOccupancyMaxActiveClusters(&n, k_w4a4_gemm<EPI_GATEUP, KIND, CG>, &cfg);
        } else {
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_w4a4_gemm<EPI_GATEUP, KIND, CG>, THREADS,
                                                              SMEM_BYTES);
            n *= num_sms();
        }
        if (e != cudaSuccess || n <= 0) {
            (void)cudaGetLastError();
            n = num_sms() / CG;  // one CTA per SM
        }
        cache[dev] = n;
    }
    return cache[dev];
}

}  // namespace

size_t w4a4_packed_size(int E, int H, int I, bool mx8) { return (size_t)w4_layout(E, H, I, mx8).total; }

nvfp4moe_status launch_w4a4_pack(const nvfp4moe_expert_weights& w, void* packed, bool mx8, cudaStream_t stream) {
    const int E = w.E, H = w.H, I = w.I;
    const W4Layout L = w4_layout(E, H, I, mx8);
    uint8_t* p = static_cast<uint8_t*>(packed);
    const int64_t gu_rows = (int64_t)E * 2 * I, d_rows = (int64_t)E * H;
    if (mx8) {
        // the E8M0 form needs every weight row's scale pairs to be one power of two
        int32_t* n_bad = reinterpret_cast<int32_t*>(p + L.status);
        NVFP4MOE_CUDA(cudaMemsetAsync(n_bad, 0, sizeof(int32_t), stream));
        const nvfp4moe_status st[3] = {
            launch_compact_rows(w.gate_codes, w.gate_sf, (int64_t)E * I, H, nullptr, nullptr, nullptr, n_bad, stream,
                                1 << 20),
            launch_compact_rows(w.up_codes, w.up_sf, (int64_t)E * I, H, nullptr, nullptr, nullptr, n_bad, stream,
                                1 << 20),
            launch_compact_rows(w.down_codes, w.down_sf, d_rows, I, nullptr, nullptr, nullptr, n_bad, stream,
                                1 << 20)};
        for (nvfp4moe_status x : st)
            if (x != NVFP4MOE_OK) return x;
        k_w4_pack_codes<<<(unsigned)ceil_div(gu_rows * (H / 32), 256), 256, 0, stream>>>(
            w.gate_codes, w.up_codes, gu_rows, H / 2, 1, I, p + L.gu_codes);
        k_w8_pack_sf<<<(unsigned)ceil_div(gu_rows * (H / 32), 256), 256, 0, stream>>>(w.gate_sf, w.up_sf, gu_rows,
                                                                                       H / 32, 1, I, p + L.gu_sf);
        k_w4_pack_codes<<<(unsigned)ceil_div(d_rows * (I / 32), 256), 256, 0, stream>>>(w.down_codes, nullptr, d_rows,
                                                                                         I / 2, 0, H, p + L.d_codes);
        k_w8_pack_sf<<<(unsigned)ceil_div(d_rows * (I / 32), 256), 256, 0, stream>>>(w.down_sf, nullptr, d_rows, I / 32,
                                                                                       0, H, p + L.d_sf);
        NVFP4MOE_CHECK_LAUNCH("w4a8 pack");
        NVFP4MOE_CUDA(cudaMemcpyAsync(p + L.globals, w.w_global, (size_t)E * 3 * sizeof(float),
                                      cudaMemcpyDeviceToDevice, stream));
        int32_t bad = 0;
        NVFP4MOE_CUDA(cudaMemcpyAsync(&bad, n_bad, sizeof(bad), cudaMemcpyDeviceToHost, stream));
        NVFP4MOE_CUDA(cudaStreamSynchronize(stream));
        if (bad != 0) {
            set_error("moe_pack_weights: %d weight rows have no E8M0 scale form (the two E4M3 scales of a 32-code "
                      "block must be one power of two, or zero over zero codes)",
                      bad);
            return NVFP4MOE_ERR_NOT_REPRESENTABLE;
        }
        return NVFP4MOE_OK;
    }
    k_w4_pack_codes<<<(unsigned)ceil_div(gu_rows * (H / 32), 256), 256, 0, stream>>>(
        w.gate_codes, w.up_codes, gu_rows, H / 2, 1, I, p + L.gu_codes);
    k_w4_pack_sf<<<(unsigned)ceil_div(gu_rows * (H / 16), 256), 256, 0, stream>>>(w.gate_sf, w.up_sf, gu_rows, H / 16,
                                                                                   1, I, p + L.gu_sf);
    k_w4_pack_codes<<<(unsigned)ceil_div(d_rows * (I / 32), 256), 256, 0, stream>>>(w.down_codes, nullptr, d_rows,
                                                                                     I / 2, 0, H, p + L.d_codes);
    k_w4_pack_sf<<<(unsigned)ceil_div(d_rows * (I / 16), 256), 256, 0, stream>>>(w.down_sf, nullptr, d_rows, I / 16, 0,
                                                                                   H, p + L.d_sf);
    NVFP4MOE_CHECK_LAUNCH("w4a4 pack");
    NVFP4MOE_CUDA(cudaMemcpyAsync(p + L.globals, w.w_global, (size_t)E * 3 * sizeof(float), cudaMemcpyDeviceToDevice,
                                  stream));
    return NVFP4MOE_OK;
}

template <int KIND, int CG>
static nvfp4moe_status run_layer(const void* packed, int H, int I, int E, float act_global_in, float act_global_mid,
                                 int64_t rows_max, int max_tiles, const RoutingPlan& plan, const uint8_t* A1c,
                                 const uint8_t* A1s, uint8_t* A2c, uint8_t* A2s, __half* Y, float* y_scale,
                                 cudaStream_t stream, cudaEvent_t mid_event) {
    constexpr bool MX8 = KIND == KIND_MXF8;
    constexpr int SMEM_BYTES = smem_bytes<KIND, CG>();
    const W4Layout L = w4_layout(E, H, I, MX8);
    const uint8_t* pk = static_cast<const uint8_t*>(packed);
    NVFP4MOE_CUDA(cudaFuncSetAttribute(k_w4a4_gemm<EPI_GATEUP, KIND, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SMEM_BYTES));
    NVFP4MOE_CUDA(cudaFuncSetAttribute(k_w4a4_gemm<EPI_DOWN, KIND, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SMEM_BYTES));
    // A rows in bytes: FP4 two codes per byte, FP8 one per byte.  B: W4A4 copies the
    // packed codes as bytes; W4A8 copies them through a map that unpacks them into
    // the padded form (coordinates in codes: a stage's 128 codes are 128 bytes of
    // shared memory either way, so the x coordinate ks * 128 serves both)
    const int64_t hb = MX8 ? H : H / 2, ib = MX8 ? I : I / 2;
    CUtensorMap mA1, mGU, mA2, mD;
    const bool ok = make_map(&mA1, A1c, hb, rows_max, BM) && make_map(&mA2, A2c, ib, rows_max, BM) &&
                    (MX8 ? make_map_u4(&mGU, pk + L.gu_codes, H, (int64_t)E * 2 * I, BN / 2) &&
                               make_map_u4(&mD, pk + L.d_codes, I, (int64_t)E * H, BN / 2)
                         : make_map(&mGU, pk + L.gu_codes, H / 2, (int64_t)E * 2 * I, BN / 2) &&
                               make_map(&mD, pk + L.d_codes, I / 2, (int64_t)E * H, BN / 2));
    if (!ok) return NVFP4MOE_ERR_CUDA;
    const int units = max_resident_units<KIND, CG>();
    if (units <= 0) return NVFP4MOE_ERR_CUDA;
    GemmParams g{};
    g.tiles = plan.tiles;
    g.n_tiles = plan.n_tiles;
    g.globals = reinterpret_cast<const float*>(pk + L.globals);
    g.err = device_error_word();
    g.wts = plan.wts;
    g.pair_of_row = plan.pair_of_row;
    // gate/up + SwiGLU + requantise: inputs carry act_global_in, the intermediate act_global_mid
    // (MXFP8 activations carry their own power-of-two scales: no global)
    g.act_global = MX8 ? 1.0f : act_global_in;
    g.out_global = MX8 ? 1.0f : act_global_mid;
    g.K = H;
    g.n_ntiles = (2 * I) / BN;
    g.b_rows_per_expert = 2 * I;
    g.sfa = A1s;
    g.sfb = pk + L.gu_sf;
    g.out_codes = A2c;
    g.out_sf = A2s;
    g.out_k = I;
    {
        const int grid = CG * (int)std::min<int64_t>(units, (int64_t)max_tiles * g.n_ntiles);
        k_w4a4_gemm<EPI_GATEUP, KIND, CG><<<grid, THREADS, SMEM_BYTES, stream>>>(mA1, mGU, g);
        NVFP4MOE_CHECK_LAUNCH(MX8 ? "w4a8 gate/up kernel" : "w4a4 gate/up kernel");
    }
    if (mid_event) cudaEventRecord(mid_event, stream);
    // down x routing weight
    g.act_global = MX8 ? 1.0f : act_global_mid;
    g.K = I;
    g.n_ntiles = H / BN;
    g.b_rows_per_expert = H;
    g.sfa = A2s;
    g.sfb = pk + L.d_sf;
    g.Y = Y;
    g.Yf = reinterpret_cast<float*>(Y);  // W4A8 stages FP32 rows in the same buffer
    g.y_scale = y_scale;
    g.ldy = H;
    {
        const int grid = CG * (int)std::min<int64_t>(units, (int64_t)max_tiles * g.n_ntiles);
        k_w4a4_gemm<EPI_DOWN, KIND, CG><<<grid, THREADS, SMEM_BYTES, stream>>>(mA2, mD, g);
        NVFP4MOE_CHECK_LAUNCH(MX8 ? "w4a8 down kernel" : "w4a4 down kernel");
    }
    return NVFP4MOE_OK;
}

nvfp4moe_status launch_w4a4_layer(const void* packed, bool mx8, int T, int H, int I, int E, int k,
                                  float act_global_in, float act_global_mid, int64_t rows_max, int max_tiles,
                                  const RoutingPlan& plan, const uint8_t* A1c, const uint8_t* A1s, uint8_t* A2c,
                                  uint8_t* A2s, __half* Y, float* y_scale, cudaStream_t stream, cudaEvent_t mid_event) {
    (void)T;
    (void)k;
    // the tile form the plan's tile list was cut for
#define W4_RUN(KD, CGV)                                                                                         \
    run_layer<KD, CGV>(packed, H, I, E, act_global_in, act_global_mid, rows_max, max_tiles, plan, A1c, A1s, A2c, \
                       A2s, Y, y_scale, stream, mid_event)
    const bool pair = plan.tile_rows == 2 * MTILE;
    if (mx8) return pair ? W4_RUN(KIND_MXF8, 2) : W4_RUN(KIND_MXF8, 1);
    return pair ? W4_RUN(KIND_NVF4, 2) : W4_RUN(KIND_NVF4, 1);
#undef W4_RUN
}

int w4a4_tile_rows(int64_t T, int k, int E) {
    // CTA pairs (256-row tiles) when experts average 1024 rows or more (their
    // tiles are mostly full, and the pair form loads half the B bytes per CTA
    // and has a deeper ring); single CTAs (128-row tiles) below that, where
    // halving the tile halves each expert's padding
    return T * k >= 1024LL * E ? 2 * MTILE : MTILE;
}

}  // namespace nvfp4moe
