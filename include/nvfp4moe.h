/*
 * nvfp4moe.h -- C ABI of the B200 (sm_100a) routed-expert MoE layer with 4-bit
 * block-scaled (NVFP4) expert weights.
 *
 * Conventions for every entry point:
 *  - Tensor pointers are DEVICE pointers owned by the caller unless a parameter
 *    says "host".  The library never allocates or frees device memory: scratch
 *    comes from a caller-provided workspace whose size a *_workspace_size()
 *    function returns.
 *  - Device pointers must be 16-byte aligned (128-bit loads); a violation
 *    returns NVFP4MOE_ERR_ALIGNMENT before anything is launched.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is the
 *    legacy default stream) and is asynchronous, except where a call says it
 *    is synchronous.
 *  - Arguments are validated on the host before any launch; on error nothing
 *    is launched and outputs are untouched.  A CUDA launch error returns
 *    NVFP4MOE_ERR_CUDA and nvfp4moe_last_error_string() describes it.
 *  - Matrices are row-major.  Packed E2M1 (FP4) holds two codes per byte, the
 *    even element in the low nibble.  NVFP4 = E2M1 codes + one E4M3 scale per 16
 *    consecutive elements of a row + one FP32 global scale per tensor; MXFP4 =
 *    E2M1 codes + one E8M0 scale per 32.
 *
 * Sources (web pages, by title and section): "AxionML / MiMo-V2.6-Flash-MOPD-
 * NVFP4" (introduction; "About NVFP4 quantization"; "Why a unit activation
 * scale"; "Usage"), "ProCreations/MiMo-V2.6-Flash-RL-NVFP4" ("What changed"),
 * "MiMo-V2.6-Flash -- REAP-50" ("Model Summary"; "Pruning Method" 1).
 */
#ifndef NVFP4MOE_H_
#define NVFP4MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum nvfp4moe_status {
    NVFP4MOE_OK = 0,
    NVFP4MOE_ERR_INVALID_ARG = 1,         /* null pointer, negative size, bad enum  */
    NVFP4MOE_ERR_ALIGNMENT = 2,           /* a device pointer is not 16-byte aligned */
    NVFP4MOE_ERR_UNSUPPORTED_SHAPE = 3,   /* a size constraint of the call is broken */
    NVFP4MOE_ERR_NAN_SCALE = 4,           /* an E8M0 scale of a non-zero block is NaN */
    NVFP4MOE_ERR_NOT_REPRESENTABLE = 5,   /* a tensor has no exact NVFP4 transcode   */
    NVFP4MOE_ERR_WORKSPACE_TOO_SMALL = 6, /* workspace_bytes below the required size */
    NVFP4MOE_ERR_CUDA = 7,                /* a CUDA runtime / launch error            */
    NVFP4MOE_ERR_TIMEOUT = 8,             /* a bounded device-side wait gave up       */
    NVFP4MOE_ERR_UNSUPPORTED_DEVICE = 9   /* the current device is not sm_100         */
} nvfp4moe_status;

/* Text of the last error raised on this host thread (never NULL). */
const char* nvfp4moe_last_error_string(void);

/* Library version, (major << 16) | minor. */
int32_t nvfp4moe_version(void);

/* ------------------------------------------------------------------------- */
/* MXFP4 -> NVFP4 exact transcode                                             */
/* ------------------------------------------------------------------------- */
/* Operation ("AxionML ... NVFP4" introduction and "Reproduce the checkpoint";
 * "ProCreations ... NVFP4", "What changed"): every E2M1 code is kept byte for
 * byte; each E8M0 scale 2^k over 32 codes becomes two equal E4M3 scales over the
 * two 16-code halves, times one power-of-two FP32 global scale per tensor, with
 * nothing re-rounded.  Per tensor, over the blocks whose 32 codes are not all
 * +-0: g = k_max - 8 and each block's E4M3 scale is exactly 2^(k - g); all-zero
 * blocks get scale 0; a tensor without non-zero blocks gets g = 0.  A tensor
 * whose exponent spread k_max - k_min exceeds 17 (E4M3 holds exactly the powers
 * 2^-9..2^8) is NOT representable: it is reported, its scales are zero-filled
 * and its global is 0 (its codes are still copied).  A NaN E8M0 (0xFF) on a
 * non-zero block is reported the same way with its own status.
 *
 * Layout: num_tensors matrices [N, K] stored contiguously.
 *   codes_in/codes_out  uint8 [num_tensors, N, K/2]; codes_out may equal
 *                       codes_in (in place: the codes are then not rewritten).
 *   e8m0_in             uint8 [num_tensors, N, K/32]
 *   e4m3_out            uint8 [num_tensors, N, K/16]
 *   global_scale_out    float [num_tensors]
 *   tensor_status_out   int32 [num_tensors]: 0 exact, 1 not representable,
 *                       2 NaN scale (NVFP4MOE_TENSOR_*)
 *   workspace           device scratch of nvfp4moe_transcode_workspace_size()
 *                       bytes; on return it holds the device-side report.
 *   report_host         HOST pointer or NULL.  Non-NULL makes the call
 *                       SYNCHRONOUS: it waits for the stream, fills the report
 *                       and returns NVFP4MOE_ERR_NOT_REPRESENTABLE or
 *                       NVFP4MOE_ERR_NAN_SCALE if any tensor failed (the other
 *                       tensors are still written).  NULL keeps it asynchronous
 *                       and the per-tensor statuses carry the outcome.
 * Constraints: K % 32 == 0, N >= 1, num_tensors >= 0 (0 is a no-op).         */
enum { NVFP4MOE_TENSOR_EXACT = 0, NVFP4MOE_TENSOR_NOT_REPRESENTABLE = 1, NVFP4MOE_TENSOR_NAN_SCALE = 2 };

typedef struct nvfp4moe_transcode_report {
    int64_t blocks;                   /* 32-code blocks examined            */
    int64_t zero_blocks;              /* blocks whose codes are all +-0     */
    int64_t nonrepresentable_tensors; /* spread > 17                        */
    int64_t nan_scale_tensors;        /* NaN E8M0 on a non-zero block       */
} nvfp4moe_transcode_report;

size_t nvfp4moe_transcode_workspace_size(int64_t num_tensors);

nvfp4moe_status transcode_mxfp4_to_nvfp4(const uint8_t* codes_in, const uint8_t* e8m0_in, int64_t num_tensors,
                                         int64_t N, int64_t K, uint8_t* codes_out, uint8_t* e4m3_out,
                                         float* global_scale_out, int32_t* tensor_status_out, void* workspace,
                                         size_t workspace_bytes, nvfp4moe_transcode_report* report_host,
                                         void* stream);

/* ------------------------------------------------------------------------- */
/* Compact scales (4.125 bits per weight)                                     */
/* ------------------------------------------------------------------------- */
/* Operation ("MiMo-V2.6-Flash-MOPD on one RTX PRO 6000", "Speed v6": a lossless
 * compact expert encoding of 4.125 instead of 4.5 bits per weight; "AxionML ...
 * NVFP4", introduction: a transcode's two E4M3 scales per 32 codes are the
 * same power of two).  Per row of K codes: one exponent r and one 4-bit field
 * n per 32 codes; the block's scale is 2^(r - n) for n = 0..14, 0 for n = 15.
 * A row has a compact form when every 32-code block's two E4M3 scales have
 * equal value and that value is an exact positive power of two 2^e, or 0 with
 * all 32 codes +-0; r = the largest such e of the row (0 if none), and each
 * block needs r - e <= 14.
 *   codes      uint8 [rows, K/2] E2M1 (read only for zero-scale blocks)
 *   e4m3_sf    uint8 [rows, K/16]
 *   nib_out    uint8 [rows, K/64]: byte j = field of block 2j (low nibble) |
 *              field of block 2j+1 << 4; 0xFF for a row without compact form
 *   row_exp_out int8 [rows]: r (0 for a row without compact form)
 *   row_status_out int32 [rows]: 0 compact form exists, 1 not
 *   n_bad_out  int32 [1] or NULL: the number of rows without compact form
 * Constraints: K % 64 == 0, rows >= 0 (0 is a no-op).  Asynchronous.        */
nvfp4moe_status nvfp4_compact_scales(const uint8_t* codes, const uint8_t* e4m3_sf, int64_t rows, int64_t K,
                                     uint8_t* nib_out, int8_t* row_exp_out, int32_t* row_status_out,
                                     int32_t* n_bad_out, void* stream);

/* ------------------------------------------------------------------------- */
/* Grouped sigmoid top-k routing                                              */
/* ------------------------------------------------------------------------- */
/* Operation ("MiMo-V2.6-Flash -- REAP-50", "Model Summary" and "Pruning Method"
 * 1): the E experts are reshaped into [n_group, E/n_group]; s = sigmoid(logit)
 * and c = s + bias (bias only steers the selection, NULL = 0); a group's score
 * is the sum of its two largest c (its largest if a group has one expert); the
 * topk_group best groups are kept and the top_k experts by c inside them are
 * chosen, ties always to the lower index; ids are written in selection order.
 * Weights: renormalize != 0: w_j = (s_j / sum of the chosen s in output order)
 * * routed_scaling_factor, else w_j = s_j * routed_scaling_factor, in IEEE FP32
 * operations.  sigmoid(x) = 1 / (1 + exp(-x)) for x >= 0, else e / (1 + e) with
 * e = exp(x), using a specified FP32 exp: clamp to [-87, 88]; n = rint(x log2 e);
 * Cody-Waite reduction r = fma(-n, ln2_hi, x), r = fma(-n, ln2_lo, r) with
 * ln2_hi = FP32(ln 2) with 12 low mantissa bits cleared and ln2_lo =
 * FP32(ln 2 - ln2_hi); degree-7 Taylor polynomial in r (coefficients FP32(1/i!),
 * Horner with fma); times 2^n.  Ids and weights are therefore bit-reproducible.
 *   logits [T, E] f32; bias [E] f32 or NULL; topk_ids [T, top_k] i32;
 *   topk_weights [T, top_k] f32.
 * Constraints: 1 <= E <= 1024, E % n_group == 0, 1 <= n_group <= 32,
 * 1 <= topk_group <= n_group, 1 <= top_k <= min(32, topk_group * E / n_group),
 * T >= 0 (0 is a no-op).  NaN logits give unspecified choices.  Bias: a NaN
 * entry makes that expert's c count as -inf (it ranks last), and a group whose
 * score is NaN (biases of +inf and -inf in one group) scores -inf; infinite
 * biases are otherwise ordinary values.  Whatever the bias, every id is in
 * [0, E) and a token's ids are distinct.                                      */
nvfp4moe_status moe_route(const float* logits, const float* bias, int32_t T, int32_t E, int32_t n_group,
                          int32_t topk_group, int32_t top_k, float routed_scaling_factor, int32_t renormalize,
                          int32_t* topk_ids, float* topk_weights, void* stream);

/* ------------------------------------------------------------------------- */
/* Router projection followed by the grouped top-k                           */
/* ------------------------------------------------------------------------- */
/* Operation ("MiMo-V2.6-Flash-MOPD on one RTX PRO 6000", "Speed v6" and "What
 * makes it fast": the router's matmul followed by a fused top-k; routers kept
 * in F32 per the tensor precision table of "baekpica MiMo-V2.6-Flash-RL
 * mixed-quant GGUF"): logits[t][e] = sum_h x[t][h] * w_router[e][h] in FP32
 * arithmetic (BF16 hidden rows, FP32 router rows; each logit summed in a fixed
 * order, so repeated calls give the same bits), written to logits_out, then
 * routed exactly as moe_route routes logits_out (same ids and weight bits).
 * Two kernel launches: the projection, then moe_route's routing kernel.  The
 * projection has two forms.  Small T: each logit is the in-order sum of KS
 * slice sums (KS = 8, 4 or 2 as H % 1024, % 512, % 256 allows), each a warp
 * butterfly over 32 lane chains of H / (32 KS) FMAs; error at most
 * (H/64 + 6) * 2^-24 * sum_h |x_h w_h|.  When ceil(T/128) * ceil(E/64) reaches
 * the device's SM count: a tiled FP32 GEMM in which each logit is the FMA
 * chain over the even 16-column chunks of H plus the chain over the odd ones;
 * error at most gamma_(H/2+1) = n 2^-24 / (1 - n 2^-24), n = H/2 + 1, times
 * the same sum.  The two forms may differ in the last bits of a logit, so the
 * routing of one token can depend on how many tokens share the call.
 *   x_bf16 [T, H] bf16 bits; w_router [E, H] f32; bias [E] f32 or NULL;
 *   logits_out [T, E] f32; topk_ids [T, top_k] i32; topk_weights [T, top_k]
 *   f32 (caller-owned device memory); workspace: device, at least
 *   moe_router_topk_workspace_size(T) bytes, caller-owned; this version
 *   neither reads nor writes it (the size is kept so callers need not change).
 * Constraints: as moe_route, plus T <= 8,388,480 (65535 x 128), H >= 256
 * with H % 256 == 0 and E % 4 == 0; all pointers 16-byte aligned.           */
size_t moe_router_topk_workspace_size(int32_t T);
nvfp4moe_status moe_router_topk(const uint16_t* x_bf16, const float* w_router, const float* bias, int32_t T,
                                int32_t H, int32_t E, int32_t n_group, int32_t topk_group, int32_t top_k,
                                float routed_scaling_factor, int32_t renormalize, float* logits_out,
                                int32_t* topk_ids, float* topk_weights, void* workspace, size_t workspace_bytes,
                                void* stream);

/* ------------------------------------------------------------------------- */
/* Token permutation                                                          */
/* ------------------------------------------------------------------------- */
/* Operation (grouped experts: "AxionML ... NVFP4", "Usage", fused grouped MoE
 * backend; "MiMo-V2.6-Flash-MOPD on one RTX PRO 6000", "Speed v4", exact grouped
 * kernel): the T*top_k (token, slot) pairs are grouped by expert so each
 * expert's rows are contiguous; inside an expert rows follow token order (a
 * token selects an expert at most once).  Expert e's rows start at
 * pad_offsets_out[e], a prefix sum of the counts each rounded up to `pad`
 * (pad = 128 is the layout of the W4A4 GEMMs, 1 gives the plain grouping).
 *   topk_ids [T, top_k] i32 (each in [0, E), distinct within a row);
 *   counts_out [E] i32; pad_offsets_out [E+1] i32; row_of_pair_out [T*top_k]
 *   i32 (row of pair t*top_k + j); workspace of moe_permute_workspace_size().
 * Constraints: 1 <= E <= 1024, 1 <= top_k <= 32, pad in {1, 128}, T >= 0;
 * T * top_k plus the padding rows fits int32 (else ERR_UNSUPPORTED_SHAPE).
 * An id outside [0, E) is skipped (not counted; its row_of_pair entry is left
 * as it was); repeated ids within a row give unspecified rows.               */
size_t moe_permute_workspace_size(int32_t T, int32_t E, int32_t top_k, int32_t pad);

nvfp4moe_status moe_permute(const int32_t* topk_ids, int32_t T, int32_t E, int32_t top_k, int32_t pad,
                            int32_t* counts_out, int32_t* pad_offsets_out, int32_t* row_of_pair_out, void* workspace,
                            size_t workspace_bytes, void* stream);

/* moe_permute without a workspace.  The pages have no counterpart to this call:
 * it exists for callers that cannot allocate device memory, such as a plugin
 * inside an inference engine that owns every device buffer and hands the plugin
 * only its inputs and outputs, or a latency-critical path where cudaMalloc
 * (which may synchronise the device) is not allowed.  Same operation, arguments
 * and outputs as moe_permute, minus the workspace: the scratch is one static
 * device array of NVFP4MOE_NOALLOC_SCRATCH_BYTES (1 MiB) inside the library,
 * held on every GPU that loads the library until the process exits.
 *   - Sizes whose moe_permute_workspace_size() exceeds that array are rejected
 *     with NVFP4MOE_ERR_UNSUPPORTED_SHAPE before anything is launched;
 *     T * top_k <= 65536 with E <= 256 always fits.
 *   - The first call on a device looks up the array's device address (with that
 *     device current), and so does the first call in a new CUDA context of the
 *     device (after cudaDeviceReset, say): make those calls before any stream
 *     capture.
 *   - No call allocates or frees device memory.
 *   - All calls share the one array and it keeps the last call's contents:
 *     calls whose work overlaps on the GPU (other streams, other host threads)
 *     race; serialise them.  Nothing in the array needs clearing between calls. */
#define NVFP4MOE_NOALLOC_SCRATCH_BYTES (1u << 20)

nvfp4moe_status moe_permute_noalloc(const int32_t* topk_ids, int32_t T, int32_t E, int32_t top_k, int32_t pad,
                                    int32_t* counts_out, int32_t* pad_offsets_out, int32_t* row_of_pair_out,
                                    void* stream);

/* ------------------------------------------------------------------------- */
/* NVFP4 activation quantisation                                              */
/* ------------------------------------------------------------------------- */
/* Operation ("AxionML ... NVFP4", "About NVFP4 quantization" and "Why a unit
 * activation scale"): per 16-element block of a row, amax = max|x|;
 * sf = E4M3 round-to-nearest-even, saturating at 448, of (amax / 6) / gs; if sf
 * decodes to 0 the 16 codes are 0, else q_i = E2M1 round-to-nearest-even,
 * saturating at 6, of x_i / (value(sf) * gs), sign kept (-0 -> code 8).  All
 * divisions are IEEE FP32.  gs is the dequantisation global scale (1.0f for the
 * pages' unit scale).
 *   x [M, K] BF16 bit patterns; codes [M, K/2]; e4m3_scales [M, K/16].
 * Constraints: K % 16 == 0, M >= 0, gs finite and > 0.                       */
nvfp4moe_status quantize_nvfp4(const uint16_t* x_bf16, int64_t M, int64_t K, float gs, uint8_t* codes,
                               uint8_t* e4m3_scales, void* stream);

/* MXFP8 activation quantisation ("MiMo-V2.6-Flash-MOPD on one RTX PRO 6000",
 * "Speed v5.2" and "Quantization, context and quality": E4M3 elements with one
 * power-of-two scale per 32 values, the prefill activations of the W4A8 mode).
 * Scale choice (the OCP microscaling one; the pages do not spell it out): per 32
 * consecutive elements of a row, X = floor(log2 amax) - 8 clamped to
 * [-127, 127] (-127 when amax is 0 or below the FP32 normal range); scale byte
 * X + 127 (E8M0); element E4M3 round-to-nearest-even, saturating to +-448, of
 * x * 2^-X (the sign of a zero result is kept).
 *   x_bf16 [M, K] BF16 bit patterns; codes [M, K] E4M3 bytes; e8m0_scales
 *   [M, K/32].  Constraints: K % 32 == 0, M >= 0 (0 is a no-op).            */
nvfp4moe_status quantize_mxfp8(const uint16_t* x_bf16, int64_t M, int64_t K, uint8_t* codes, uint8_t* e8m0_scales,
                               void* stream);

/* ------------------------------------------------------------------------- */
/* The MoE layer                                                              */
/* ------------------------------------------------------------------------- */
/* Expert MLP ("MiMo-V2.6-Flash -- REAP-50", "Pruning Method" 1):
 *   out[t] = sum_j w_{t,j} * W_down,e( SiLU(W_gate,e x_t) (.) (W_up,e x_t) ),
 * e = topk_ids[t, j].  Modes ("AxionML ... NVFP4", "Usage" and "Accuracy"):
 *   NVFP4MOE_W4A16: BF16 activations x NVFP4 weights (weights dequantised in
 *                   registers to BF16 tensor-core MMA); SwiGLU output rounded
 *                   to BF16.  Meant for decode-sized batches.
 *   NVFP4MOE_W4A16C: NVFP4MOE_W4A16 arithmetic on weights stored with compact
 *                   scales (see nvfp4_compact_scales): 4.125 instead of 4.5
 *                   bits per weight, the same values, the same outputs bit for
 *                   bit.  Needs weights whose scale pairs are equal powers of
 *                   two (the MXFP4 transcode gives exactly that).
 *   NVFP4MOE_W4A4:  activations quantised to NVFP4 with global act_global (1.0
 *                   in the pages' recipe); FP4 x FP4 block-scaled tcgen05 MMA;
 *                   SwiGLU output requantised per 16 with the same global
 *                   (moe_forward_ex takes a separate global for it).
 *   NVFP4MOE_W4A8:  activations (layer input and SwiGLU output) quantised to
 *                   MXFP8 (see quantize_mxfp8) on the block-scaled FP8 x FP4
 *                   tcgen05 MMA ("MiMo-V2.6-Flash-MOPD on one RTX PRO 6000",
 *                   "Speed v5.2"); the weights keep their E2M1 codes and take
 *                   each 32-code block's power-of-two scale as E8M0, so they
 *                   must have that form (the MXFP4 transcode gives it); the
 *                   activation globals are not used.
 * FP32 accumulation throughout; the combine adds the k weighted expert rows of a
 * token in slot order in FP32 and rounds once to the output type.
 *
 * Weights: expert weights in the checkpoint layout (one NVFP4 tensor per expert
 * projection), which moe_pack_weights rearranges once into the layout the GEMM
 * kernels read:
 */
typedef enum nvfp4moe_mode {
    NVFP4MOE_W4A16 = 0,
    NVFP4MOE_W4A4 = 1,
    NVFP4MOE_W4A16C = 2,
    NVFP4MOE_W4A8 = 3
} nvfp4moe_mode;

typedef struct nvfp4moe_expert_weights {
    const uint8_t* gate_codes; /* [E, I, H/2]  */
    const uint8_t* gate_sf;    /* [E, I, H/16] E4M3 */
    const uint8_t* up_codes;   /* [E, I, H/2]  */
    const uint8_t* up_sf;      /* [E, I, H/16] */
    const uint8_t* down_codes; /* [E, H, I/2]  */
    const uint8_t* down_sf;    /* [E, H, I/16] */
    const float* w_global;     /* [E, 3] global scales: gate, up, down */
    int32_t E, H, I;
} nvfp4moe_expert_weights;

/* Bytes of the packed weights for `mode` (a pure function of the sizes). */
size_t moe_packed_weights_size(nvfp4moe_mode mode, int32_t E, int32_t H, int32_t I);

/* One-time rearrangement of the checkpoint tensors into `packed` (device,
 * moe_packed_weights_size bytes, owned by the caller).  No counterpart on the
 * pages: a layout step for the GEMMs below.  Values are unchanged:
 * the packed buffer holds the same codes, scales and globals, reordered (gate and
 * up rows interleaved, MMA scale-factor layout for W4A4, fragment order for
 * W4A16).  Constraints: H % 128 == 0, I % 128 == 0, E >= 1.
 * NVFP4MOE_W4A16C re-encodes the scales (nvfp4_compact_scales) and is
 * SYNCHRONOUS: it waits for `stream` and returns NVFP4MOE_ERR_NOT_REPRESENTABLE
 * when any weight row has no compact form (the packed buffer is then unusable).
 * NVFP4MOE_W4A8 keeps the 4-bit codes and stores E8M0 scales per 32 (the MMA's
 * scale type), and is SYNCHRONOUS in the same way: a row whose
 * 32-code blocks do not each have one power-of-two scale (or zero scale over
 * zero codes) makes it return NVFP4MOE_ERR_NOT_REPRESENTABLE.               */
nvfp4moe_status moe_pack_weights(nvfp4moe_mode mode, const nvfp4moe_expert_weights* weights_host_struct,
                                 void* packed, void* stream);

/* Scratch bytes moe_forward needs for these sizes. */
size_t moe_forward_workspace_size(nvfp4moe_mode mode, int32_t T, int32_t H, int32_t I, int32_t E, int32_t top_k);

/* The whole layer: route -> permute -> (quantise) -> gate/up GEMM + SwiGLU
 * (+ requantise) -> down GEMM x routing weight -> weighted un-permute.
 * Operation: out[t] = sum over the token's k routed experts j of
 * g[t][j] * W_down,j (SiLU(W_gate,j x_t) * (W_up,j x_t)), the expert output and
 * gate inside the saliency criterion of "patrickbdevaney/MiMo-V2.6-Flash-REAP50",
 * "Pruning Method".  Mode NVFP4MOE_W4A4 quantises the activations to NVFP4 with
 * a unit global (the default deployment); NVFP4MOE_W4A16 keeps them BF16 with
 * the same FP4 weights ("AxionML / MiMo-V2.6-Flash-MOPD-NVFP4", "Usage",
 * BF16-activation mode).
 *   x [T, H] BF16 bit patterns; router_logits [T, E] f32; bias [E] f32 or NULL;
 *   packed_weights from moe_pack_weights(mode, ...); out [T, H] BF16 bit
 *   patterns (out_is_fp32 == 0) or f32 (out_is_fp32 != 0).
 *   topk_ids_out [T, top_k] i32 and topk_weights_out [T, top_k] f32 are
 *   optional (NULL = not returned).
 * Constraints: as moe_route and moe_pack_weights; T >= 0 (0: no-op);
 * act_global finite and > 0; workspace_bytes >= moe_forward_workspace_size();
 * the permuted rows (T * top_k, plus up to 127 padding rows per expert in the
 * tensor-core modes) fit int32 indices, else NVFP4MOE_ERR_UNSUPPORTED_SHAPE.
 * Device-side waits are bounded; a wait that gives up makes the call's next
 * synchronous status check return NVFP4MOE_ERR_TIMEOUT (see
 * nvfp4moe_check_device_status).                                              */
nvfp4moe_status moe_forward(nvfp4moe_mode mode, const uint16_t* x, const float* router_logits, const float* bias,
                            const void* packed_weights, float act_global, int32_t T, int32_t H, int32_t I, int32_t E,
                            int32_t n_group, int32_t topk_group, int32_t top_k, float routed_scaling_factor,
                            int32_t renormalize, void* workspace, size_t workspace_bytes, void* out,
                            int32_t out_is_fp32, int32_t* topk_ids_out, float* topk_weights_out, void* stream);

/* Same layer from precomputed routing (topk_ids [T, top_k] i32, topk_weights
 * [T, top_k] f32, device): runs permute .. combine only.  No counterpart on the
 * pages: it lets the GEMM steps be driven without the router.  Arguments,
 * constraints and errors as moe_forward's.  A token's ids must lie in [0, E)
 * and be distinct; the ids are device data, so this is checked on the device:
 * a token that breaks the rule is computed with zero weights (its output row is
 * 0) and the next nvfp4moe_check_device_status returns NVFP4MOE_ERR_INVALID_ARG. */
nvfp4moe_status moe_forward_routed(nvfp4moe_mode mode, const uint16_t* x, const int32_t* topk_ids,
                                   const float* topk_weights, const void* packed_weights, float act_global, int32_t T,
                                   int32_t H, int32_t I, int32_t E, int32_t top_k, void* workspace,
                                   size_t workspace_bytes, void* out, int32_t out_is_fp32, void* stream);

/* moe_forward with one activation global scale per GEMM input
 * ("AxionML / MiMo-V2.6-Flash-MOPD-NVFP4", "Why a unit activation scale": a
 * calibrated scale per layer, optionally with the down-projection input's
 * amax capped, is the alternative to the shipped unit scale).
 *   act_global_in:  global of the layer input's NVFP4 codes (W4A4): the input is
 *                   quantised as x / act_global_in per 16-element block and the
 *                   gate/up products are scaled back by it.
 *   act_global_mid: global of the SwiGLU output's NVFP4 codes, the
 *                   down-projection input (W4A4).
 * Both finite and > 0 (also in W4A16 mode, where they are not used: that mode
 * keeps its activations in BF16).  moe_forward(..., g, ...) is
 * moe_forward_ex(..., g, g, ...).  A unit global covers magnitudes up to
 * 6 * 448 = 2688 (largest E2M1 code times largest E4M3 block scale); a
 * calibrated global is amax / 2688 of the tensor it quantises.              */
nvfp4moe_status moe_forward_ex(nvfp4moe_mode mode, const uint16_t* x, const float* router_logits, const float* bias,
                               const void* packed_weights, float act_global_in, float act_global_mid, int32_t T,
                               int32_t H, int32_t I, int32_t E, int32_t n_group, int32_t topk_group, int32_t top_k,
                               float routed_scaling_factor, int32_t renormalize, void* workspace,
                               size_t workspace_bytes, void* out, int32_t out_is_fp32, int32_t* topk_ids_out,
                               float* topk_weights_out, void* stream);

/* The down projection's input of the last moe_forward, moe_forward_ex or
 * moe_forward_routed call made with `workspace` (same mode, T, H, I, E and
 * top_k; nothing may have used the workspace since): for each listed pair
 * p = t * top_k + j (pairs: device int32 [n_pairs]) the row of the requantised
 * SwiGLU output, in the checkpoint layout.  No counterpart on the pages: it lets
 * a caller (the parity checks) hold the gate/up half and the down half of the
 * layer separately.
 *   W4A4:   codes_out [n_pairs, I/2] NVFP4 (even element in the low nibble),
 *           scales_out [n_pairs, I/16] E4M3;
 *   W4A8:   codes_out [n_pairs, I] E4M3, scales_out [n_pairs, I/32] E8M0;
 *   W4A16, W4A16C: codes_out [n_pairs, 2 I] (BF16 bit patterns), scales_out
 *           unused (may be NULL).
 * A pair index outside [0, T * top_k) leaves its output row untouched.
 * Asynchronous on `stream`. */
nvfp4moe_status moe_forward_intermediate(nvfp4moe_mode mode, int32_t T, int32_t H, int32_t I, int32_t E,
                                         int32_t top_k, const void* workspace, size_t workspace_bytes,
                                         const int32_t* pairs, int32_t n_pairs, uint8_t* codes_out,
                                         uint8_t* scales_out, void* stream);

/* Stage tracing.  When `events` is non-NULL, every later moe_forward /
 * moe_forward_routed call on this host thread records the cudaEvent_t handles
 * events[0..6] on its stream at its stage boundaries: [0] start, [1] after
 * routing, [2] after the permutation, [3] after the activation quantisation
 * (W4A4; same point as [2] for W4A16), [4] after the gate/up GEMM, [5] after
 * the down GEMM, [6] after the combine.  The events are owned by the caller and
 * must have been created with timing enabled; the library never synchronises on
 * them.  n_events must be 0 (tracing off, events ignored) or >= 7.           */
nvfp4moe_status nvfp4moe_set_trace_events(void* const* events, int32_t n_events);

/* SYNCHRONOUS: waits for `stream`, then reads and clears the device error word
 * that bounded waits inside the GEMM kernels set when they give up, and that
 * moe_forward_routed sets for routing ids outside [0, E) or repeated within a
 * token.  Returns NVFP4MOE_OK, NVFP4MOE_ERR_TIMEOUT (a wait gave up; reported
 * first) or NVFP4MOE_ERR_INVALID_ARG (bad precomputed routing). */
nvfp4moe_status nvfp4moe_check_device_status(void* stream);

/* Test hooks for the error paths; both inject on the host's side and neither
 * can fault the GPU.
 * nvfp4moe_raise_device_error ORs `bits` (1 = timeout, 2 = bad routing; a
 * non-empty subset, else NVFP4MOE_ERR_INVALID_ARG) into the device error word,
 * ordered on `stream`.  While the timeout bit is set, every bounded wait of the
 * GEMM kernels that is not satisfied within a few hundred polls gives up as if
 * another thread had timed out: the kernels take their error paths (copies and
 * MMAs already issued are drained before the CTA leaves), their outputs are
 * undefined, and the next nvfp4moe_check_device_status reports
 * NVFP4MOE_ERR_TIMEOUT and clears the word.
 * nvfp4moe_selftest_wait_timeout launches one thread that waits, bounded by
 * about `limit_cycles` SM clocks (0 .. 4e9), for a barrier nothing arrives on;
 * when the bound runs out it sets the timeout bit.  Both asynchronous on
 * `stream`; the context stays usable afterwards. */
nvfp4moe_status nvfp4moe_raise_device_error(int32_t bits, void* stream);
nvfp4moe_status nvfp4moe_selftest_wait_timeout(int64_t limit_cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4MOE_H_ */
