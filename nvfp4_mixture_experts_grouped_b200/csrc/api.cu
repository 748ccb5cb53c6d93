// api.cu -- the C ABI: argument validation, workspace carving and launches.
// Every entry point validates on the host before enqueueing anything.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "moe_internal.cuh"
#include "tc_ptx.cuh"

namespace nvfp4moe {

static thread_local char g_err[512] = "no error";
static thread_local cudaEvent_t g_trace[7] = {};
static thread_local bool g_trace_on = false;

static void trace(int i, cudaStream_t st) {
    if (g_trace_on) cudaEventRecord(g_trace[i], st);
}

void set_error(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
}

__device__ int32_t g_device_error = 0;

unsigned long long current_context_id() {
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}


// The word's device address, cached per device with the id of the context it
// belongs to: a new context on the device (after cudaDeviceReset, for instance)
// holds the word at a new address and makes the next call look it up again.
int32_t* device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    static int32_t* cache[64] = {};
    static unsigned long long cache_ctx[64] = {};
    static std::mutex mu;
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lk(mu);
    if (!cache[dev] || ctx == 0 || cache_ctx[dev] != ctx) {
        void* p = nullptr;
        cache[dev] = cudaGetSymbolAddress(&p, g_device_error) == cudaSuccess ? static_cast<int32_t*>(p) : nullptr;
        cache_ctx[dev] = current_context_id();
    }
    return cache[dev];
}

int num_sms() {
    int dev = 0;
    cudaGetDevice(&dev);
    static int cache[64] = {};
    if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev];
    int n = 148;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (dev >= 0 && dev < 64) cache[dev] = n;
    return n;
}

static nvfp4moe_status fail(nvfp4moe_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

static nvfp4moe_status check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(NVFP4MOE_ERR_CUDA, "no CUDA device");
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
        return fail(NVFP4MOE_ERR_UNSUPPORTED_DEVICE, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                    major, minor);
    return NVFP4MOE_OK;
}

#define REQUIRE(cond, status, ...)                          \
    do {                                                    \
        if (!(cond)) return fail(status, __VA_ARGS__);      \
    } while (0)

#define RETURN_IF(expr)                                     \
    do {                                                    \
        nvfp4moe_status _s = (expr);                        \
        if (_s != NVFP4MOE_OK) return _s;                   \
    } while (0)

// ---------------------------------------------------------------------------
// workspace of moe_forward
// ---------------------------------------------------------------------------
// Permuted rows (pairs plus their padding) are addressed by int32 indices in
// the routing plan (row_of_pair, pair_of_row): more than INT32_MAX of them is
// refused up front (no device could hold their workspace anyway).
static nvfp4moe_status check_row_count(int64_t rows) {
    REQUIRE(rows <= INT32_MAX, NVFP4MOE_ERR_UNSUPPORTED_SHAPE,
            "%lld permuted rows (T * top_k with padding) exceed the int32 row indices", (long long)rows);
    return NVFP4MOE_OK;
}

struct ForwardLayout {
    int64_t P, rows_max, n_chunks, max_tiles;
    int pad;
    // byte offsets
    int64_t ids, wts, chunk_counts, counts, offsets, pad_offsets, row_of_pair, pair_of_row, tiles, n_tiles, active,
        n_active;
    int64_t a1c, a1s, a2c, a2s, a2bf, y, ys, w16s;
    int64_t total;
};

static int64_t al(int64_t v) { return (v + 255) / 256 * 256; }

static ForwardLayout forward_layout(nvfp4moe_mode mode, int64_t T, int64_t H, int64_t I, int64_t E, int64_t k) {
    ForwardLayout L{};
    L.P = T * k;
    const bool tc = mode == NVFP4MOE_W4A4 || mode == NVFP4MOE_W4A8;  // tcgen05 GEMMs, rows padded to 128
    L.pad = tc ? MTILE : 1;
    const int64_t occupied = std::min<int64_t>(E, L.P);
    L.rows_max = tc ? round_up(L.P + occupied * (MTILE - 1), MTILE) : std::max<int64_t>(L.P, 1);
    L.n_chunks = std::max<int64_t>(ceil_div(T, PERM_CHUNK), 1);
    L.max_tiles = ceil_div(L.P, MTILE) + occupied + 1;
    int64_t o = 0;
    auto take = [&](int64_t bytes) {
        const int64_t at = o;
        o = al(o + std::max<int64_t>(bytes, 1));
        return at;
    };
    L.ids = take(L.P * 4);
    L.wts = take(L.P * 4);
    L.chunk_counts = take(L.n_chunks * E * 4);
    L.counts = take(E * 4);
    L.offsets = take((E + 1) * 4);
    L.pad_offsets = take((E + 1) * 4);
    L.row_of_pair = take(L.P * 4);
    L.pair_of_row = take(L.rows_max * 4);
    L.tiles = take(L.max_tiles * 16);
    L.n_tiles = take(4);
    L.active = take(E * 4);
    L.n_active = take(4);
    if (mode == NVFP4MOE_W4A8) {
        // E4M3 elements + E8M0 per 32 (atom layout); FP32 staged rows
        L.a1c = take(L.rows_max * H);
        L.a1s = take(L.rows_max * H / 32);
        L.a2c = take(L.rows_max * I);
        L.a2s = take(L.rows_max * I / 32);
        L.a2bf = -1;
        L.y = take(L.rows_max * H * 4);
        L.ys = -1;
    } else if (mode == NVFP4MOE_W4A4) {
        // NVFP4 codes + E4M3 per 16 (atom layout); FP16 staged rows + their
        // power-of-two scales per 64 columns
        L.a1c = take(L.rows_max * H / 2);
        L.a1s = take(L.rows_max * H / 16);
        L.a2c = take(L.rows_max * I / 2);
        L.a2s = take(L.rows_max * I / 16);
        L.a2bf = -1;
        L.y = take(L.rows_max * H * 2);
        L.ys = take(L.rows_max * (H / 64) * 4);
    } else {
        L.a1c = L.a1s = L.a2c = L.a2s = L.ys = -1;
        L.a2bf = take(L.rows_max * I * 2);
        L.y = take(L.rows_max * H * 4);  // FP32 staged rows
        L.w16s = take((int64_t)w4a16_scratch_size((int)T, (int)H, (int)I, (int)k));
    }
    L.total = o;
    return L;
}

static RoutingPlan carve_plan(const ForwardLayout& L, uint8_t* ws) {
    RoutingPlan p;
    p.ids = reinterpret_cast<int32_t*>(ws + L.ids);
    p.wts = reinterpret_cast<float*>(ws + L.wts);
    p.chunk_counts = reinterpret_cast<int32_t*>(ws + L.chunk_counts);
    p.counts = reinterpret_cast<int32_t*>(ws + L.counts);
    p.offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
    p.pad_offsets = reinterpret_cast<int32_t*>(ws + L.pad_offsets);
    p.row_of_pair = reinterpret_cast<int32_t*>(ws + L.row_of_pair);
    p.pair_of_row = reinterpret_cast<int32_t*>(ws + L.pair_of_row);
    p.tiles = reinterpret_cast<int4*>(ws + L.tiles);
    p.n_tiles = reinterpret_cast<int32_t*>(ws + L.n_tiles);
    p.active = reinterpret_cast<int32_t*>(ws + L.active);
    p.n_active = reinterpret_cast<int32_t*>(ws + L.n_active);
    return p;
}

static nvfp4moe_status validate_routing(int32_t E, int32_t n_group, int32_t topk_group, int32_t top_k) {
    REQUIRE(E >= 1 && E <= 1024, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "E=%d outside [1, 1024]", E);
    REQUIRE(n_group >= 1 && n_group <= 32, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "n_group=%d outside [1, 32]", n_group);
    REQUIRE(E % n_group == 0, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "E=%d is not a multiple of n_group=%d", E, n_group);
    REQUIRE(topk_group >= 1 && topk_group <= n_group, NVFP4MOE_ERR_UNSUPPORTED_SHAPE,
            "topk_group=%d outside [1, n_group=%d]", topk_group, n_group);
    const int avail = topk_group * (E / n_group);
    REQUIRE(top_k >= 1 && top_k <= 32 && top_k <= avail, NVFP4MOE_ERR_UNSUPPORTED_SHAPE,
            "top_k=%d outside [1, min(32, %d)]", top_k, avail);
    return NVFP4MOE_OK;
}

static nvfp4moe_status validate_layer_shape(int32_t H, int32_t I, int32_t E) {
    REQUIRE(E >= 1 && E <= 1024, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "E=%d outside [1, 1024]", E);
    REQUIRE(H >= 256 && H % 256 == 0, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "H=%d must be a positive multiple of 256", H);
    REQUIRE(I >= 128 && I % 128 == 0, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "I=%d must be a positive multiple of 128", I);
    return NVFP4MOE_OK;
}

}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" {

const char* nvfp4moe_last_error_string(void) { return g_err; }

int32_t nvfp4moe_version(void) { return (1 << 16) | 0; }

size_t nvfp4moe_transcode_workspace_size(int64_t num_tensors) { return transcode_ws_size(num_tensors); }

nvfp4moe_status transcode_mxfp4_to_nvfp4(const uint8_t* codes_in, const uint8_t* e8m0_in, int64_t num_tensors,
                                         int64_t N, int64_t K, uint8_t* codes_out, uint8_t* e4m3_out,
                                         float* global_scale_out, int32_t* tensor_status_out, void* workspace,
                                         size_t workspace_bytes, nvfp4moe_transcode_report* report_host,
                                         void* stream) {
    REQUIRE(num_tensors >= 0 && N >= 1 && K >= 32, NVFP4MOE_ERR_INVALID_ARG,
            "bad sizes num_tensors=%lld N=%lld K=%lld", (long long)num_tensors, (long long)N, (long long)K);
    REQUIRE(K % 32 == 0, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "K=%lld is not a multiple of 32", (long long)K);
    REQUIRE(workspace && workspace_bytes >= transcode_ws_size(num_tensors), NVFP4MOE_ERR_WORKSPACE_TOO_SMALL,
            "transcode workspace of %zu bytes is below the required %zu", workspace_bytes,
            transcode_ws_size(num_tensors));
    REQUIRE(aligned16(workspace), NVFP4MOE_ERR_ALIGNMENT, "workspace is not 16-byte aligned");
    if (num_tensors > 0) {
        REQUIRE(codes_in && e8m0_in && codes_out && e4m3_out && global_scale_out && tensor_status_out,
                NVFP4MOE_ERR_INVALID_ARG, "null tensor pointer");
        REQUIRE(aligned16(codes_in) && aligned16(e8m0_in) && aligned16(codes_out) && aligned16(e4m3_out) &&
                    aligned16(global_scale_out) && aligned16(tensor_status_out),
                NVFP4MOE_ERR_ALIGNMENT, "a tensor pointer is not 16-byte aligned");
        const int64_t bytes = num_tensors * N * K / 2;
        const uint8_t *a0 = codes_in, *a1 = codes_in + bytes, *b0 = codes_out, *b1 = codes_out + bytes;
        REQUIRE(codes_in == codes_out || a1 <= b0 || b1 <= a0, NVFP4MOE_ERR_INVALID_ARG,
                "codes_out overlaps codes_in without being equal to it");
    }
    RETURN_IF(check_device());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    RETURN_IF(launch_transcode(codes_in, e8m0_in, num_tensors, N, K, codes_out, e4m3_out, global_scale_out,
                               tensor_status_out, workspace, st));
    if (report_host) return read_transcode_report(workspace, report_host, st);
    return NVFP4MOE_OK;
}

nvfp4moe_status nvfp4_compact_scales(const uint8_t* codes, const uint8_t* e4m3_sf, int64_t rows, int64_t K,
                                     uint8_t* nib_out, int8_t* row_exp_out, int32_t* row_status_out,
                                     int32_t* n_bad_out, void* stream) {
    REQUIRE(rows >= 0 && K >= 64, NVFP4MOE_ERR_INVALID_ARG, "bad sizes rows=%lld K=%lld", (long long)rows,
            (long long)K);
    REQUIRE(K % 64 == 0, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "K=%lld is not a multiple of 64", (long long)K);
    if (rows == 0) return NVFP4MOE_OK;
    REQUIRE(codes && e4m3_sf && nib_out && row_exp_out && row_status_out, NVFP4MOE_ERR_INVALID_ARG,
            "null tensor pointer");
    const void* al16[] = {codes, e4m3_sf, nib_out, row_exp_out, row_status_out, n_bad_out};
    for (const void* q : al16) REQUIRE(!q || aligned16(q), NVFP4MOE_ERR_ALIGNMENT, "a pointer is not 16-byte aligned");
    RETURN_IF(check_device());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (n_bad_out) NVFP4MOE_CUDA(cudaMemsetAsync(n_bad_out, 0, sizeof(int32_t), st));
    return launch_compact_rows(codes, e4m3_sf, rows, K, row_exp_out, nib_out, row_status_out, n_bad_out, st);
}

nvfp4moe_status moe_route(const float* logits, const float* bias, int32_t T, int32_t E, int32_t n_group,
                          int32_t topk_group, int32_t top_k, float routed_scaling_factor, int32_t renormalize,
                          int32_t* topk_ids, float* topk_weights, void* stream) {
    REQUIRE(T >= 0, NVFP4MOE_ERR_INVALID_ARG, "T=%d is negative", T);
    RETURN_IF(validate_routing(E, n_group, topk_group, top_k));
    REQUIRE(std::isfinite(routed_scaling_factor), NVFP4MOE_ERR_INVALID_ARG, "routed_scaling_factor is not finite");
    if (T == 0) return NVFP4MOE_OK;
    REQUIRE(logits && topk_ids && topk_weights, NVFP4MOE_ERR_INVALID_ARG, "null tensor pointer");
    REQUIRE(aligned16(logits) && aligned16(topk_ids) && aligned16(topk_weights) && (!bias || aligned16(bias)),
            NVFP4MOE_ERR_ALIGNMENT, "a tensor pointer is not 16-byte aligned");
    RETURN_IF(check_device());
    return launch_route(logits, bias, T, E, n_group, topk_group, top_k, routed_scaling_factor, renormalize, topk_ids,
                        topk_weights, static_cast<cudaStream_t>(stream));
}

size_t moe_router_topk_workspace_size(int32_t T) { return T > 0 ? router_ws_size(T) : 0; }

nvfp4moe_status moe_router_topk(const uint16_t* x_bf16, const float* w_router, const float* bias, int32_t T,
                                int32_t H, int32_t E, int32_t n_group, int32_t topk_group, int32_t top_k,
                                float routed_scaling_factor, int32_t renormalize, float* logits_out,
                                int32_t* topk_ids, float* topk_weights, void* workspace, size_t workspace_bytes,
                                void* stream) {
    REQUIRE(T >= 0 && T <= ROUTER_MAX_T, NVFP4MOE_ERR_INVALID_ARG, "T=%d is outside [0, %lld]", T,
            (long long)ROUTER_MAX_T);
    RETURN_IF(validate_routing(E, n_group, topk_group, top_k));
    REQUIRE(E % 4 == 0, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "E=%d is not a multiple of 4", E);
    REQUIRE(H >= 256 && H % 256 == 0, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "H=%d must be a positive multiple of 256", H);
    REQUIRE(std::isfinite(routed_scaling_factor), NVFP4MOE_ERR_INVALID_ARG, "routed_scaling_factor is not finite");
    if (T == 0) return NVFP4MOE_OK;
    REQUIRE(x_bf16 && w_router && logits_out && topk_ids && topk_weights && workspace, NVFP4MOE_ERR_INVALID_ARG,
            "null pointer");
    REQUIRE(workspace_bytes >= router_ws_size(T), NVFP4MOE_ERR_WORKSPACE_TOO_SMALL,
            "workspace of %zu bytes, %zu needed", workspace_bytes, router_ws_size(T));
    REQUIRE(aligned16(x_bf16) && aligned16(w_router) && aligned16(logits_out) && aligned16(topk_ids) &&
                aligned16(topk_weights) && aligned16(workspace) && (!bias || aligned16(bias)),
            NVFP4MOE_ERR_ALIGNMENT, "a pointer is not 16-byte aligned");
    RETURN_IF(check_device());
    return launch_router_topk(x_bf16, w_router, bias, T, H, E, n_group, topk_group, top_k, routed_scaling_factor,
                              renormalize, logits_out, topk_ids, topk_weights, workspace,
                              static_cast<cudaStream_t>(stream));
}

nvfp4moe_status quantize_nvfp4(const uint16_t* x_bf16, int64_t M, int64_t K, float gs, uint8_t* codes,
                               uint8_t* e4m3_scales, void* stream) {
    REQUIRE(M >= 0 && K >= 16, NVFP4MOE_ERR_INVALID_ARG, "bad sizes M=%lld K=%lld", (long long)M, (long long)K);
    REQUIRE(K % 16 == 0, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "K=%lld is not a multiple of 16", (long long)K);
    REQUIRE(std::isfinite(gs) && gs > 0.0f, NVFP4MOE_ERR_INVALID_ARG, "global scale must be finite and > 0");
    if (M == 0) return NVFP4MOE_OK;
    REQUIRE(x_bf16 && codes && e4m3_scales, NVFP4MOE_ERR_INVALID_ARG, "null tensor pointer");
    REQUIRE(aligned16(x_bf16) && aligned16(codes) && aligned16(e4m3_scales), NVFP4MOE_ERR_ALIGNMENT,
            "a tensor pointer is not 16-byte aligned");
    RETURN_IF(check_device());
    return launch_quantize_linear(x_bf16, M, K, gs, codes, e4m3_scales, static_cast<cudaStream_t>(stream));
}

nvfp4moe_status quantize_mxfp8(const uint16_t* x_bf16, int64_t M, int64_t K, uint8_t* codes, uint8_t* e8m0_scales,
                               void* stream) {
    REQUIRE(M >= 0 && K >= 32, NVFP4MOE_ERR_INVALID_ARG, "bad sizes M=%lld K=%lld", (long long)M, (long long)K);
    REQUIRE(K % 32 == 0, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "K=%lld is not a multiple of 32", (long long)K);
    if (M == 0) return NVFP4MOE_OK;
    REQUIRE(x_bf16 && codes && e8m0_scales, NVFP4MOE_ERR_INVALID_ARG, "null tensor pointer");
    REQUIRE(aligned16(x_bf16) && aligned16(codes) && aligned16(e8m0_scales), NVFP4MOE_ERR_ALIGNMENT,
            "a tensor pointer is not 16-byte aligned");
    RETURN_IF(check_device());
    return launch_quantize_mx8_linear(x_bf16, M, K, codes, e8m0_scales, static_cast<cudaStream_t>(stream));
}

size_t moe_permute_workspace_size(int32_t T, int32_t E, int32_t top_k, int32_t pad) {
    if (T < 0 || E < 1 || top_k < 1 || pad < 1) return 0;
    const int64_t P = (int64_t)T * top_k;
    const int64_t rows_max = P + std::min<int64_t>(E, P) * (pad - 1);
    const int64_t n_chunks = std::max<int64_t>(ceil_div(T, PERM_CHUNK), 1);
    const int64_t max_tiles = ceil_div(P, MTILE) + std::min<int64_t>(E, P) + 1;
    return (size_t)(al(n_chunks * E * 4) + al((E + 1) * 4) + al(std::max<int64_t>(rows_max, 1) * 4) +
                    al(max_tiles * 16) + al(4) + al(E * 4) + al(4));
}

nvfp4moe_status moe_permute(const int32_t* topk_ids, int32_t T, int32_t E, int32_t top_k, int32_t pad,
                            int32_t* counts_out, int32_t* pad_offsets_out, int32_t* row_of_pair_out, void* workspace,
                            size_t workspace_bytes, void* stream) {
    REQUIRE(T >= 0, NVFP4MOE_ERR_INVALID_ARG, "T=%d is negative", T);
    REQUIRE(E >= 1 && E <= 1024, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "E=%d outside [1, 1024]", E);
    REQUIRE(top_k >= 1 && top_k <= 32 && top_k <= E, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "top_k=%d outside [1, 32]", top_k);
    REQUIRE(pad == 1 || pad == MTILE, NVFP4MOE_ERR_INVALID_ARG, "pad=%d must be 1 or %d", pad, MTILE);
    RETURN_IF(check_row_count((int64_t)T * top_k + std::min<int64_t>(E, (int64_t)T * top_k) * (pad - 1)));
    REQUIRE(counts_out && pad_offsets_out && workspace, NVFP4MOE_ERR_INVALID_ARG, "null pointer");
    const size_t need = moe_permute_workspace_size(T, E, top_k, pad);
    REQUIRE(workspace_bytes >= need, NVFP4MOE_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes is below %zu",
            workspace_bytes, need);
    const void* al16[] = {topk_ids, counts_out, pad_offsets_out, row_of_pair_out, workspace};
    for (const void* q : al16) REQUIRE(!q || aligned16(q), NVFP4MOE_ERR_ALIGNMENT, "a pointer is not 16-byte aligned");
    RETURN_IF(check_device());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        NVFP4MOE_CUDA(cudaMemsetAsync(counts_out, 0, (size_t)E * 4, st));
        NVFP4MOE_CUDA(cudaMemsetAsync(pad_offsets_out, 0, (size_t)(E + 1) * 4, st));
        return NVFP4MOE_OK;
    }
    REQUIRE(topk_ids && row_of_pair_out, NVFP4MOE_ERR_INVALID_ARG, "null pointer");
    const int64_t P = (int64_t)T * top_k;
    const int64_t rows_max = P + std::min<int64_t>(E, P) * (pad - 1);
    const int64_t n_chunks = ceil_div(T, PERM_CHUNK);
    const int64_t max_tiles = ceil_div(P, MTILE) + std::min<int64_t>(E, P) + 1;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int64_t o = 0;
    auto take = [&](int64_t bytes) {
        uint8_t* at = ws + o;
        o += al(std::max<int64_t>(bytes, 1));
        return at;
    };
    RoutingPlan plan;
    plan.ids = const_cast<int32_t*>(topk_ids);
    plan.wts = nullptr;
    plan.chunk_counts = reinterpret_cast<int32_t*>(take(n_chunks * E * 4));
    plan.counts = counts_out;
    plan.offsets = reinterpret_cast<int32_t*>(take((E + 1) * 4));
    plan.pad_offsets = pad_offsets_out;
    plan.row_of_pair = row_of_pair_out;
    plan.pair_of_row = reinterpret_cast<int32_t*>(take(rows_max * 4));
    plan.tiles = reinterpret_cast<int4*>(take(max_tiles * 16));
    plan.n_tiles = reinterpret_cast<int32_t*>(take(4));
    plan.active = reinterpret_cast<int32_t*>(take(E * 4));
    plan.n_active = reinterpret_cast<int32_t*>(take(4));
    return launch_permute(topk_ids, T, top_k, E, pad, plan, st);
}

static bool valid_mode(nvfp4moe_mode mode) {
    return mode == NVFP4MOE_W4A16 || mode == NVFP4MOE_W4A4 || mode == NVFP4MOE_W4A16C || mode == NVFP4MOE_W4A8;
}

size_t moe_packed_weights_size(nvfp4moe_mode mode, int32_t E, int32_t H, int32_t I) {
    if (E < 1 || H < 1 || I < 1 || !valid_mode(mode)) return 0;
    if (mode == NVFP4MOE_W4A4 || mode == NVFP4MOE_W4A8) return w4a4_packed_size(E, H, I, mode == NVFP4MOE_W4A8);
    return w4a16_packed_size(E, H, I, mode == NVFP4MOE_W4A16C);
}

nvfp4moe_status moe_pack_weights(nvfp4moe_mode mode, const nvfp4moe_expert_weights* w, void* packed, void* stream) {
    REQUIRE(valid_mode(mode), NVFP4MOE_ERR_INVALID_ARG, "unknown mode %d", (int)mode);
    REQUIRE(w && packed, NVFP4MOE_ERR_INVALID_ARG, "null pointer");
    RETURN_IF(validate_layer_shape(w->H, w->I, w->E));
    const void* ptrs[7] = {w->gate_codes, w->gate_sf, w->up_codes, w->up_sf, w->down_codes, w->down_sf, w->w_global};
    for (const void* q : ptrs) {
        REQUIRE(q, NVFP4MOE_ERR_INVALID_ARG, "null weight pointer");
        REQUIRE(aligned16(q), NVFP4MOE_ERR_ALIGNMENT, "a weight pointer is not 16-byte aligned");
    }
    REQUIRE(aligned16(packed), NVFP4MOE_ERR_ALIGNMENT, "packed buffer is not 16-byte aligned");
    RETURN_IF(check_device());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (mode == NVFP4MOE_W4A4 || mode == NVFP4MOE_W4A8) return launch_w4a4_pack(*w, packed, mode == NVFP4MOE_W4A8, st);
    return launch_w4a16_pack(*w, packed, mode == NVFP4MOE_W4A16C, st);
}

size_t moe_forward_workspace_size(nvfp4moe_mode mode, int32_t T, int32_t H, int32_t I, int32_t E, int32_t top_k) {
    if (T < 0 || H < 1 || I < 1 || E < 1 || top_k < 1) return 0;
    return (size_t)forward_layout(mode, T, H, I, E, top_k).total;
}

static nvfp4moe_status forward_common(nvfp4moe_mode mode, const uint16_t* x, const float* logits, const float* bias,
                                      const int32_t* ids_in, const float* wts_in, const void* packed,
                                      float act_global, float act_global_mid, int32_t T, int32_t H, int32_t I,
                                      int32_t E, int32_t n_group,
                                      int32_t topk_group, int32_t top_k, float rsf, int32_t renorm, void* workspace,
                                      size_t workspace_bytes, void* out, int32_t out_is_fp32, int32_t* ids_out,
                                      float* wts_out, void* stream) {
    REQUIRE(valid_mode(mode), NVFP4MOE_ERR_INVALID_ARG, "unknown mode %d", (int)mode);
    REQUIRE(T >= 0, NVFP4MOE_ERR_INVALID_ARG, "T=%d is negative", T);
    RETURN_IF(validate_layer_shape(H, I, E));
    if (logits) {
        RETURN_IF(validate_routing(E, n_group, topk_group, top_k));
    } else {
        REQUIRE(top_k >= 1 && top_k <= 32 && top_k <= E, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "top_k=%d outside [1, %d]",
                top_k, std::min(32, (int)E));
    }
    REQUIRE(std::isfinite(act_global) && act_global > 0.0f, NVFP4MOE_ERR_INVALID_ARG,
            "act_global must be finite and > 0");
    REQUIRE(std::isfinite(act_global_mid) && act_global_mid > 0.0f, NVFP4MOE_ERR_INVALID_ARG,
            "act_global_mid must be finite and > 0");
    REQUIRE(std::isfinite(rsf), NVFP4MOE_ERR_INVALID_ARG, "routed_scaling_factor is not finite");
    if (T == 0) return NVFP4MOE_OK;
    REQUIRE(x && packed && workspace && out, NVFP4MOE_ERR_INVALID_ARG, "null pointer");
    REQUIRE(logits || (ids_in && wts_in), NVFP4MOE_ERR_INVALID_ARG, "no routing input");
    const void* al16[] = {x, packed, workspace, out, logits, bias, ids_in, wts_in, ids_out, wts_out};
    for (const void* q : al16) REQUIRE(!q || aligned16(q), NVFP4MOE_ERR_ALIGNMENT, "a pointer is not 16-byte aligned");
    const ForwardLayout L = forward_layout(mode, T, H, I, E, top_k);
    RETURN_IF(check_row_count(L.rows_max));
    REQUIRE(workspace_bytes >= (size_t)L.total, NVFP4MOE_ERR_WORKSPACE_TOO_SMALL,
            "workspace of %zu bytes is below the required %lld", workspace_bytes, (long long)L.total);
    RETURN_IF(check_device());

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    RoutingPlan plan = carve_plan(L, ws);
    trace(0, st);
    if (logits) {
        RETURN_IF(launch_route(logits, bias, T, E, n_group, topk_group, top_k, rsf, renorm, plan.ids, plan.wts, st));
    } else {
        RETURN_IF(launch_check_routing(ids_in, wts_in, T, top_k, E, plan.ids, plan.wts, st));
    }
    trace(1, st);
    if (mode == NVFP4MOE_W4A4 || mode == NVFP4MOE_W4A8)
        plan.tile_rows = w4a4_tile_rows(T, top_k, E);  // the GEMMs' tile form
    RETURN_IF(launch_permute(plan.ids, T, top_k, E, L.pad, plan, st));
    trace(2, st);
    void* Y = ws + L.y;
    const bool tc = mode == NVFP4MOE_W4A4 || mode == NVFP4MOE_W4A8;
    float* ys = mode == NVFP4MOE_W4A4 ? reinterpret_cast<float*>(ws + L.ys) : nullptr;  // else FP32 rows
    if (tc) {
        uint8_t* a1c = ws + L.a1c;
        uint8_t* a1s = ws + L.a1s;
        const bool mx8 = mode == NVFP4MOE_W4A8;
        if (mx8)
            RETURN_IF(launch_quantize_mx8_scatter(x, T, H, a1c, a1s, plan.row_of_pair, top_k, st));
        else
            RETURN_IF(launch_quantize_scatter(x, T, H, act_global, a1c, a1s, plan.row_of_pair, top_k, st));
        trace(3, st);
        RETURN_IF(launch_w4a4_layer(packed, mx8, T, H, I, E, top_k, act_global, act_global_mid, L.rows_max,
                                    (int)L.max_tiles, plan, a1c, a1s, ws + L.a2c, ws + L.a2s, static_cast<__half*>(Y),
                                    mx8 ? nullptr : ys, st, g_trace_on ? g_trace[4] : nullptr));
    } else {
        trace(3, st);
        RETURN_IF(launch_w4a16_layer(x, packed, mode == NVFP4MOE_W4A16C, T, H, I, E, top_k, plan, reinterpret_cast<uint16_t*>(ws + L.a2bf),
                                     static_cast<float*>(Y), ws + L.w16s, st, g_trace_on ? g_trace[4] : nullptr));
    }
    trace(5, st);
    RETURN_IF(launch_combine(Y, ys, plan.row_of_pair, T, H, top_k, out, out_is_fp32 != 0, st));
    trace(6, st);
    if (ids_out) NVFP4MOE_CUDA(cudaMemcpyAsync(ids_out, plan.ids, (size_t)L.P * 4, cudaMemcpyDeviceToDevice, st));
    if (wts_out) NVFP4MOE_CUDA(cudaMemcpyAsync(wts_out, plan.wts, (size_t)L.P * 4, cudaMemcpyDeviceToDevice, st));
    return NVFP4MOE_OK;
}

nvfp4moe_status moe_forward(nvfp4moe_mode mode, const uint16_t* x, const float* router_logits, const float* bias,
                            const void* packed_weights, float act_global, int32_t T, int32_t H, int32_t I, int32_t E,
                            int32_t n_group, int32_t topk_group, int32_t top_k, float routed_scaling_factor,
                            int32_t renormalize, void* workspace, size_t workspace_bytes, void* out,
                            int32_t out_is_fp32, int32_t* topk_ids_out, float* topk_weights_out, void* stream) {
    if (T > 0 && !router_logits) return fail(NVFP4MOE_ERR_INVALID_ARG, "router_logits is null");
    return forward_common(mode, x, router_logits, bias, nullptr, nullptr, packed_weights, act_global, act_global, T,
                          H, I, E, n_group, topk_group, top_k, routed_scaling_factor, renormalize, workspace,
                          workspace_bytes, out, out_is_fp32, topk_ids_out, topk_weights_out, stream);
}

nvfp4moe_status moe_forward_ex(nvfp4moe_mode mode, const uint16_t* x, const float* router_logits, const float* bias,
                               const void* packed_weights, float act_global_in, float act_global_mid, int32_t T,
                               int32_t H, int32_t I, int32_t E, int32_t n_group, int32_t topk_group, int32_t top_k,
                               float routed_scaling_factor, int32_t renormalize, void* workspace,
                               size_t workspace_bytes, void* out, int32_t out_is_fp32, int32_t* topk_ids_out,
                               float* topk_weights_out, void* stream) {
    if (T > 0 && !router_logits) return fail(NVFP4MOE_ERR_INVALID_ARG, "router_logits is null");
    return forward_common(mode, x, router_logits, bias, nullptr, nullptr, packed_weights, act_global_in,
                          act_global_mid, T, H, I, E, n_group, topk_group, top_k, routed_scaling_factor, renormalize,
                          workspace, workspace_bytes, out, out_is_fp32, topk_ids_out, topk_weights_out, stream);
}

nvfp4moe_status moe_forward_routed(nvfp4moe_mode mode, const uint16_t* x, const int32_t* topk_ids,
                                   const float* topk_weights, const void* packed_weights, float act_global, int32_t T,
                                   int32_t H, int32_t I, int32_t E, int32_t top_k, void* workspace,
                                   size_t workspace_bytes, void* out, int32_t out_is_fp32, void* stream) {
    if (T > 0 && (!topk_ids || !topk_weights)) return fail(NVFP4MOE_ERR_INVALID_ARG, "routing input is null");
    return forward_common(mode, x, nullptr, nullptr, topk_ids, topk_weights, packed_weights, act_global, act_global, T,
                          H, I, E, 1, 1, top_k, 1.0f, 0, workspace, workspace_bytes, out, out_is_fp32, nullptr, nullptr, stream);
}

nvfp4moe_status moe_forward_intermediate(nvfp4moe_mode mode, int32_t T, int32_t H, int32_t I, int32_t E,
                                         int32_t top_k, const void* workspace, size_t workspace_bytes,
                                         const int32_t* pairs, int32_t n_pairs, uint8_t* codes_out,
                                         uint8_t* scales_out, void* stream) {
    REQUIRE(valid_mode(mode), NVFP4MOE_ERR_INVALID_ARG, "unknown mode %d", (int)mode);
    REQUIRE(T >= 0 && n_pairs >= 0, NVFP4MOE_ERR_INVALID_ARG, "T=%d, n_pairs=%d", T, n_pairs);
    RETURN_IF(validate_layer_shape(H, I, E));
    REQUIRE(top_k >= 1 && top_k <= 32 && top_k <= E, NVFP4MOE_ERR_UNSUPPORTED_SHAPE, "top_k=%d outside [1, %d]", top_k,
            std::min(32, (int)E));
    if (T == 0 || n_pairs == 0) return NVFP4MOE_OK;
    const bool scaled = mode == NVFP4MOE_W4A4 || mode == NVFP4MOE_W4A8;
    REQUIRE(workspace && pairs && codes_out && (!scaled || scales_out), NVFP4MOE_ERR_INVALID_ARG, "null pointer");
    const ForwardLayout L = forward_layout(mode, T, H, I, E, top_k);
    REQUIRE(workspace_bytes >= (size_t)L.total, NVFP4MOE_ERR_WORKSPACE_TOO_SMALL,
            "workspace of %zu bytes is below the required %lld", workspace_bytes, (long long)L.total);
    RETURN_IF(check_device());
    const uint8_t* ws = static_cast<const uint8_t*>(workspace);
    const int32_t* rop = reinterpret_cast<const int32_t*>(ws + L.row_of_pair);
    const uint8_t* codes = ws + (scaled ? L.a2c : L.a2bf);
    const uint8_t* scales = scaled ? ws + L.a2s : nullptr;
    return launch_read_intermediate((int)mode, pairs, n_pairs, L.P, rop, codes, scales, I, codes_out, scales_out,
                                    static_cast<cudaStream_t>(stream));
}

nvfp4moe_status nvfp4moe_set_trace_events(void* const* events, int32_t n_events) {
    if (!events || n_events == 0) {
        g_trace_on = false;
        return NVFP4MOE_OK;
    }
    REQUIRE(n_events >= 7, NVFP4MOE_ERR_INVALID_ARG, "n_events=%d: tracing needs 7 events", n_events);
    for (int i = 0; i < 7; ++i) {
        REQUIRE(events[i], NVFP4MOE_ERR_INVALID_ARG, "trace event %d is null", i);
        g_trace[i] = static_cast<cudaEvent_t>(events[i]);
    }
    g_trace_on = true;
    return NVFP4MOE_OK;
}

// Test hooks for the error paths (host-side injection; nothing here faults).
namespace {
__global__ void k_raise_device_error(int32_t* w, int32_t bits) { atomicOr(w, bits); }
// One thread waits for a phase of a barrier that nothing arrives on; its bounded
// wait gives up after about limit_cycles and sets the timeout bit.
__global__ void k_wait_nothing(int32_t* err, long long limit_cycles) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        nvfp4moe::tc::mbar_init(&bar, 1);
        nvfp4moe::tc::fence_mbar_init();
        (void)nvfp4moe::tc::mbar_wait(&bar, 0u, err, limit_cycles);
    }
}
}  // namespace

nvfp4moe_status nvfp4moe_raise_device_error(int32_t bits, void* stream) {
    REQUIRE(bits > 0 && (bits & ~(DEV_ERR_TIMEOUT | DEV_ERR_BAD_ROUTING)) == 0, NVFP4MOE_ERR_INVALID_ARG,
            "bits=%d must be a non-empty subset of %d", bits, DEV_ERR_TIMEOUT | DEV_ERR_BAD_ROUTING);
    RETURN_IF(check_device());
    int32_t* w = device_error_word();
    if (!w) return fail(NVFP4MOE_ERR_CUDA, "device error word unavailable");
    k_raise_device_error<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(w, bits);
    NVFP4MOE_CHECK_LAUNCH("device error injection");
    return NVFP4MOE_OK;
}

nvfp4moe_status nvfp4moe_selftest_wait_timeout(int64_t limit_cycles, void* stream) {
    REQUIRE(limit_cycles >= 0 && limit_cycles <= 4000000000LL, NVFP4MOE_ERR_INVALID_ARG,
            "limit_cycles=%lld outside [0, 4e9]", (long long)limit_cycles);
    RETURN_IF(check_device());
    int32_t* w = device_error_word();
    if (!w) return fail(NVFP4MOE_ERR_CUDA, "device error word unavailable");
    k_wait_nothing<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(w, (long long)limit_cycles);
    NVFP4MOE_CHECK_LAUNCH("bounded-wait self-test");
    return NVFP4MOE_OK;
}

nvfp4moe_status nvfp4moe_check_device_status(void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    NVFP4MOE_CUDA(cudaStreamSynchronize(st));
    int32_t* w = device_error_word();
    if (!w) return fail(NVFP4MOE_ERR_CUDA, "device error word unavailable");
    int32_t v = 0;
    NVFP4MOE_CUDA(cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost));
    if (v != 0) {
        const int32_t zero = 0;
        NVFP4MOE_CUDA(cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice));
        if (v & DEV_ERR_TIMEOUT) return fail(NVFP4MOE_ERR_TIMEOUT, "a bounded device-side wait gave up");
        return fail(NVFP4MOE_ERR_INVALID_ARG,
                    "precomputed routing named an expert outside [0, E) or one expert twice for a token; "
                    "those tokens were computed with zero weights");
    }
    return NVFP4MOE_OK;
}

}  // extern "C"
