// transcode.cu -- exact MXFP4 -> NVFP4 scale transcode on sm_100a.
//
// "AxionML / MiMo-V2.6-Flash-MOPD-NVFP4" (introduction, "Reproduce the
// checkpoint") and "ProCreations/MiMo-V2.6-Flash-RL-NVFP4" ("What changed"):
// codes are kept byte for byte; each E8M0 scale 2^k over 32 codes becomes two
// E4M3 scales 2^(k-g) over the 16-code halves with one power-of-two global 2^g
// per tensor; nothing is re-rounded.  g = k_max - 8 over the non-zero blocks.
//
// Design: one 8-CTA thread-block cluster per tensor.  Each CTA streams its
// slice of the tensor once (coalesced 16-byte code loads, one E8M0 byte per
// block), copies the codes when the output is a separate buffer, keeps one byte
// per block in shared memory (the E8M0 byte, or 0xFF for an all-zero block) and
// reduces k_min / k_max / zero count / NaN flag.  The eight partial results are
// combined through distributed shared memory, then every CTA writes its scale
// pairs from shared memory.  HBM traffic is therefore the minimum: codes read
// once (and written once out of place), E8M0 read once, E4M3 written once.
#include <cooperative_groups.h>

#include "common.cuh"
#include "formats.cuh"

namespace cg = cooperative_groups;

namespace nvfp4moe {

constexpr int TC_CLUSTER = 8;
constexpr int TC_THREADS = 512;
constexpr int TC_UNROLL = 4;
constexpr int64_t TC_MAX_CACHE = 192 * 1024;  // bytes of shared memory per CTA for the block cache

struct TranscodeReportDev {
    unsigned long long blocks, zero_blocks, nonrep_tensors, nan_tensors;
};

template <bool CACHE>
__global__ void __cluster_dims__(TC_CLUSTER, 1, 1) __launch_bounds__(TC_THREADS)
    k_transcode(const uint4* __restrict__ codes_in, const uint8_t* __restrict__ e8m0, int64_t blocks, int64_t chunk,
                uint4* __restrict__ codes_out, uint16_t* __restrict__ e4m3_out, float* __restrict__ global_out,
                int32_t* __restrict__ status_out, TranscodeReportDev* __restrict__ report) {
    extern __shared__ uint8_t s_cache[];
    __shared__ int s_red[TC_THREADS / 32][4];
    __shared__ int s_part[4];  // k_min, k_max (biased E8M0 values), zero blocks, NaN seen

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int64_t tensor = blockIdx.x / TC_CLUSTER;
    const int64_t b0 = rank * chunk;
    const int64_t b1 = min(b0 + chunk, blocks);
    const uint4* cin = codes_in + tensor * blocks;
    const uint8_t* sin = e8m0 + tensor * blocks;
    uint4* cout = codes_out ? codes_out + tensor * blocks : nullptr;

    int kmin = 255, kmax = -1, zeros = 0, nan_seen = 0;
    for (int64_t base = b0 + threadIdx.x; base < b1; base += (int64_t)TC_THREADS * TC_UNROLL) {
        uint4 q[TC_UNROLL];
        uint32_t s[TC_UNROLL];
#pragma unroll
        for (int u = 0; u < TC_UNROLL; ++u) {
            const int64_t b = base + (int64_t)u * TC_THREADS;
            if (b < b1) {
                q[u] = __ldcs(cin + b);
                s[u] = __ldcs(sin + b);
            }
        }
#pragma unroll
        for (int u = 0; u < TC_UNROLL; ++u) {
            const int64_t b = base + (int64_t)u * TC_THREADS;
            if (b < b1) {
                if (cout) __stcs(cout + b, q[u]);
                const bool zero = ((q[u].x | q[u].y | q[u].z | q[u].w) & 0x77777777u) == 0;
                if (zero) {
                    ++zeros;
                } else if (s[u] == 0xFFu) {
                    nan_seen = 1;
                } else {
                    kmin = min(kmin, (int)s[u]);
                    kmax = max(kmax, (int)s[u]);
                }
                if (CACHE) s_cache[b - b0] = zero ? (uint8_t)0xFF : (uint8_t)s[u];
            }
        }
    }
    // block reduction
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
        zeros += __shfl_xor_sync(0xffffffffu, zeros, o);
        nan_seen |= __shfl_xor_sync(0xffffffffu, nan_seen, o);
    }
    if (lane_id() == 0) {
        s_red[warp_id()][0] = kmin;
        s_red[warp_id()][1] = kmax;
        s_red[warp_id()][2] = zeros;
        s_red[warp_id()][3] = nan_seen;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < TC_THREADS / 32; ++w) {
            kmin = min(kmin, s_red[w][0]);
            kmax = max(kmax, s_red[w][1]);
            zeros += s_red[w][2];
            nan_seen |= s_red[w][3];
        }
        s_part[0] = kmin;
        s_part[1] = kmax;
        s_part[2] = zeros;
        s_part[3] = nan_seen;
    }
    cluster.sync();  // partials of all eight CTAs are visible
    __shared__ int s_tensor[3];  // status, kmax, zero blocks of the whole tensor
    if (threadIdx.x == 0) {
        int tkmin = 255, tkmax = -1, tzeros = 0, tnan = 0;
        for (int r = 0; r < TC_CLUSTER; ++r) {
            const int* p = cluster.map_shared_rank(s_part, r);
            tkmin = min(tkmin, p[0]);
            tkmax = max(tkmax, p[1]);
            tzeros += p[2];
            tnan |= p[3];
        }
        int status = NVFP4MOE_TENSOR_EXACT;
        if (tnan)
            status = NVFP4MOE_TENSOR_NAN_SCALE;
        else if (tkmax >= 0 && tkmax - tkmin > 17)
            status = NVFP4MOE_TENSOR_NOT_REPRESENTABLE;
        s_tensor[0] = status;
        s_tensor[1] = tkmax;
        s_tensor[2] = tzeros;
        if (rank == 0) {
            float glob = 0.0f;
            if (status == NVFP4MOE_TENSOR_EXACT) {
                const int g = tkmax >= 0 ? (tkmax - 127) - 8 : 0;  // in [-135, 119]
                glob = g >= -126 ? __uint_as_float((uint32_t)(g + 127) << 23) : __uint_as_float(1u << (g + 149));
            }
            global_out[tensor] = glob;
            status_out[tensor] = status;
            atomicAdd(&report->blocks, (unsigned long long)blocks);
            atomicAdd(&report->zero_blocks, (unsigned long long)tzeros);
            if (status == NVFP4MOE_TENSOR_NOT_REPRESENTABLE) atomicAdd(&report->nonrep_tensors, 1ull);
            if (status == NVFP4MOE_TENSOR_NAN_SCALE) atomicAdd(&report->nan_tensors, 1ull);
        }
    }
    cluster.sync();  // nobody leaves while a peer may still read its partial
    const int status = s_tensor[0];
    const int tkmax = s_tensor[1];
    uint16_t* sout = e4m3_out + tensor * blocks;
    for (int64_t b = b0 + threadIdx.x; b < b1; b += TC_THREADS) {
        uint32_t v;
        if (CACHE) {
            v = s_cache[b - b0];
        } else {
            const uint4 q = __ldcs(cin + b);
            v = (((q.x | q.y | q.z | q.w) & 0x77777777u) == 0) ? 0xFFu : (uint32_t)__ldcs(sin + b);
        }
        uint32_t byte = 0;
        if (status == NVFP4MOE_TENSOR_EXACT && v != 0xFFu) byte = e4m3_pow2_byte((int)v - tkmax + 8);
        __stcs(sout + b, (uint16_t)(byte | (byte << 8)));
    }
}

size_t transcode_ws_size(int64_t) { return sizeof(TranscodeReportDev); }

nvfp4moe_status launch_transcode(const uint8_t* codes_in, const uint8_t* e8m0_in, int64_t num_tensors, int64_t N,
                                 int64_t K, uint8_t* codes_out, uint8_t* e4m3_out, float* global_out,
                                 int32_t* status_out, void* workspace, cudaStream_t stream) {
    TranscodeReportDev* rep = static_cast<TranscodeReportDev*>(workspace);
    NVFP4MOE_CUDA(cudaMemsetAsync(rep, 0, sizeof(TranscodeReportDev), stream));
    if (num_tensors == 0) return NVFP4MOE_OK;
    const int64_t blocks = N * K / 32;
    const int64_t chunk = ceil_div(blocks, TC_CLUSTER);
    uint4* cout = (codes_out == codes_in) ? nullptr : reinterpret_cast<uint4*>(codes_out);
    const dim3 grid((unsigned)(num_tensors * TC_CLUSTER));
    if (chunk <= TC_MAX_CACHE) {
        NVFP4MOE_CUDA(cudaFuncSetAttribute(k_transcode<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)TC_MAX_CACHE));
        k_transcode<true><<<grid, TC_THREADS, (size_t)chunk, stream>>>(
            reinterpret_cast<const uint4*>(codes_in), e8m0_in, blocks, chunk, cout,
            reinterpret_cast<uint16_t*>(e4m3_out), global_out, status_out, rep);
    } else {
        k_transcode<false><<<grid, TC_THREADS, 0, stream>>>(reinterpret_cast<const uint4*>(codes_in), e8m0_in,
                                                            blocks, chunk, cout, reinterpret_cast<uint16_t*>(e4m3_out),
                                                            global_out, status_out, rep);
    }
    NVFP4MOE_CHECK_LAUNCH("transcode kernel");
    return NVFP4MOE_OK;
}

nvfp4moe_status read_transcode_report(const void* workspace, nvfp4moe_transcode_report* out, cudaStream_t stream) {
    TranscodeReportDev h;
    NVFP4MOE_CUDA(cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, stream));
    NVFP4MOE_CUDA(cudaStreamSynchronize(stream));
    out->blocks = (int64_t)h.blocks;
    out->zero_blocks = (int64_t)h.zero_blocks;
    out->nonrepresentable_tensors = (int64_t)h.nonrep_tensors;
    out->nan_scale_tensors = (int64_t)h.nan_tensors;
    if (h.nan_tensors) return NVFP4MOE_ERR_NAN_SCALE;
    if (h.nonrep_tensors) return NVFP4MOE_ERR_NOT_REPRESENTABLE;
    return NVFP4MOE_OK;
}

}  // namespace nvfp4moe
