"""GPU parity of the W4A8 mode (MXFP8 activations x FP4 weights on the
block-scaled FP8 x FP4 tcgen05 MMA): the MXFP8 quantiser bit-exact against the
oracle, the layer against the float64 oracle's W4A8 layer (mode 3) within the
layer tolerance."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import nvfp4_mixture_experts_grouped_b200 as moe
import oracle
from nvfp4_mixture_experts_grouped_b200 import inputs

from helpers import (GpuLayer, bf16_tensor, check_layer_split, compare_layer, covering_tokens, dev, host,
                     nvfp4_weights_from_inputs, oracle_layer, out_to_f64)

pytestmark = pytest.mark.gpu


def gpu_mx8(x_bits: np.ndarray):
    M, K = x_bits.shape
    codes = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    scales = torch.empty((M, K // 32), dtype=torch.uint8, device="cuda")
    moe.quantize_mxfp8(bf16_tensor(x_bits), M, K, codes, scales)
    torch.cuda.synchronize()
    return host(codes), host(scales)


@pytest.mark.parametrize("M,K,scale", [(7, 32, 1.0), (64, 4096, 1.0), (33, 2048, 1e-30), (16, 96, 1e30)])
def test_quantize_mxfp8_bit_exact(M, K, scale):
    rng = np.random.default_rng(M + K)
    x = (rng.standard_normal((M, K)) * scale * np.exp(rng.uniform(-8, 8, (M, 1)))).astype(np.float32)
    x[0, :32] = 0.0                     # zero block
    x[min(1, M - 1), 3] = -0.0
    if M > 4:
        x[2, :] = np.float32(2.0 ** -130)  # BF16 subnormals
        x[3, 5] = 3.0e38
    bits = inputs.bf16_bits(x)
    c, s = gpu_mx8(bits)
    rc, rs = oracle.quantize_mxfp8_bf16(bits)
    assert np.array_equal(s, rs)
    assert np.array_equal(c, rc)


def test_quantize_mxfp8_ties_and_saturation():
    # every BF16 value in [1, 2) and its negation against a block max of 2^8 - 1 ulp:
    # the rounding ties of the E4M3 grid and the saturation at 448 all appear
    vals = np.arange(0x3F80, 0x4000, dtype=np.uint32) << 16
    f = vals.view(np.float32)
    x = np.concatenate([f, -f, f * 300.0, -f * 300.0]).astype(np.float32)
    x = x[: (len(x) // 32) * 32].reshape(-1, 32)
    bits = inputs.bf16_bits(x)
    c, s = gpu_mx8(bits)
    rc, rs = oracle.quantize_mxfp8_bf16(bits)
    assert np.array_equal(s, rs) and np.array_equal(c, rc)


def test_w4a8_layer_tiny_all_tokens():
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl)
    w = nvfp4_weights_from_inputs(d, use_oracle_transcode=True)
    layer = GpuLayer(moe.W4A8, w, wl.T, wl.n_group, wl.topk_group, wl.top_k)
    x, lg = bf16_tensor(d["x"]), dev(d["logits"])
    ref = oracle_layer(moe.W4A8, d, w, wl)
    out, _, _ = layer.forward(x, lg, out_fp32=True)
    compare_layer(out_to_f64(out), ref)
    out16, _, _ = layer.forward(x, lg)
    compare_layer(out_to_f64(out16), ref, bf16_output=True)
    # it is not the W4A4 layer
    w4 = oracle_layer(moe.W4A4, d, w, wl)
    assert np.linalg.norm(ref - w4) > 1e-3 * np.linalg.norm(ref)


def test_w4a8_layer_edges():
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl)
    w = nvfp4_weights_from_inputs(d, use_oracle_transcode=True)
    layer = GpuLayer(moe.W4A8, w, 1, wl.n_group, wl.topk_group, wl.top_k)
    out, _, _ = layer.forward(bf16_tensor(d["x"][:1]), dev(d["logits"][:1]), out_fp32=True)
    compare_layer(out_to_f64(out), oracle_layer(moe.W4A8, {"x": d["x"][:1], "logits": d["logits"][:1]}, w, wl))
    # 300 tokens on 4 experts: more than two 128-row tiles per expert, an odd last half
    T = 300
    rng = np.random.default_rng(29)
    x = inputs.activations(rng, T, wl.H, outliers=True)
    lg = np.full((T, wl.E), -8.0, np.float32)
    lg[:, [1, 2, 7, 12]] = 8.0
    lg += rng.standard_normal((T, wl.E)).astype(np.float32) * 0.01
    out, _, _ = layer.forward(bf16_tensor(x), dev(lg), out_fp32=True)
    compare_layer(out_to_f64(out), oracle_layer(moe.W4A8, {"x": x, "logits": lg}, w, wl))
    a, _, _ = layer.forward(bf16_tensor(x), dev(lg))
    b, _, _ = layer.forward(bf16_tensor(x), dev(lg))
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))  # deterministic
    empty = torch.empty((0, wl.H), dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(moe.W4A8, empty, torch.empty((0, wl.E), device="cuda"), None, layer.packed, 1.0, 0, wl.H, wl.I,
                    wl.E, wl.n_group, wl.topk_group, wl.top_k, wl.rsf, True, layer.ws, empty)


def test_w4a8_pack_rejects_weights_without_power_of_two_scales():
    wl = inputs.WORKLOADS["tiny"]
    rng = np.random.default_rng(5)
    E, H, I = wl.E, wl.H, wl.I
    gc, gs, gg = inputs.nvfp4_tensors(rng, E, I, H)
    uc, us, ug = inputs.nvfp4_tensors(rng, E, I, H)
    dc, ds, dg = inputs.nvfp4_tensors(rng, E, H, I)
    w = dict(gate_codes=gc, gate_sf=gs, up_codes=uc, up_sf=us, down_codes=dc, down_sf=ds,
             w_global=np.stack([gg, ug, dg], axis=1).astype(np.float32))
    with pytest.raises(moe.NVFP4MoEError) as ei:
        GpuLayer(moe.W4A8, w, 4, wl.n_group, wl.topk_group, wl.top_k)
    assert ei.value.status == 5


def test_w4a8_prefill_full_size_sampled():
    wl = inputs.WORKLOADS["prefill_pow2"]
    d = inputs.moe_inputs(wl)
    w = nvfp4_weights_from_inputs(d, False)
    layer = GpuLayer(moe.W4A8, w, wl.T, wl.n_group, wl.topk_group, wl.top_k)
    out16, _, _ = layer.forward(bf16_tensor(d["x"]), dev(d["logits"]))
    out, ids, _ = layer.forward(bf16_tensor(d["x"]), dev(d["logits"]), out_fp32=True)
    # >= 512 seeded tokens covering every 128-row run of every expert, held in
    # two halves at the down projection's input (see check_layer_split)
    toks = covering_tokens(host(ids), wl.E, wl.seed)
    check_layer_split(layer, d, w, wl, toks, out, out16)
    del layer
    torch.cuda.empty_cache()
