"""GPU parity of the compact (4.125-bit) scale form: the encoding
(nvfp4_compact_scales) bit-exact against the oracle, and the layer in mode
W4A16C against the float64 oracle (W4A16 arithmetic on the same weight values)
and bit for bit against mode W4A16 on the same weights: the compact form only
moves a power of two per row from the weights to the accumulators."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import nvfp4_mixture_experts_grouped_b200 as moe
import oracle
from nvfp4_mixture_experts_grouped_b200 import inputs

from helpers import GpuLayer, bf16_tensor, compare_layer, dev, host, nvfp4_weights_from_inputs, oracle_layer, out_to_f64

pytestmark = pytest.mark.gpu


def gpu_compact(codes: np.ndarray, sf: np.ndarray, rows: int, K: int):
    nib = torch.empty((rows, K // 64), dtype=torch.uint8, device="cuda")
    rexp = torch.empty(rows, dtype=torch.int8, device="cuda")
    status = torch.empty(rows, dtype=torch.int32, device="cuda")
    n_bad = torch.full((4,), -7, dtype=torch.int32, device="cuda")
    moe.nvfp4_compact_scales(dev(codes.reshape(rows, K // 2)), dev(sf.reshape(rows, K // 16)), rows, K, nib, rexp,
                             status, n_bad)
    torch.cuda.synchronize()
    return host(nib), host(rexp), host(status), int(host(n_bad)[0])


def assert_compact_equal(codes, sf, rows, K):
    got = gpu_compact(codes, sf, rows, K)
    ref = oracle.compact_scales(codes.reshape(rows, K // 2), sf.reshape(rows, K // 16), rows, K)
    assert np.array_equal(got[0], ref[0])
    assert np.array_equal(got[1], ref[1])
    assert np.array_equal(got[2], ref[2])
    assert got[3] == ref[3]
    return ref[3]


@pytest.mark.parametrize("lo,hi,rows,K", [(-8, -3, 37, 256), (-9, 8, 300, 512), (-20, -6, 64, 4096), (3, 17, 9, 192),
                                          (-9, 8, 1000, 2048)])
def test_compact_scales_of_transcoded_tensors(lo, hi, rows, K):
    rng = np.random.default_rng(rows + K)
    codes, e8 = inputs.mxfp4_tensors(rng, 1, rows, K, lo, hi)
    codes[0, 1, 0:16] = 0x80  # an all-zero block
    codes[0, 2, :] = 0x08     # an all-zero row
    c2, e4, *_ = oracle.transcode(codes, e8, 1, rows, K)
    bad = assert_compact_equal(c2[0], e4[0], rows, K)
    if hi - lo > 14:
        assert bad > 0  # rows past the 4-bit range are reported


def test_compact_scales_reject_general_nvfp4_and_crafted_blocks():
    rng = np.random.default_rng(3)
    codes, sf, _ = inputs.nvfp4_tensors(rng, 1, 40, 256)
    assert assert_compact_equal(codes[0], sf[0], 40, 256) > 0
    # crafted rows: unequal halves, non-power-of-two, NaN, negative, zero scale over
    # non-zero codes, +0/-0 halves over zero codes, spread 14 and 15, subnormal powers
    rows = [((0x38, 0x30),), ((0x39, 0x39),), ((0x7F, 0x7F),), ((0xB8, 0xB8),), ((0x00, 0x00),), ((0x00, 0x80),),
            ((0x78, 0x78), (0x08, 0x08)), ((0x78, 0x78), (0x04, 0x04)), ((0x01, 0x01), (0x02, 0x02), (0x04, 0x04))]
    R, K = len(rows), 128
    codes = np.full((R, K // 2), 0x11, np.uint8)
    sf = np.full((R, K // 16), 0x38, np.uint8)
    for r, blocks in enumerate(rows):
        for b, (s0, s1) in enumerate(blocks):
            sf[r, 2 * b], sf[r, 2 * b + 1] = s0, s1
    codes[5, 0:16] = 0x00  # the +0/-0 row has zero codes in that block
    assert assert_compact_equal(codes, sf, R, K) == 6


def test_compact_layer_tiny_matches_oracle_and_w4a16_bits():
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl)
    w = nvfp4_weights_from_inputs(d, use_oracle_transcode=True)
    x, lg = bf16_tensor(d["x"]), dev(d["logits"])
    c = GpuLayer(moe.W4A16C, w, wl.T, wl.n_group, wl.topk_group, wl.top_k)
    ref16 = GpuLayer(moe.W4A16, w, wl.T, wl.n_group, wl.topk_group, wl.top_k)
    assert c.packed.numel() < ref16.packed.numel()
    ref = oracle_layer(moe.W4A16C, d, w, wl)
    for fp32 in (True, False):
        out, _, _ = c.forward(x, lg, out_fp32=fp32)
        base, _, _ = ref16.forward(x, lg, out_fp32=fp32)
        assert torch.equal(out.view(torch.int32 if fp32 else torch.int16), base.view(torch.int32 if fp32 else torch.int16))
        compare_layer(out_to_f64(out), ref, bf16_output=not fp32)


def test_compact_layer_edges():
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl)
    w = nvfp4_weights_from_inputs(d, use_oracle_transcode=True)
    layer = GpuLayer(moe.W4A16C, w, 1, wl.n_group, wl.topk_group, wl.top_k)
    out, _, _ = layer.forward(bf16_tensor(d["x"][:1]), dev(d["logits"][:1]), out_fp32=True)
    compare_layer(out_to_f64(out), oracle_layer(moe.W4A16C, {"x": d["x"][:1], "logits": d["logits"][:1]}, w, wl))
    # 100 tokens on the same 4 experts: several 16-token passes per expert
    T = 100
    rng = np.random.default_rng(19)
    x = inputs.activations(rng, T, wl.H)
    lg = np.full((T, wl.E), -8.0, np.float32)
    lg[:, [3, 5, 6, 9]] = 8.0
    lg += rng.standard_normal((T, wl.E)).astype(np.float32) * 0.01
    out, _, _ = layer.forward(bf16_tensor(x), dev(lg), out_fp32=True)
    compare_layer(out_to_f64(out), oracle_layer(moe.W4A16C, {"x": x, "logits": lg}, w, wl))
    empty = torch.empty((0, wl.H), dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(moe.W4A16C, empty, torch.empty((0, wl.E), device="cuda"), None, layer.packed, 1.0, 0, wl.H, wl.I,
                    wl.E, wl.n_group, wl.topk_group, wl.top_k, wl.rsf, True, layer.ws, empty)


def test_compact_pack_rejects_weights_without_compact_form():
    wl = inputs.WORKLOADS["tiny"]
    rng = np.random.default_rng(4)
    E, H, I = wl.E, wl.H, wl.I
    gc, gs, gg = inputs.nvfp4_tensors(rng, E, I, H)
    uc, us, ug = inputs.nvfp4_tensors(rng, E, I, H)
    dc, ds, dg = inputs.nvfp4_tensors(rng, E, H, I)
    w = dict(gate_codes=gc, gate_sf=gs, up_codes=uc, up_sf=us, down_codes=dc, down_sf=ds,
             w_global=np.stack([gg, ug, dg], axis=1).astype(np.float32))
    with pytest.raises(moe.NVFP4MoEError) as ei:
        GpuLayer(moe.W4A16C, w, 4, wl.n_group, wl.topk_group, wl.top_k)
    assert ei.value.status == 5  # NVFP4MOE_ERR_NOT_REPRESENTABLE


def test_compact_decode_full_size_sampled():
    wl = inputs.WORKLOADS["decode_pow2"]
    d = inputs.moe_inputs(wl)
    w = nvfp4_weights_from_inputs(d, False)
    x, lg = bf16_tensor(d["x"]), dev(d["logits"])
    c = GpuLayer(moe.W4A16C, w, wl.T, wl.n_group, wl.topk_group, wl.top_k)
    out, _, _ = c.forward(x, lg, out_fp32=True)
    del c
    torch.cuda.empty_cache()
    ref16 = GpuLayer(moe.W4A16, w, wl.T, wl.n_group, wl.topk_group, wl.top_k)
    base, _, _ = ref16.forward(x, lg, out_fp32=True)
    del ref16
    torch.cuda.empty_cache()
    assert torch.equal(out.view(torch.int32), base.view(torch.int32))
    compare_layer(out_to_f64(out), oracle_layer(moe.W4A16C, d, w, wl))  # all 16 tokens
