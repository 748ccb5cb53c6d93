"""GPU parity of the layer modes on shapes and entry points the workload tests
do not reach: the W4A16 stream with 2-chunk groups at a mid size (I not a
multiple of 256), the compact form there, the precomputed-routing entry point
in every mode, and W4A8 with a selection bias and without renormalisation."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import nvfp4_mixture_experts_grouped_b200 as moe
import oracle
from nvfp4_mixture_experts_grouped_b200 import inputs

from helpers import GpuLayer, bf16_tensor, compare_layer, dev, host, out_to_f64

pytestmark = pytest.mark.gpu

MID = dict(T=24, H=1024, I=384, E=32, ng=4, tg=2, k=4)  # I % 256 != 0: 2-chunk groups


def mid_weights(pow2: bool, seed: int):
    rng = np.random.default_rng(seed)
    gen = inputs.nvfp4_pow2_tensors if pow2 else inputs.nvfp4_tensors
    E, H, I = MID["E"], MID["H"], MID["I"]
    gc, gs, gg = gen(rng, E, I, H)
    uc, us, ug = gen(rng, E, I, H)
    dc, ds, dg = gen(rng, E, H, I)
    w = dict(gate_codes=gc, gate_sf=gs, up_codes=uc, up_sf=us, down_codes=dc, down_sf=ds,
             w_global=np.stack([gg, ug, dg], axis=1).astype(np.float32))
    x = inputs.activations(rng, MID["T"], H)
    logits = inputs.router_logits(rng, MID["T"], E)
    return w, x, logits


def oracle_mid(mode, w, x, logits, bias=None, renorm=True, rsf=2.827):
    return oracle.moe_layer(mode, x, logits, bias, w["gate_codes"], w["gate_sf"], w["up_codes"], w["up_sf"],
                            w["down_codes"], w["down_sf"], w["w_global"], 1.0, MID["ng"], MID["tg"], MID["k"], rsf,
                            renorm)


def run(layer, x, logits, bias=None, renorm=True, out_fp32=True):
    out, ids, wts = layer.forward(bf16_tensor(x), dev(logits), bias=None if bias is None else dev(bias),
                                  out_fp32=out_fp32, renormalize=renorm)
    return out, ids, wts


def test_w4a16_two_chunk_groups_mid_size():
    w, x, lg = mid_weights(False, 31)
    layer = GpuLayer(moe.W4A16, w, MID["T"], MID["ng"], MID["tg"], MID["k"])
    out, _, _ = run(layer, x, lg)
    compare_layer(out_to_f64(out), oracle_mid(0, w, x, lg))


def test_compact_two_chunk_groups_mid_size_equals_w4a16():
    w, x, lg = mid_weights(True, 32)
    c = GpuLayer(moe.W4A16C, w, MID["T"], MID["ng"], MID["tg"], MID["k"])
    b = GpuLayer(moe.W4A16, w, MID["T"], MID["ng"], MID["tg"], MID["k"])
    oc, _, _ = run(c, x, lg)
    ob, _, _ = run(b, x, lg)
    assert torch.equal(oc.view(torch.int32), ob.view(torch.int32))
    compare_layer(out_to_f64(oc), oracle_mid(0, w, x, lg))


@pytest.mark.parametrize("mode", [moe.W4A16, moe.W4A16C, moe.W4A4, moe.W4A8])
def test_routed_entry_point_equals_full_layer(mode):
    w, x, lg = mid_weights(True, 33)
    layer = GpuLayer(mode, w, MID["T"], MID["ng"], MID["tg"], MID["k"])
    full, ids, wts = run(layer, x, lg, out_fp32=False)
    out = torch.empty_like(full)
    moe.moe_forward_routed(mode, bf16_tensor(x), ids, wts, layer.packed, 1.0, MID["T"], MID["H"], MID["I"], MID["E"],
                           MID["k"], layer.ws, out)
    torch.cuda.synchronize()
    moe.nvfp4moe_check_device_status()
    assert torch.equal(out.view(torch.int16), full.view(torch.int16))


def test_w4a8_bias_without_renormalisation():
    w, x, lg = mid_weights(True, 34)
    rng = np.random.default_rng(35)
    bias = (rng.standard_normal(MID["E"]) * 0.5).astype(np.float32)
    layer = GpuLayer(moe.W4A8, w, MID["T"], MID["ng"], MID["tg"], MID["k"])
    out, ids, wts = run(layer, x, lg, bias=bias, renorm=False)
    ri, rw = oracle.route(lg, bias, MID["ng"], MID["tg"], MID["k"], 2.827, False)
    assert np.array_equal(host(ids), ri) and np.array_equal(host(wts).view(np.uint32), rw.view(np.uint32))
    compare_layer(out_to_f64(out), oracle_mid(3, w, x, lg, bias=bias, renorm=False))


@pytest.mark.parametrize("mode", [moe.W4A16, moe.W4A4, moe.W4A8])
def test_single_expert_layer(mode):
    # E = 1, top-1: every token on the one expert (several 256-row tiles and a ragged last one)
    rng = np.random.default_rng(36)
    E, H, I, T = 1, 512, 256, 300
    gen = inputs.nvfp4_pow2_tensors
    gc, gs, gg = gen(rng, E, I, H)
    uc, us, ug = gen(rng, E, I, H)
    dc, ds, dg = gen(rng, E, H, I)
    w = dict(gate_codes=gc, gate_sf=gs, up_codes=uc, up_sf=us, down_codes=dc, down_sf=ds,
             w_global=np.stack([gg, ug, dg], axis=1).astype(np.float32))
    x = inputs.activations(rng, T, H)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    layer = GpuLayer(mode, w, T, 1, 1, 1)
    out, ids, wts = layer.forward(bf16_tensor(x), dev(logits), out_fp32=True)
    assert not host(ids).any()
    ref = oracle.moe_layer(mode, x, logits, None, gc, gs, uc, us, dc, ds, w["w_global"], 1.0, 1, 1, 1, 2.827, True)
    compare_layer(out_to_f64(out), ref)
