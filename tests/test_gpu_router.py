"""GPU parity of the router projection followed by grouped top-k
(moe_router_topk) against the oracle.

Logits: FP32 against the float64 oracle within the rounding bound of the
kernel's fixed summation order, plus the oracle's own one rounding to FP32.
Small token counts: a chain of at most H/64 FMAs per lane, a 5-level butterfly
and the in-order sum of the K slices, |err| <= (H/64 + 6) * 2^-24 * sum|x_h w_h|.
Token counts that fill a wave of 128 x 64 tiles (the tiled projection): an FMA
chain over the even 16-column chunks plus one over the odd chunks, added once,
|err| <= gamma_n * sum|x_h w_h|, n = H/2 + 1, gamma_n = n 2^-24 / (1 - n 2^-24).  At those sizes the logits are compared on sampled
tokens, at least eight from every 128-token tile, on all experts.  Routing:
bit-exact against the oracle's routing of the kernel's own logits (ids, order,
weight bits), which is also what moe_route gives on them."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import nvfp4_mixture_experts_grouped_b200 as moe
import oracle
from nvfp4_mixture_experts_grouped_b200 import inputs

from helpers import dev, host

pytestmark = pytest.mark.gpu

CASES = {
    # name: T, H, E, n_group, topk_group, top_k, bias, seed
    "tiny": (32, 256, 16, 4, 2, 4, False, 11),
    "decode": (16, 4096, 256, 8, 4, 8, False, 12),
    "groups16_bias": (64, 4096, 128, 8, 4, 8, True, 13),
    "general_groups_ragged": (40, 512, 96, 4, 2, 6, True, 14),
    "many_tiles": (300, 1024, 256, 8, 4, 8, False, 15),
    "one_group": (20, 768, 64, 1, 1, 8, False, 16),
    # hidden rows too long for the shared-memory tile (16 x 8192 BF16 = 256 KB):
    # the projection reads them from global memory in its loop
    "long_rows": (24, 8192, 64, 8, 4, 8, True, 17),
    # the tiled projection (ceil(T/128) * ceil(E/64) >= the SM count): a ragged
    # last token tile, and a ragged last expert tile (100 = 64 + 36)
    "prefill_tiled": (8200, 4096, 256, 8, 4, 8, True, 18),
    "tiled_ragged_experts": (9500, 768, 100, 4, 2, 6, False, 19),
}

U = 2.0 ** -24


def uses_tiled(T, E):
    return -(-T // 128) * -(-E // 64) >= torch.cuda.get_device_properties(0).multi_processor_count


def logit_bound_units(T, H, E):
    """The kernel's error bound in units of 2^-24 * sum|x_h w_h|, plus one for
    the oracle's rounding of the float64 sum to FP32."""
    if uses_tiled(T, E):
        n = H / 2 + 1
        return n / (1.0 - n * U) + 1.0
    return H / 64 + 7


def sampled_rows(T, seed, per_tile=8):
    """At least per_tile tokens from every 128-token tile, plus the first and the last."""
    rng = np.random.default_rng(seed)
    rows = {0, T - 1}
    for lo in range(0, T, 128):
        hi = min(T, lo + 128)
        rows.update(rng.choice(np.arange(lo, hi), size=min(per_tile, hi - lo), replace=False).tolist())
    return np.array(sorted(rows))


def run_router(x_bits, w, bias, ng, tg, k, rsf=2.827, renorm=True):
    T, H = x_bits.shape
    E = w.shape[0]
    xd = dev(x_bits.view(np.int16))
    wd = dev(w)
    bd = None if bias is None else dev(bias)
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(16, moe.moe_router_topk_workspace_size(T)), dtype=torch.uint8, device="cuda")
    moe.moe_router_topk(xd, wd, bd, ng, tg, k, rsf, renorm, logits, ids, wts, ws)
    moe.nvfp4moe_check_device_status()
    torch.cuda.synchronize()
    return host(logits), host(ids), host(wts), host(ws)


def case_inputs(name):
    T, H, E, ng, tg, k, with_bias, seed = CASES[name]
    rng = np.random.default_rng(seed)
    x = inputs.bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    w = inputs.router_weights(rng, E, H)
    bias = (rng.standard_normal(E).astype(np.float32) * 0.05) if with_bias else None
    return x, w, bias, ng, tg, k


@pytest.mark.parametrize("name", list(CASES))
def test_router_topk_matches_oracle(name):
    x, w, bias, ng, tg, k = case_inputs(name)
    T, H = x.shape
    E = w.shape[0]
    logits, ids, wts, ws = run_router(x, w, bias, ng, tg, k)
    rows = sampled_rows(T, T) if T > 1024 else np.arange(T)
    if T > 1024:
        assert len(np.unique(rows // 128)) == -(-T // 128)  # every token tile holds a checked token
    ref_logits, mag = oracle.router_logits(x[rows], w)
    bound = logit_bound_units(T, H, E) * U * mag
    err = np.abs(logits[rows].astype(np.float64) - ref_logits.astype(np.float64))
    assert np.all(err <= bound), f"logit error {float((err / np.maximum(mag, 1e-30)).max()):.3e} x sum|xw|"
    # routing of the kernel's own logits: bit-exact
    rid, rw = oracle.route(logits, bias, ng, tg, k, 2.827, True)
    assert np.array_equal(ids, rid)
    assert np.array_equal(wts.view(np.uint32), rw.view(np.uint32))
    # the workspace is not touched
    assert not ws.any()


def test_router_topk_equals_moe_route_on_its_logits_and_is_deterministic():
    x, w, bias, ng, tg, k = case_inputs("decode")
    l1, i1, w1, _ = run_router(x, w, bias, ng, tg, k, renorm=False)
    l2, i2, w2, _ = run_router(x, w, bias, ng, tg, k, renorm=False)
    assert np.array_equal(l1.view(np.uint32), l2.view(np.uint32))
    assert np.array_equal(i1, i2) and np.array_equal(w1.view(np.uint32), w2.view(np.uint32))
    T = x.shape[0]
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(dev(l1), None, ng, tg, k, 2.827, False, ids, wts)
    torch.cuda.synchronize()
    assert np.array_equal(host(ids), i1) and np.array_equal(host(wts).view(np.uint32), w1.view(np.uint32))


@pytest.mark.parametrize("T,H,E", [(24, 1024, 64), (5000, 256, 256)])
def test_router_topk_exact_integer_logits(T, H, E):
    # integer-valued x and router rows: every logit is an exact integer, so the
    # kernel's FP32 sums equal the oracle's bit for bit (5000 tokens: the tiled
    # projection, run twice for bit identity)
    rng = np.random.default_rng(21)
    xi = rng.integers(-4, 5, size=(T, H)).astype(np.float32)
    wi = rng.integers(-8, 9, size=(E, H)).astype(np.float32)
    logits, ids, wts, _ = run_router(inputs.bf16_bits(xi), wi, None, 8, 2, 4)
    ref, _ = oracle.router_logits(inputs.bf16_bits(xi), wi)
    assert np.array_equal(logits, ref)
    rid, rw = oracle.route(ref, None, 8, 2, 4, 2.827, True)
    assert np.array_equal(ids, rid) and np.array_equal(wts.view(np.uint32), rw.view(np.uint32))
    if T > 1024:
        x = rng.standard_normal((T, H), dtype=np.float32)
        w = rng.standard_normal((E, H), dtype=np.float32)
        l1, _, _, _ = run_router(inputs.bf16_bits(x), w, None, 8, 2, 4)
        l2, _, _, _ = run_router(inputs.bf16_bits(x), w, None, 8, 2, 4)
        assert np.array_equal(l1.view(np.uint32), l2.view(np.uint32))
