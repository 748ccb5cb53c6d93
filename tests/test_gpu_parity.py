"""GPU parity: every step of the CUDA path against the CPU oracle, through the
C ABI.  Integer results (transcode codes/scales/globals, routing ids, routing
weights as bits, quantised codes and scales, permutation) must be bit-exact;
layer outputs must be within rel-L2 2e-3 and max-abs 1e-2 * rms(out) of the
float64 oracle."""
import numpy as np
import pytest
import torch

import nvfp4_mixture_experts_grouped_b200 as moe
import oracle
from nvfp4_mixture_experts_grouped_b200 import inputs

from helpers import (GpuLayer, bf16_tensor, check_layer_split, compare_layer, covering_tokens, dev, gpu_transcode,
                     host, nvfp4_weights_from_inputs, oracle_layer, out_to_f64)

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------------------
# transcode
# ---------------------------------------------------------------------------

def _assert_transcode_equal(codes, e8m0, in_place=False):
    nt, N, kh = codes.shape
    rc, re4, rg, rst, rrep, rworst = oracle.transcode(codes, e8m0, nt, N, kh * 2)
    gc, ge4, gg, gst, grep, gstatus = gpu_transcode(codes, e8m0, in_place=in_place)
    assert np.array_equal(gst, rst)
    assert np.array_equal(gc.reshape(-1), rc.reshape(-1))
    assert np.array_equal(ge4, re4)
    assert np.array_equal(gg.view(np.uint32), rg.view(np.uint32))
    assert grep["blocks"] == rrep[0] and grep["zero_blocks"] == rrep[1]
    assert grep["nonrepresentable_tensors"] == rrep[2] and grep["nan_scale_tensors"] == rrep[3]
    expect_status = {0: 0, 1: 5, 2: 4}[rworst]
    assert gstatus == expect_status


def test_transcode_tiny_layer_weights():
    d = inputs.moe_inputs(inputs.WORKLOADS["tiny"])
    for name in ("gate", "up", "down"):
        _assert_transcode_equal(*d["mx"][name])


@pytest.mark.parametrize("in_place", [False, True])
def test_transcode_windows_edges_and_failures(in_place):
    rng = np.random.default_rng(77)
    nt, N, K = 12, 64, 256
    lo = rng.integers(-30, 20, nt)
    w = rng.integers(0, 18, nt)
    codes, e8 = inputs.mxfp4_tensors(rng, nt, N, K, lo, lo + w)
    e8[0] = 127 - 120  # extreme but uniform exponents
    e8[1, 0, 0] = 127 + 17
    e8[1, 1:] = 127  # spread 17: exact
    e8[2, 0, 0] = 127 + 18
    e8[2, 1:] = 127  # spread 18: not representable
    codes[3] = 0x88  # all blocks +-0
    e8[4, 5, 3] = 0xFF  # NaN scale on a non-zero block
    codes[5, 7, 0:16] = 0x80  # one all-zero block whose E8M0 is NaN: ignored
    e8[5, 7, 0] = 0xFF
    _assert_transcode_equal(codes, e8, in_place=in_place)


def test_transcode_large_tensor_uncached_path():
    # 2^21+ blocks per tensor: more than the per-CTA shared-memory cache holds
    rng = np.random.default_rng(5)
    codes, e8 = inputs.mxfp4_tensors(rng, 1, 8192, 8448, -12, 3)
    _assert_transcode_equal(codes, e8)


def test_transcode_full_layer_all_tensors():
    """The full transcode workload on the GPU: 768 expert tensors of one layer
    (gate and up [2048, 4096] out of place, down [4096, 2048] in place) plus the
    adversarial tensor; every tensor's E4M3 scales, global and status equal the
    oracle's, the codes are byte-identical and the report counts agree."""
    rng = np.random.default_rng(inputs.TRANSCODE_SEED)
    layer = inputs.transcode_layer(rng)
    batches = (("gate", 2048, 4096, False, True), ("up", 2048, 4096, False, False), ("down", 4096, 2048, True, False))
    n_checked = 0
    for name, N, K, in_place, with_adversarial in batches:
        codes, e8 = layer[name]
        if with_adversarial:
            codes = np.concatenate([codes, layer["adversarial"][0]])
            e8 = np.concatenate([e8, layer["adversarial"][1]])
        nt = codes.shape[0]
        gc, ge4, gg, gst, grep, gstatus = gpu_transcode(codes, e8, in_place=in_place)
        rc, re4, rg, rst, rrep, _ = oracle.transcode(codes, e8, nt, N, K)
        assert np.array_equal(gc, codes) and np.array_equal(rc.reshape(codes.shape), codes)
        assert np.array_equal(ge4, re4)
        assert np.array_equal(gg.view(np.uint32), rg.view(np.uint32))
        assert np.array_equal(gst, rst)
        assert [grep["blocks"], grep["zero_blocks"], grep["nonrepresentable_tensors"], grep["nan_scale_tensors"]] == \
            rrep.tolist()
        if with_adversarial:
            assert gstatus == 5 and gst[-1] == 1 and np.all(gst[:-1] == 0)
        else:
            assert gstatus == 0 and np.all(gst == 0)
        n_checked += nt
        del codes, e8, gc, ge4, rc, re4
    assert n_checked == 769


# ---------------------------------------------------------------------------
# routing
# ---------------------------------------------------------------------------

def _gpu_route(logits, bias, ng, tg, k, rsf, renorm=True):
    T, E = logits.shape
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(dev(logits), None if bias is None else dev(bias), ng, tg, k, rsf, renorm, ids, w)
    torch.cuda.synchronize()
    return host(ids), host(w)


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "skewed"])
def test_route_workloads_bit_exact(name):
    wl = inputs.WORKLOADS[name]
    rng = np.random.default_rng(wl.seed)
    logits = inputs.router_logits(rng, wl.T, wl.E, wl.zipf)
    gi, gw = _gpu_route(logits, None, wl.n_group, wl.topk_group, wl.top_k, wl.rsf)
    ri, rw = oracle.route(logits, None, wl.n_group, wl.topk_group, wl.top_k, wl.rsf)
    assert np.array_equal(gi, ri)
    assert np.array_equal(gw.view(np.uint32), rw.view(np.uint32))


@pytest.mark.parametrize("E,ng,tg,k", [(16, 4, 2, 4), (256, 8, 4, 8), (128, 8, 4, 8), (64, 1, 1, 6), (96, 3, 2, 5),
                                       (1024, 32, 8, 32), (32, 32, 32, 32), (8, 8, 3, 3)])
@pytest.mark.parametrize("ties", [False, True])
def test_route_shapes_ties_bias(E, ng, tg, k, ties):
    rng = np.random.default_rng(E + ng + k)
    T = 97
    if ties:
        logits = rng.integers(-3, 4, size=(T, E)).astype(np.float32) * 0.5
        bias = None
    else:
        logits = (rng.standard_normal((T, E)) * 3).astype(np.float32)
        logits[0, :] = 0.0  # every expert ties
        bias = (rng.standard_normal(E) * 0.05).astype(np.float32)
    for renorm in (True, False):
        gi, gw = _gpu_route(logits, bias, ng, tg, k, 2.827, renorm)
        ri, rw = oracle.route(logits, bias, ng, tg, k, 2.827, renorm)
        assert np.array_equal(gi, ri)
        assert np.array_equal(gw.view(np.uint32), rw.view(np.uint32))


def test_route_extreme_logits():
    rng = np.random.default_rng(3)
    logits = rng.uniform(-120, 120, size=(64, 256)).astype(np.float32)
    gi, gw = _gpu_route(logits, None, 8, 4, 8, 2.827)
    ri, rw = oracle.route(logits, None, 8, 4, 8, 2.827)
    assert np.array_equal(gi, ri) and np.array_equal(gw.view(np.uint32), rw.view(np.uint32))


@pytest.mark.parametrize("E,ng,tg,k", [(256, 8, 4, 8), (128, 8, 4, 8), (16, 4, 2, 4), (96, 4, 2, 6), (60, 5, 2, 4)])
def test_route_nan_and_infinite_bias(E, ng, tg, k):
    # NaN bias entries rank their experts last (as -inf); +inf and -inf in one
    # group give that group a -inf score.  Covers the row, segment and general
    # per-token routines: ids, order and weight bits as the oracle, every id a
    # distinct expert.
    rng = np.random.default_rng(E + k)
    T = 64
    logits = rng.standard_normal((T, E)).astype(np.float32)
    gsz = E // ng
    for case in range(3):
        bias = (rng.standard_normal(E) * 0.05).astype(np.float32)
        if case == 0:
            bias[rng.choice(E, E // 3, replace=False)] = np.nan
        elif case == 1:
            bias[:] = np.nan
        else:
            bias[0], bias[min(1, E - 1)] = np.inf, -np.inf
            bias[gsz:2 * gsz] = np.nan
        for kk in (k, min(32, tg * gsz)):
            gi, gw = _gpu_route(logits, bias, ng, tg, kk, 2.827)
            ri, rw = oracle.route(logits, bias, ng, tg, kk, 2.827)
            assert np.array_equal(gi, ri)
            assert np.array_equal(gw.view(np.uint32), rw.view(np.uint32))
            assert gi.min() >= 0 and gi.max() < E
            assert all(len(set(r)) == kk for r in gi.tolist())


def test_routed_entry_point_reports_bad_ids():
    # precomputed routing with an id outside [0, E), a negative id and a repeated
    # id: those tokens come out as zero rows, the others exactly as with good
    # routing, and the device status reports INVALID_ARG once, then clears
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl)
    w = nvfp4_weights_from_inputs(d, False)
    for mode in (moe.W4A4, moe.W4A16):
        layer = GpuLayer(mode, w, wl.T, wl.n_group, wl.topk_group, wl.top_k)
        x = bf16_tensor(d["x"])
        good, ids, wts = layer.forward(x, dev(d["logits"]), out_fp32=True)
        bad_ids = ids.clone()
        bad_ids[3, 1] = wl.E
        bad_ids[7, 2] = bad_ids[7, 0]
        bad_ids[9, 0] = -1
        out = torch.empty_like(good)
        moe.moe_forward_routed(mode, x, bad_ids, wts, layer.packed, 1.0, wl.T, wl.H, wl.I, wl.E, wl.top_k, layer.ws,
                               out)
        with pytest.raises(moe.NVFP4MoEError) as ei:
            moe.nvfp4moe_check_device_status()
        assert ei.value.status == 1  # ERR_INVALID_ARG
        moe.nvfp4moe_check_device_status()  # cleared
        o, g = host(out), host(good)
        bad = [3, 7, 9]
        assert np.all(o[bad] == 0.0)
        keep = [t for t in range(wl.T) if t not in bad]
        assert np.array_equal(o[keep].view(np.uint32), g[keep].view(np.uint32))


# ---------------------------------------------------------------------------
# permutation
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,E,k,pad", [(32, 16, 4, 128), (16, 256, 8, 1), (1000, 64, 6, 128), (8192, 256, 8, 128),
                                       (3, 8, 8, 1), (600, 1024, 32, 1),
                                       # both sides of the one-CTA path's limit (8192 pairs, E <= 256)
                                       (1024, 256, 8, 128), (1025, 256, 8, 128), (2048, 256, 4, 1), (64, 257, 8, 1)])
def test_permute_against_oracle(T, E, k, pad):
    rng = np.random.default_rng(T + E)
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    poff = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    rop = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.moe_permute_workspace_size(T, E, k, pad), dtype=torch.uint8, device="cuda")
    assert moe.load().moe_permute(None, 4, E, k, pad, None, None, None, None, 0, None) != 0  # null pointers
    moe.moe_permute(dev(ids), E, pad, counts, poff, rop, ws)
    torch.cuda.synchronize()
    rc, ro, rrop, _ = oracle.permute(ids, E)
    gc, gpo, grop = host(counts), host(poff), host(rop)
    assert np.array_equal(gc, rc)
    padded = ((rc + pad - 1) // pad) * pad
    assert np.array_equal(gpo, np.concatenate([[0], np.cumsum(padded)]).astype(np.int32))
    e_of = ids.reshape(-1)
    assert np.array_equal(grop - gpo[e_of], rrop - ro[e_of])  # identical rank inside each expert


# ---------------------------------------------------------------------------
# quantisation
# ---------------------------------------------------------------------------

def _gpu_quant(xbits, gs=1.0):
    M, K = xbits.shape
    c = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    s = torch.empty((M, K // 16), dtype=torch.uint8, device="cuda")
    moe.quantize_nvfp4(bf16_tensor(xbits), gs, c, s)
    torch.cuda.synchronize()
    return host(c), host(s)


@pytest.mark.parametrize("gs", [1.0, 0.375, 3.0])
def test_quantize_random_and_outliers_bit_exact(gs):
    rng = np.random.default_rng(int(gs * 8))
    x = inputs.activations(rng, 257, 4096, outliers=True)
    gc, gsf = _gpu_quant(x, gs)
    rc, rs = oracle.quantize_bf16(x, gs)
    assert np.array_equal(gsf, rs)
    assert np.array_equal(gc, rc)


def test_quantize_ties_signed_zeros_subnormal_scales():
    blocks = []
    mags = [0.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 7.0]
    for s in (1.0, 0.5, 2.0 ** -8, 2.0 ** -10, 448.0, 2 ** -12):  # block scales incl. E4M3 subnormals
        for sign in (1.0, -1.0):
            b = np.array(mags, np.float32) * np.float32(s) * sign
            b[0] = 6.0 * s  # pins the scale
            blocks.append(b)
    blocks.append(np.array([-0.0] * 16, np.float32))
    blocks.append(np.array([1e-30, -1e-30] * 8, np.float32))
    blocks.append(np.array([3e5, -3e5] + [1.0] * 14, np.float32))
    x = inputs.bf16_bits(np.concatenate(blocks).reshape(-1, 16))
    gc, gsf = _gpu_quant(x)
    rc, rs = oracle.quantize_bf16(x)
    assert np.array_equal(gsf, rs)
    assert np.array_equal(gc, rc)


def test_quantize_exhaustive_bf16_ratios():
    # every positive BF16 bit pattern in [2^-12, 2^9), fifteen per block after a 6
    vals = np.arange(0x3980, 0x4400, dtype=np.uint32)  # bit patterns
    f = (vals << 16).view(np.float32)
    n = (len(f) // 15) * 15
    body = f[:n].reshape(-1, 15)
    x = np.concatenate([np.full((body.shape[0], 1), 6.0, np.float32), body], axis=1)
    x = np.concatenate([x, -x], axis=0)
    xb = inputs.bf16_bits(x.reshape(-1, 32))
    gc, gsf = _gpu_quant(xb)
    rc, rs = oracle.quantize_bf16(xb)
    assert np.array_equal(gsf, rs) and np.array_equal(gc, rc)


def _blocks_below(anchor_bits, lo_bits, hi_bits):
    """Blocks of 16 BF16 values: the anchor (the block's amax, which fixes its
    scale) followed by every BF16 pattern in [lo_bits, hi_bits) with both signs,
    fifteen per block (zeros pad the last)."""
    mags = np.arange(lo_bits, hi_bits, dtype=np.uint32)
    body = np.concatenate([mags, mags | 0x8000]).astype(np.uint16)
    n = -(-len(body) // 15) * 15
    body = np.concatenate([body, np.zeros(n - len(body), np.uint16)]).reshape(-1, 15)
    return np.concatenate([np.full((body.shape[0], 1), anchor_bits, np.uint16), body], axis=1)


def test_quantize_unit_global_every_scale_every_magnitude():
    # gs == 1 takes the division-free quantiser; its codes must be the IEEE
    # division's for every (x, scale) pair a block can hold.  Anchors: every
    # positive BF16 amax from 2^-10 (scale 0 and the E4M3 subnormal scales) to
    # 2^12 (past the 448 saturation), each with every BF16 magnitude in
    # [amax/32, amax]; below that quotients are < 0.29 and fall to codes 0/0.5
    # only through other anchors of the same scale.  Then a few anchors with every
    # tiny BF16 value (FP32-subnormal range included) and huge anchors up to the
    # BF16 maximum (saturated scale 448, codes 6).
    parts = [_blocks_below(a, a - (5 << 7), a + 1) for a in range(117 << 7, (139 << 7) + 1)]
    for a in (0x3A80, 0x3C00, 0x3F80, 0x4300, 0x4580):
        parts.append(_blocks_below(a, 0x0001, 0x0A80))
    for a in range(139 << 7, 0x7F80, 61):
        parts.append(_blocks_below(a, a - (5 << 7), a + 1))
    x = np.concatenate(parts)
    pad = (-x.shape[0]) % 16
    x = np.concatenate([x, np.zeros((pad, 16), np.uint16)]).reshape(-1, 256)
    gc, gsf = _gpu_quant(x, 1.0)
    rc, rs = oracle.quantize_bf16(x, 1.0)
    assert np.array_equal(gsf, rs)
    assert np.array_equal(gc, rc)


# ---------------------------------------------------------------------------
# the layer
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [moe.W4A4, moe.W4A16])
def test_layer_tiny_all_tokens(mode):
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl)
    w_gpu = nvfp4_weights_from_inputs(d, use_oracle_transcode=False)
    w_ref = nvfp4_weights_from_inputs(d, use_oracle_transcode=True)
    for k in w_ref:
        assert np.array_equal(w_gpu[k].view(np.uint8), w_ref[k].view(np.uint8))
    layer = GpuLayer(mode, w_gpu, wl.T, wl.n_group, wl.topk_group, wl.top_k)
    out, ids, wts = layer.forward(bf16_tensor(d["x"]), dev(d["logits"]))
    ref = oracle_layer(mode, d, w_ref, wl)
    ri, rw = oracle.route(d["logits"], None, wl.n_group, wl.topk_group, wl.top_k, wl.rsf)
    assert np.array_equal(host(ids), ri) and np.array_equal(host(wts).view(np.uint32), rw.view(np.uint32))
    compare_layer(out_to_f64(out), ref, bf16_output=True)
    out32, _, _ = layer.forward(bf16_tensor(d["x"]), dev(d["logits"]), out_fp32=True)
    compare_layer(out_to_f64(out32), ref)
    check_layer_split(layer, d, w_ref, wl, np.arange(wl.T, dtype=np.int32), out32, out)


def test_layer_decode_w4a16_full():
    wl = inputs.WORKLOADS["decode"]
    d = inputs.moe_inputs(wl)
    w = nvfp4_weights_from_inputs(d, False)
    layer = GpuLayer(moe.W4A16, w, wl.T, wl.n_group, wl.topk_group, wl.top_k)
    out, _, _ = layer.forward(bf16_tensor(d["x"]), dev(d["logits"]), out_fp32=True)
    ref = oracle_layer(moe.W4A16, d, w, wl)
    compare_layer(out_to_f64(out), ref)
    out16, _, _ = layer.forward(bf16_tensor(d["x"]), dev(d["logits"]))
    compare_layer(out_to_f64(out16), ref, bf16_output=True)
    check_layer_split(layer, d, w, wl, np.arange(wl.T, dtype=np.int32), out, out16)


def test_layer_w4a16_wide_dynamic_range_rows():
    # W4A16 multiplies FP16 rows (each BF16 row scaled by a power of two so that
    # its largest element sits just below 2^15) on FP16 tensor cores: elements
    # far below their row's largest lose relative precision as FP16 subnormals.
    # Rows spanning 2^36 (one element of 2^16 among N(0,1) x 2^-20 ones), a zero
    # row and a row at 2^-60 (its SwiGLU products near 2^-110, still normal FP32)
    # are held to the oracle token by token.
    wl = inputs.WORKLOADS["decode"]
    d = inputs.moe_inputs(wl)
    rng = np.random.default_rng(77)
    x = (rng.standard_normal((wl.T, wl.H)) * 2.0 ** -20).astype(np.float32)
    cols = rng.integers(0, wl.H, size=wl.T)
    x[np.arange(wl.T), cols] = np.where(rng.random(wl.T) < 0.5, -1.0, 1.0) * 2.0 ** 16
    x[3] = 0.0
    x[5] = rng.standard_normal(wl.H).astype(np.float32) * 2.0 ** -60
    x[9] = rng.standard_normal(wl.H).astype(np.float32)  # an ordinary row beside them
    d["x"] = inputs.bf16_bits(x)
    w = nvfp4_weights_from_inputs(d, False)
    layer = GpuLayer(moe.W4A16, w, wl.T, wl.n_group, wl.topk_group, wl.top_k)
    out, _, _ = layer.forward(bf16_tensor(d["x"]), dev(d["logits"]), out_fp32=True)
    ref = oracle_layer(moe.W4A16, d, w, wl)
    got = out_to_f64(out)
    assert np.all(got[3] == 0.0) and np.all(ref[3] == 0.0)
    assert np.any(ref[5] != 0.0)
    for t in range(wl.T):
        if t != 3:
            compare_layer(got[t:t + 1], ref[t:t + 1])
    out16, _, _ = layer.forward(bf16_tensor(d["x"]), dev(d["logits"]))
    for t in range(wl.T):
        if t != 3:
            compare_layer(out_to_f64(out16)[t:t + 1], ref[t:t + 1], bf16_output=True)
    # (no split check here: its error model is the FP32 accumulation alone, and
    # the intermediates these rows make through a zero weight at the outlier's
    # column come from the FP16-subnormal elements only -- large relative error
    # on values that are negligible in the output, which the bounds above hold)


@pytest.mark.parametrize("name", ["prefill", "skewed"])
def test_layer_w4a4_full_size_sampled(name):
    # full-size layers: at least 512 seeded tokens whose rows cover every
    # 128-row run of every expert (tile halves, ragged last chunks, each
    # expert's last row), held in two halves at the down projection's input:
    # the intermediate codes against the oracle's up to boundary flips, the
    # output against the oracle's down half of the GPU's intermediate at the bare
    # bound (BF16 output with its own rounding allowed), and the whole layer
    # (rel-L2 over all, max-abs over tokens without a flip)
    wl = inputs.WORKLOADS[name]
    d = inputs.moe_inputs(wl)
    w = nvfp4_weights_from_inputs(d, False)
    layer = GpuLayer(wl.mode, w, wl.T, wl.n_group, wl.topk_group, wl.top_k)
    out16, _, _ = layer.forward(bf16_tensor(d["x"]), dev(d["logits"]))
    out, ids, _ = layer.forward(bf16_tensor(d["x"]), dev(d["logits"]), out_fp32=True)
    h_ids = host(ids)
    ri, _ = oracle.route(d["logits"], None, wl.n_group, wl.topk_group, wl.top_k, wl.rsf)
    assert np.array_equal(h_ids, ri)
    toks = covering_tokens(h_ids, wl.E, wl.seed)
    assert len(toks) >= 512
    check_layer_split(layer, d, w, wl, toks, out, out16)
    del layer
    torch.cuda.empty_cache()


def test_layer_edge_cases():
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl)
    w = nvfp4_weights_from_inputs(d, False)
    for mode in (moe.W4A4, moe.W4A16):
        layer = GpuLayer(mode, w, 1, wl.n_group, wl.topk_group, wl.top_k)
        # T = 1
        out, _, _ = layer.forward(bf16_tensor(d["x"][:1]), dev(d["logits"][:1]), out_fp32=True)
        compare_layer(out_to_f64(out), oracle_layer(mode, {"x": d["x"][:1], "logits": d["logits"][:1]}, w, wl))
        # every token routed to the same experts (one expert gets > 2 M-tiles of rows)
        T = 300
        rng = np.random.default_rng(9)
        x = inputs.activations(rng, T, wl.H)
        lg = np.full((T, wl.E), -8.0, np.float32)
        lg[:, [0, 1, 2, 3]] = 8.0
        lg += rng.standard_normal((T, wl.E)).astype(np.float32) * 0.01
        out, ids, _ = layer.forward(bf16_tensor(x), dev(lg), out_fp32=True)
        assert set(np.unique(host(ids)).tolist()) == {0, 1, 2, 3}
        ref = oracle_layer(mode, {"x": x, "logits": lg}, w, wl)
        compare_layer(out_to_f64(out), ref)
        # T = 0 is a no-op
        empty = torch.empty((0, wl.H), dtype=torch.bfloat16, device="cuda")
        moe.moe_forward(mode, empty, torch.empty((0, wl.E), device="cuda"), None, layer.packed, 1.0, 0, wl.H, wl.I,
                        wl.E, wl.n_group, wl.topk_group, wl.top_k, wl.rsf, True, layer.ws, empty)


def test_layer_deterministic_and_routed_entry_point():
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl, T=200)
    w = nvfp4_weights_from_inputs(d, False)
    layer = GpuLayer(moe.W4A4, w, 200, wl.n_group, wl.topk_group, wl.top_k)
    x, lg = bf16_tensor(d["x"]), dev(d["logits"])
    a, ids, wts = layer.forward(x, lg)
    b, _, _ = layer.forward(x, lg)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    out = torch.empty_like(a)
    moe.moe_forward_routed(moe.W4A4, x, ids, wts, layer.packed, 1.0, 200, wl.H, wl.I, wl.E, wl.top_k, layer.ws, out)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), a.view(torch.int16))


def test_layer_non_unit_activation_global():
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl)
    w = nvfp4_weights_from_inputs(d, False)
    layer = GpuLayer(moe.W4A4, w, wl.T, wl.n_group, wl.topk_group, wl.top_k)
    out, _, _ = layer.forward(bf16_tensor(d["x"]), dev(d["logits"]), act_global=0.25, out_fp32=True)
    ref = oracle_layer(moe.W4A4, d, w, wl, act_global=0.25)
    compare_layer(out_to_f64(out), ref)


@pytest.mark.parametrize("g_in,g_mid", [("calibrated", 1.0), (1.0, 0.03125), (0.37, 2.5), ("calibrated", 0.125)])
def test_layer_separate_input_and_intermediate_globals(g_in, g_mid):
    # moe_forward_ex: the layer input quantised with g_in, the SwiGLU output
    # (down-projection input) requantised with g_mid.  "calibrated" is the
    # input's amax / 2688, the global that maps it onto the largest E4M3 block
    # scale times the largest E2M1 code.
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl)
    w = nvfp4_weights_from_inputs(d, False)
    if g_in == "calibrated":
        amax = float(np.abs((d["x"].astype(np.uint32) << 16).view(np.float32)).max())
        g_in = float(np.float32(amax / 2688.0))
    layer = GpuLayer(moe.W4A4, w, wl.T, wl.n_group, wl.topk_group, wl.top_k)
    x, lg = bf16_tensor(d["x"]), dev(d["logits"])
    out, _, _ = layer.forward(x, lg, act_global=g_in, act_global_mid=g_mid, out_fp32=True)
    ref = oracle_layer(moe.W4A4, d, w, wl, act_global=g_in, act_global_mid=g_mid)
    compare_layer(out_to_f64(out), ref)
    # the single-global entry point is the same call with both globals equal
    a, _, _ = layer.forward(x, lg, act_global=g_in, act_global_mid=g_in)
    b, _, _ = layer.forward(x, lg, act_global=g_in)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_layer_w4a16_ignores_activation_globals():
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl)
    w = nvfp4_weights_from_inputs(d, False)
    layer = GpuLayer(moe.W4A16, w, wl.T, wl.n_group, wl.topk_group, wl.top_k)
    x, lg = bf16_tensor(d["x"]), dev(d["logits"])
    a, _, _ = layer.forward(x, lg, act_global=0.3, act_global_mid=7.0)
    b, _, _ = layer.forward(x, lg)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_layer_prefill_calibrated_globals_sampled():
    # full prefill size, input global calibrated from the input, the
    # down-projection input's global capped at 1 (amax capped at 2688)
    wl = inputs.WORKLOADS["prefill"]
    d = inputs.moe_inputs(wl)
    w = nvfp4_weights_from_inputs(d, False)
    amax = float(np.abs((d["x"].astype(np.uint32) << 16).view(np.float32)).max())
    g_in = float(np.float32(amax / 2688.0))
    layer = GpuLayer(moe.W4A4, w, wl.T, wl.n_group, wl.topk_group, wl.top_k)
    out16, _, _ = layer.forward(bf16_tensor(d["x"]), dev(d["logits"]), act_global=g_in, act_global_mid=0.5)
    out, ids, _ = layer.forward(bf16_tensor(d["x"]), dev(d["logits"]), act_global=g_in, act_global_mid=0.5,
                                out_fp32=True)
    toks = covering_tokens(host(ids), wl.E, wl.seed + 1)
    check_layer_split(layer, d, w, wl, toks, out, out16, act_global=g_in, act_global_mid=0.5)
    del layer
    torch.cuda.empty_cache()
