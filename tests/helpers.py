"""Shared helpers of the GPU parity tests: upload seeded inputs, run the CUDA
path through the C ABI binding, run the oracle on the same bytes, compare."""
from __future__ import annotations

import numpy as np
import torch

import nvfp4_mixture_experts_grouped_b200 as moe
import oracle
from nvfp4_mixture_experts_grouped_b200 import inputs

# spec tolerance for layer outputs against the float64 oracle
REL_L2 = 2e-3
MAX_ABS_OF_RMS = 1e-2


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def bf16_tensor(bits: np.ndarray) -> torch.Tensor:
    return dev(bits.view(np.int16)).view(torch.bfloat16)


def gpu_transcode(codes: np.ndarray, e8m0: np.ndarray, in_place: bool = False):
    nt, N, kh = codes.shape
    K = kh * 2
    c = dev(codes)
    s = dev(e8m0)
    co = c if in_place else torch.empty_like(c)
    e4 = torch.empty((nt, N, K // 16), dtype=torch.uint8, device="cuda")
    g = torch.empty(nt, dtype=torch.float32, device="cuda")
    st = torch.empty(nt, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.nvfp4moe_transcode_workspace_size(nt), dtype=torch.uint8, device="cuda")
    status, rep = moe.transcode_mxfp4_to_nvfp4(c, s, nt, N, K, co, e4, g, st, ws, report=True)
    torch.cuda.synchronize()
    return host(co), host(e4), host(g), host(st), rep, status


def nvfp4_weights_from_inputs(d: dict, use_oracle_transcode: bool):
    """NVFP4 checkpoint-layout weights for a workload: direct NVFP4 draws, or the
    transcode of the tiny workload's MXFP4 draws (oracle or GPU transcode)."""
    if "mx" not in d:
        return {k: d[k] for k in ("gate_codes", "gate_sf", "up_codes", "up_sf", "down_codes", "down_sf",
                                  "w_global")}
    out = {}
    globs = []
    for name in ("gate", "up", "down"):
        codes, e8 = d["mx"][name]
        nt, N, kh = codes.shape
        if use_oracle_transcode:
            c2, e4, g, st, _, _ = oracle.transcode(codes, e8, nt, N, kh * 2)
        else:
            c2, e4, g, st, _, _ = gpu_transcode(codes, e8)
        assert np.all(st == 0)
        out[f"{name}_codes"] = c2.reshape(codes.shape)
        out[f"{name}_sf"] = e4
        globs.append(g)
    out["w_global"] = np.stack(globs, axis=1).astype(np.float32)
    return out


class GpuLayer:
    """Packed weights + workspace for one layer shape and mode."""

    def __init__(self, mode: int, w: dict, T: int, n_group: int, topk_group: int, top_k: int):
        self.mode = mode
        self.E, self.I, hh = w["gate_codes"].shape
        self.H = hh * 2
        self.n_group, self.topk_group, self.top_k = n_group, topk_group, top_k
        tw = {k: dev(v) for k, v in w.items()}
        self.packed = torch.empty(moe.moe_packed_weights_size(mode, self.E, self.H, self.I), dtype=torch.uint8,
                                  device="cuda")
        moe.moe_pack_weights(mode, tw["gate_codes"], tw["gate_sf"], tw["up_codes"], tw["up_sf"], tw["down_codes"],
                             tw["down_sf"], tw["w_global"], self.packed)
        torch.cuda.synchronize()
        del tw
        self.resize(T)

    def resize(self, T: int):
        self.T = T
        self.ws = torch.empty(max(1, moe.moe_forward_workspace_size(self.mode, T, self.H, self.I, self.E,
                                                                      self.top_k)), dtype=torch.uint8, device="cuda")

    def forward(self, x: torch.Tensor, logits: torch.Tensor, rsf: float = 2.827, act_global: float = 1.0,
                bias=None, out_fp32: bool = False, renormalize: bool = True, act_global_mid: float | None = None):
        T = x.shape[0]
        if T != self.T:
            self.resize(T)
        out = torch.empty((T, self.H), dtype=torch.float32 if out_fp32 else torch.bfloat16, device="cuda")
        ids = torch.empty((T, self.top_k), dtype=torch.int32, device="cuda")
        wts = torch.empty((T, self.top_k), dtype=torch.float32, device="cuda")
        if act_global_mid is None:
            moe.moe_forward(self.mode, x, logits, bias, self.packed, act_global, T, self.H, self.I, self.E,
                            self.n_group, self.topk_group, self.top_k, rsf, renormalize, self.ws, out, ids, wts)
        else:
            moe.moe_forward_ex(self.mode, x, logits, bias, self.packed, act_global, act_global_mid, T, self.H, self.I,
                               self.E, self.n_group, self.topk_group, self.top_k, rsf, renormalize, self.ws, out, ids,
                               wts)
        moe.nvfp4moe_check_device_status()
        return out, ids, wts


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half a BF16 unit in the last place at |v| (the output format's own rounding)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 8), 0.0)


def compare_layer(got: np.ndarray, ref: np.ndarray, rel_l2: float = REL_L2, max_abs_of_rms: float = MAX_ABS_OF_RMS,
                  bf16_output: bool = False):
    """Spec bounds against the float64 oracle: rel-L2 <= 2e-3 and
    max|err| <= 1e-2 * rms(ref).  A BF16 output is additionally allowed the half
    ulp its own final rounding adds (that rounding is the output dtype, not the
    kernels' arithmetic); FP32 outputs get no allowance."""
    got = got.astype(np.float64)
    err = np.abs(got - ref)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    assert np.all(np.isfinite(got)), "non-finite output"
    assert rel <= rel_l2, f"rel-L2 {rel:.3e} > {rel_l2}"
    allow = max_abs_of_rms * rms + (bf16_half_ulp(ref) if bf16_output else 0.0)
    worst = float(np.max(err - allow))
    assert worst <= 0.0, f"max-abs above the bound by {worst:.3e} (max err {err.max():.3e}, rms {rms:.3e})"
    return rel, float(err.max()) / rms


def oracle_layer(mode: int, d: dict, w: dict, wl, tokens=None, act_global: float = 1.0, renormalize: bool = True,
                 act_global_mid: float | None = None):
    # the compact-scale mode computes W4A16 on the same weight values; W4A8 is the
    # oracle's mode 3 (its numbering matches the library's)
    mode = moe.W4A16 if mode == moe.W4A16C else mode
    return oracle.moe_layer(mode, d["x"], d["logits"], None, w["gate_codes"], w["gate_sf"], w["up_codes"], w["up_sf"],
                            w["down_codes"], w["down_sf"], w["w_global"], act_global, wl.n_group, wl.topk_group,
                            wl.top_k, wl.rsf, renormalize, tokens, act_global_mid=act_global_mid)


def row_units(ids: np.ndarray, E: int, group: int = 128):
    """Cuts every expert's permuted rows (pairs in token order, then slot: the
    library's grouping) into runs of `group` rows.  Returns the unit of every
    (token, slot) pair [T, k], the pairs of each unit (flat pair indices, grouped)
    with each unit's start, and the number of units."""
    T, k = ids.shape
    flat = ids.reshape(-1).astype(np.int64)
    order = np.lexsort((np.arange(T * k), flat))  # by expert, then pair index
    counts = np.bincount(flat, minlength=E)
    starts = np.concatenate([[0], np.cumsum(counts)[:-1]])
    e_sorted = flat[order]
    rank = np.arange(T * k) - starts[e_sorted]
    n_units = (counts + group - 1) // group
    unit_base = np.concatenate([[0], np.cumsum(n_units)[:-1]])
    unit_sorted = unit_base[e_sorted] + rank // group
    unit_of_pair = np.empty(T * k, np.int64)
    unit_of_pair[order] = unit_sorted
    unit_start = np.searchsorted(unit_sorted, np.arange(int(n_units.sum()) + 1))
    return unit_of_pair.reshape(T, k), order, unit_start, int(n_units.sum())


def covering_tokens(ids: np.ndarray, E: int, seed: int, group: int = 128, n_min: int = 512) -> np.ndarray:
    """A seeded token sample for full-size layer checks: every run of `group`
    consecutive permuted rows of every expert (so every 128-row half of every
    256-row tile, the odd halves and each expert's ragged last tile included)
    holds a row of a sampled token, and so does every expert's last row; random
    tokens top the sample up to n_min.  Each token's output depends only on its
    own rows, so the oracle checks exactly the rows the sample holds."""
    T, k = ids.shape
    unit_tok, order, unit_start, n_units = row_units(ids, E, group)
    rng = np.random.default_rng(seed)
    chosen = set()
    covered = np.zeros(n_units, bool)

    def take(t):
        if t not in chosen:
            chosen.add(int(t))
            covered[unit_tok[t]] = True

    counts = np.bincount(ids.reshape(-1), minlength=E)
    for e_last in np.cumsum(counts)[counts > 0] - 1:  # every expert's last row
        take(int(order[e_last]) // k)
    for u in rng.permutation(n_units):
        if not covered[u]:
            take(int(order[rng.integers(unit_start[u], unit_start[u + 1])]) // k)
    rest = np.setdiff1d(np.arange(T), np.fromiter(chosen, np.int64))
    for t in rng.choice(rest, min(len(rest), max(0, n_min - len(chosen))), replace=False):
        take(int(t))
    toks = np.array(sorted(chosen), np.int32)
    assert_units_covered(toks, ids, E, group)
    return toks


def assert_units_covered(toks: np.ndarray, ids: np.ndarray, E: int, group: int = 128):
    """Every `group`-row run of every expert holds a row of one of `toks`."""
    unit_tok, _, _, n_units = row_units(ids, E, group)
    hit = np.zeros(n_units, bool)
    hit[unit_tok[toks].reshape(-1)] = True
    assert hit.all(), f"{int((~hit).sum())} of {n_units} row runs hold no sampled token"


def out_to_f64(out: torch.Tensor) -> np.ndarray:
    return out.float().cpu().numpy().astype(np.float64)


# ---------------------------------------------------------------------------
# the layer checked in two halves, split at the down projection's input
# ---------------------------------------------------------------------------
# The intermediate quantisation turns FP32 SwiGLU outputs into codes.  The GPU's
# gate/up sums are FP32 tensor-core accumulations, the oracle's float64 sums
# rounded once, so the two can take a rounding decision differently where a value
# sits within the GPU arithmetic's error of a boundary; one such flip moves the
# output of a large-scale block by a whole code step.  So the layer is held in
# two halves:
#   1. the GPU's intermediate equals the oracle's quantisation of the oracle's
#      FP32 SwiGLU output, except at decisions whose input lies within the
#      oracle's error bound of an FP32 evaluation (ACC_REL below) of the
#      boundary between the two neighbouring outcomes, and such flips are rare
#      (FLIP_FRACTION);
#   2. the GPU's output equals, within the benchmark spec's bounds, the oracle's down
#      projection and combine of the GPU's own intermediate;
# and the whole-layer bounds against the oracle hold for every token whose
# intermediate took all of the oracle's decisions (at least half of the tokens).
# ACC_REL: error of a gate/up dot product relative to sum |x_h w_h|.  The products
# are exact in FP32 (E2M1 x E2M1 x two E4M3 scales: at most 12 significant bits;
# FP16 x FP16 for W4A16) and the tensor cores sum K/64 (W4A4), K/32 (W4A8) or K/16
# (W4A16) MMA steps into an FP32 accumulator: at most (steps + terms per step)
# roundings of 2^-24 of the sum of magnitudes, 2^-17 at K = 4096 for W4A4, taken
# with a factor 2 margin (2^-16; 2^-15 for the 256-step W4A16 MMA).
ACC_REL = {moe.W4A4: 2.0 ** -16, moe.W4A8: 2.0 ** -16, moe.W4A16: 2.0 ** -15}
# Flipped decisions allowed, as a fraction of all: rare on the coarse NVFP4 and
# MXFP8 grids; BF16's 8-bit grid sits closer to the FP32 accumulation error (a
# flip there moves one element by one BF16 ulp).
FLIP_FRACTION = {moe.W4A4: 1e-3, moe.W4A8: 1e-3, moe.W4A16: 1e-2}
E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
_E4M3 = None


def e4m3_values() -> np.ndarray:
    global _E4M3
    if _E4M3 is None:
        _E4M3 = np.array([oracle.e4m3_value(b) for b in range(256)], np.float64)
    return _E4M3


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """packed NVFP4 bytes [n, K/2] -> signed E2M1 values [n, K] (no scale)"""
    nib = np.stack([codes & 15, codes >> 4], axis=-1).reshape(codes.shape[0], -1)
    return np.where(nib & 8, -1.0, 1.0) * E2M1_MAG[nib & 7]


def gpu_intermediate(layer: "GpuLayer", toks: np.ndarray):
    """The GPU's down-projection input rows of every slot of `toks` (pairs
    t * top_k + j, token-major): (codes, scales) in the checkpoint layout."""
    k, I = layer.top_k, layer.I
    pairs = (toks.astype(np.int64)[:, None] * k + np.arange(k)).reshape(-1).astype(np.int32)
    n = len(pairs)
    row = I // 2 if layer.mode == moe.W4A4 else I if layer.mode == moe.W4A8 else 2 * I
    sc = I // 16 if layer.mode == moe.W4A4 else I // 32 if layer.mode == moe.W4A8 else 0
    codes = torch.empty((n, row), dtype=torch.uint8, device="cuda")
    scales = torch.empty((n, max(sc, 1)), dtype=torch.uint8, device="cuda") if sc else None
    moe.moe_forward_intermediate(layer.mode, layer.T, layer.H, I, layer.E, k, layer.ws, dev(pairs), codes, scales)
    torch.cuda.synchronize()
    return host(codes), (host(scales) if sc else None)


def _within(value, boundary, err):
    """|value| within err of the boundary between two outcomes (err > 0)"""
    return np.abs(np.abs(value) - boundary) <= err


def check_nvfp4_requant(a32: np.ndarray, err: np.ndarray, gs: float, codes: np.ndarray, scales: np.ndarray):
    """Rows [n, I] of FP32 SwiGLU outputs (oracle) with their error bounds against
    the GPU's NVFP4 codes and E4M3 scales; returns the per-row count of flipped
    decisions and the GPU rows' values."""
    n, I = a32.shape
    E4 = e4m3_values()
    oc, osf = oracle.quantize_f32(a32, gs)
    flips = np.zeros(n, np.int64)
    x = a32.astype(np.float64).reshape(n, I // 16, 16)
    ex = err.astype(np.float64).reshape(n, I // 16, 16)
    amax = np.abs(a32.reshape(n, I // 16, 16)).max(-1).astype(np.float64)
    bad_sf = scales != osf
    if bad_sf.any():  # sf = E4M3((amax / 6) / gs): amax moves by at most the block's largest bound
        vg, vo = E4[scales[bad_sf]], E4[osf[bad_sf]]
        adjacent = np.abs(scales[bad_sf].astype(int) - osf[bad_sf].astype(int)) == 1
        ok = adjacent & _within(amax[bad_sf] / 6.0 / gs, (vg + vo) / 2, ex.max(-1)[bad_sf] / 6.0 / gs)
        assert ok.all(), f"{int((~ok).sum())} block scales differ beyond the error bound of a rounding boundary"
        flips += bad_sf.sum(1)
    # codes against the oracle's rounding under the GPU's scale of each block
    d = (E4[scales] * gs)[:, :, None]
    safe = np.where(d > 0, d, 1.0)
    q = np.where(d > 0, x / safe, 0.0)
    got = e2m1_decode(codes).reshape(n, I // 16, 16)
    exp = e2m1_decode(oc).reshape(n, I // 16, 16)
    for r, b in zip(*np.nonzero(bad_sf)):  # the oracle's codes under the GPU's scale where the scales differ
        for i in range(16):
            cq = oracle.e2m1_rne_sat(float(np.float32(x[r, b, i]) / np.float32(E4[scales[r, b]] * gs)))
            exp[r, b, i] = (-1.0 if cq & 8 else 1.0) * E2M1_MAG[cq & 7]
    bad = got != exp
    if bad.any():
        mg, me = np.abs(got[bad]), np.abs(exp[bad])
        ig, ie = np.searchsorted(E2M1_MAG, mg), np.searchsorted(E2M1_MAG, me)
        same_sign = (np.sign(got[bad]) == np.sign(exp[bad])) | (mg == 0) | (me == 0)
        ok = (np.abs(ig - ie) == 1) & same_sign & _within(q[bad], (mg + me) / 2, (ex / safe)[bad])
        assert ok.all(), f"{int((~ok).sum())} intermediate codes differ beyond the error bound of a rounding boundary"
        flips += bad.reshape(n, -1).sum(1)
    assert flips.sum() <= FLIP_FRACTION[moe.W4A4] * n * I, f"{int(flips.sum())} flipped decisions of {n * I}"
    return flips, e2m1_decode(codes) * np.repeat(E4[scales], 16, axis=1) * gs


def check_mxfp8_requant(a32: np.ndarray, err: np.ndarray, codes: np.ndarray, scales: np.ndarray):
    """Rows [n, I] of FP32 SwiGLU outputs (with error bounds) against the GPU's
    MXFP8 codes / E8M0 scales; returns the per-row flips and the GPU rows' values."""
    n, I = a32.shape
    E4 = e4m3_values()
    oc, osf = oracle.quantize_mxfp8_f32(a32)
    flips = np.zeros(n, np.int64)
    x = a32.astype(np.float64).reshape(n, I // 32, 32)
    ex = err.astype(np.float64).reshape(n, I // 32, 32)
    amax = np.abs(x).max(-1)
    bad_sf = scales != osf
    if bad_sf.any():  # X = floor(log2 amax) - 8 moves by one only where amax crosses a power of two
        p2 = 2.0 ** (np.maximum(scales[bad_sf], osf[bad_sf]).astype(np.float64) - 127 + 8)
        ok = (np.abs(scales[bad_sf].astype(int) - osf[bad_sf].astype(int)) == 1) & \
            (np.abs(amax[bad_sf] - p2) <= ex.max(-1)[bad_sf])
        assert ok.all(), f"{int((~ok).sum())} E8M0 scales differ beyond the error bound of a power of two"
        flips += bad_sf.sum(1)
    sg = np.repeat(2.0 ** (scales.astype(np.float64) - 127), 32, axis=1).reshape(n, I // 32, 32)
    got = E4[codes].reshape(n, I // 32, 32)
    exp = E4[oc].reshape(n, I // 32, 32)
    for r, b in zip(*np.nonzero(bad_sf)):
        for i in range(32):
            exp[r, b, i] = E4[oracle.e4m3_rne_satfinite(float(np.float32(x[r, b, i] / sg[r, b, i])))]
    bad = got != exp
    if bad.any():
        y = (x / sg)[bad]
        ok = _within(y, (np.abs(got[bad]) + np.abs(exp[bad])) / 2, (ex / sg)[bad]) & \
            (np.sign(got[bad]) * np.sign(exp[bad]) >= 0)
        assert ok.all(), f"{int((~ok).sum())} intermediate codes differ beyond the error bound of a rounding boundary"
        flips += bad.reshape(n, -1).sum(1)
    assert flips.sum() <= FLIP_FRACTION[moe.W4A8] * n * I, f"{int(flips.sum())} flipped decisions of {n * I}"
    return flips, (got * sg).reshape(n, I)


def check_bf16_round(a32: np.ndarray, err: np.ndarray, codes: np.ndarray):
    """W4A16: the intermediate is the SwiGLU output rounded to BF16; rows [n, I]."""
    n, I = a32.shape
    got = (codes.view(np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(n, I)
    exp_bits = torch.from_numpy(np.ascontiguousarray(a32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    exp = (exp_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    bad = got != exp
    flips = bad.sum(1)
    if bad.any():
        ok = _within(a32.astype(np.float64)[bad], (np.abs(got[bad]) + np.abs(exp[bad])) / 2,
                     err.astype(np.float64)[bad]) & (np.sign(got[bad]) * np.sign(exp[bad]) >= 0)
        assert ok.all(), f"{int((~ok).sum())} BF16 intermediates differ beyond the error bound of a rounding boundary"
    assert flips.sum() <= FLIP_FRACTION[moe.W4A16] * n * I, f"{int(flips.sum())} flipped decisions of {n * I}"
    return flips, got


def check_layer_split(layer: "GpuLayer", d: dict, w: dict, wl, toks: np.ndarray, out32: torch.Tensor,
                      out16: torch.Tensor | None = None, act_global: float = 1.0, act_global_mid: float | None = None):
    """The two-halves check above for the sampled tokens `toks` of the last
    forward call on `layer` (FP32 output `out32`, optionally its BF16 output).
    Returns (flipped decisions, tokens with a flip)."""
    mid = act_global if act_global_mid is None else act_global_mid
    mode = moe.W4A16 if layer.mode == moe.W4A16C else layer.mode
    a32, ids, wts, err = oracle.moe_intermediate(mode, d["x"], d["logits"], None, w["gate_codes"], w["gate_sf"],
                                                 w["up_codes"], w["up_sf"], w["w_global"], act_global, wl.n_group,
                                                 wl.topk_group, wl.top_k, wl.rsf, True, toks, acc_rel=ACC_REL[mode])
    n, k, I = a32.shape
    codes, scales = gpu_intermediate(layer, toks)
    flat, ferr = a32.reshape(n * k, I), err.reshape(n * k, I)
    if mode == moe.W4A4:
        flips, vals = check_nvfp4_requant(flat, ferr, mid, codes, scales)
    elif mode == moe.W4A8:
        flips, vals = check_mxfp8_requant(flat, ferr, codes, scales)
    else:
        flips, vals = check_bf16_round(flat, ferr, codes)
    # 2. the down half from the GPU's own intermediate: the bare bounds
    half = oracle.moe_down(vals.reshape(n, k, I), ids, wts, w["down_codes"], w["down_sf"], w["w_global"])
    got = out_to_f64(out32)[toks]
    compare_layer(got, half)
    if out16 is not None:
        compare_layer(out_to_f64(out16)[toks], half, bf16_output=True)
    # 3. the whole layer against the oracle, on every token whose intermediate
    #    took the oracle's decisions (a flipped token differs by its flips, which
    #    halves 1 and 2 have already accounted for)
    ref = oracle.moe_layer(mode, d["x"], d["logits"], None, w["gate_codes"], w["gate_sf"], w["up_codes"], w["up_sf"],
                           w["down_codes"], w["down_sf"], w["w_global"], act_global, wl.n_group, wl.topk_group,
                           wl.top_k, wl.rsf, True, toks, act_global_mid=mid)
    clean = flips.reshape(n, k).sum(1) == 0
    if mode == moe.W4A16:
        # a BF16 flip moves one element by one BF16 ulp, far inside the bounds:
        # the whole layer is held on every token
        clean[:] = True
    assert clean.mean() >= 0.5, f"only {clean.mean():.3f} of the tokens have no flipped decision"
    compare_layer(got[clean], ref[clean])
    return int(flips.sum()), int((~clean).sum())
