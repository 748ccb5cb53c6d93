"""Pins of the CPU oracle against facts that do not come from the oracle itself:
values printed on the pages (golden files), format definitions, closed forms,
library routines (torch FP8 casts, numpy float64 matmul) and brute force on
tiny inputs.  CPU only."""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from nvfp4_mixture_experts_grouped_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------------------
# codebooks
# ---------------------------------------------------------------------------

def test_e2m1_codebook_matches_pages():
    rows = _rows("e2m1_codebook.txt")
    for code, mag in rows:
        c = int(code)
        assert oracle.e2m1_value(c) == float(mag)
        assert oracle.e2m1_value(c | 8) == -float(mag)
    assert {oracle.e2m1_value(c) for c in range(8)} == {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0}
    # no NaN / Inf encodings, max magnitude 6
    assert max(abs(oracle.e2m1_value(c)) for c in range(16)) == 6.0


def test_e4m3_points_and_structure():
    for byte, val in _rows("e4m3_points.txt"):
        v = oracle.e4m3_value(int(byte, 16))
        if val == "nan":
            assert math.isnan(v)
        else:
            assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val))
    vals = [oracle.e4m3_value(b) for b in range(256)]
    assert sum(math.isnan(v) for v in vals) == 2
    pos = vals[:0x7F]
    assert all(a < b for a, b in zip(pos, pos[1:]))  # monotone over 0x00..0x7E
    assert max(pos) == 448.0
    # every finite value has at most 4 significant bits
    for v in pos[1:]:
        m, e = math.frexp(v)
        assert (m * 16) == int(m * 16)


def test_e4m3_table_matches_torch_fp8():
    # independent library decode of every finite byte
    b = torch.arange(256, dtype=torch.uint8)
    ref = b.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for i in range(256):
        v = oracle.e4m3_value(i)
        if math.isnan(ref[i]):
            assert math.isnan(v)
        else:
            assert v == ref[i]


def test_e8m0():
    assert oracle.e8m0_value(127) == 1.0
    assert oracle.e8m0_value(0) == 2.0 ** -127
    assert oracle.e8m0_value(254) == 2.0 ** 127
    assert math.isnan(oracle.e8m0_value(255))


def test_e4m3_rounding_against_torch_cast():
    rng = np.random.default_rng(7)
    xs = np.concatenate([
        rng.uniform(0, 448, 3000), np.exp(rng.uniform(-14, 6, 3000)),
        # exact midpoints between neighbours
        np.array([(oracle.e4m3_value(c) + oracle.e4m3_value(c + 1)) / 2 for c in range(0, 0x7E)]),
    ]).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_rne_satfinite(float(x)) for x in xs], np.uint8)
    assert np.array_equal(got, ref)
    # satfinite: beyond 448 the result is the largest finite code, not NaN
    for x in (448.0, 460.0, 464.0, 1e6, 3.0e38):
        assert oracle.e4m3_rne_satfinite(x) == 0x7E


def test_e2m1_rounding_golden():
    for ratio, code in _rows("e2m1_rounding.txt"):
        assert oracle.e2m1_rne_sat(float(ratio)) == int(code), ratio


def test_e2m1_rounding_is_nearest():
    rng = np.random.default_rng(3)
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    for x in rng.uniform(-8, 8, 2000).astype(np.float32):
        c = oracle.e2m1_rne_sat(float(x))
        d = abs(abs(float(x)) - mags[c & 7])
        assert d <= np.min(np.abs(abs(float(x)) - mags)) + 0.0


def test_page_count_identities():
    d = {k: int(v) for k, v in _rows("page_counts.txt")}
    # blocks x block size == verified values; values == matrices x 4096*2048
    assert d["scale_blocks"] * d["mxfp4_block"] == d["expert_values"]
    assert d["values_per_matrix"] == 4096 * 2048
    assert d["expert_values"] % d["values_per_matrix"] == 0
    # unit-scale clip point == E2M1 max x E4M3 max
    assert d["unit_scale_clip"] == oracle.e2m1_value(7) * oracle.e4m3_value(0x7E)


# ---------------------------------------------------------------------------
# transcode
# ---------------------------------------------------------------------------

def _mx(num, N, K, lo, hi, seed=11):
    rng = np.random.default_rng(seed)
    return inputs.mxfp4_tensors(rng, num, N, K, lo, hi)


@pytest.mark.parametrize("lo,hi", [(-8, -3), (-20, -3), (0, 17), (-127, -110), (110, 127), (5, 5)])
def test_transcode_decode_equality(lo, hi):
    num, N, K = 3, 8, 128
    codes, e8 = _mx(num, N, K, lo, hi)
    # one all-zero block (codes 0x0 and 0x8 only) in tensor 0
    codes[0, 1, 0:16] = np.array([0x00, 0x88, 0x08, 0x80] * 4, np.uint8)
    c2, e4, g, st, rep, worst = oracle.transcode(codes, e8, num, N, K)
    assert worst == 0 and np.all(st == 0)
    assert np.array_equal(c2, codes)  # codes byte for byte
    assert rep[0] == num * N * K // 32 and rep[1] >= 1
    for t in range(num):
        ref = oracle.decode_mxfp4(codes[t], e8[t], N, K)
        got = oracle.decode_nvfp4(c2[t], e4[t], float(g[t]), N, K)
        assert np.array_equal(ref, got)
        m, _ = math.frexp(float(g[t]))
        assert m == 0.5  # exact power of two
        # two equal scales per 32-block, each a finite exact power of two
        s = e4[t].reshape(-1, 2)
        assert np.all(s[:, 0] == s[:, 1])
        for b in np.unique(s):
            v = oracle.e4m3_value(int(b))
            assert not math.isnan(v)
            if v:
                assert math.frexp(v)[0] == 0.5
    assert e4[0, 1, 0] == 0 and e4[0, 1, 1] == 0  # the all-zero block


def test_transcode_spread_boundary():
    N, K = 4, 64
    codes, e8 = _mx(2, N, K, 0, 0)
    codes[:] = 0x11
    e8[0] = 127
    e8[0, 0, 0] = 127 + 17  # spread 17: representable
    e8[1] = 127
    e8[1, 0, 0] = 127 + 18  # spread 18: not representable
    _, e4, g, st, rep, worst = oracle.transcode(codes, e8, 2, N, K)
    assert list(st) == [0, 1] and worst == 1 and rep[2] == 1
    assert g[1] == 0.0 and np.all(e4[1] == 0)
    assert g[0] == 2.0 ** 9 and e4[0, 0, 0] == 0x78 and e4[0, 0, 2] == 0x01  # 2^8 and 2^-9


def test_transcode_nan_scale_and_empty_tensor():
    codes, e8 = _mx(2, 2, 64, 0, 0)
    e8[0, 0, 1] = 0xFF
    codes[1] = 0x00  # tensor with no non-zero block
    _, e4, g, st, rep, _ = oracle.transcode(codes, e8, 2, 2, 64)
    assert st[0] == 2 and rep[3] == 1
    assert st[1] == 0 and g[1] == 1.0 and np.all(e4[1] == 0)


def test_transcode_adversarial_tensor_of_the_layer_recipe():
    rng = np.random.default_rng(inputs.TRANSCODE_SEED)
    adv_codes, adv_e8 = inputs.mxfp4_tensors(rng, 1, 64, 128, -9, 9)
    adv_codes[0, 0, :16] = 0x77
    adv_codes[0, 1, :16] = 0x77
    adv_e8[0, 0, 0] = 127 - 9
    adv_e8[0, 1, 0] = 127 + 9
    *_, st, rep, worst = oracle.transcode(adv_codes, adv_e8, 1, 64, 128)
    assert st[0] == 1 and worst == 1


# ---------------------------------------------------------------------------
# compact scales (4.125 bits per weight)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("lo,hi", [(-8, -3), (-20, -6), (3, 17), (-9, 8)])
def test_compact_of_a_transcode_is_the_e8m0_exponent_distance(lo, hi):
    # after the transcode every block scale is 2^(k - g); the compact field of a
    # block is then (row max of k) - k, computed here from the E8M0 bytes alone
    num, N, K = 2, 16, 256
    codes, e8 = _mx(num, N, K, lo, hi, seed=5)
    codes[0, 3, 0:16] = 0x80  # an all-zero block (codes +-0)
    codes[1, 7, :] = 0x08     # an all-zero row
    c2, e4, g, st, _, worst = oracle.transcode(codes, e8, num, N, K)
    spread_ok = hi - lo <= 14
    assert worst == 0
    for t in range(num):
        nib, rexp, status, bad = oracle.compact_scales(c2[t], e4[t], N, K)
        k = e8[t].astype(np.int64) - 127
        zero = np.array([[not np.any(codes[t, r, 16 * b:16 * b + 16] & 0x77) for b in range(K // 32)]
                         for r in range(N)])
        gexp = math.frexp(float(g[t]))[1] - 1
        for r in range(N):
            live = ~zero[r]
            if not live.any():
                assert status[r] == 0 and rexp[r] == 0 and np.all(nib[r] == 0xFF)
                continue
            kmax = int(k[r][live].max())
            ok = kmax - int(k[r][live].min()) <= 14
            assert status[r] == (0 if ok else 1)
            if not ok:
                continue
            assert rexp[r] == kmax - gexp
            want = np.where(live, kmax - k[r], 15)
            got = np.stack([nib[r] & 15, nib[r] >> 4], 1).reshape(-1)
            assert np.array_equal(got, want)
        if spread_ok:
            assert bad == 0
        else:
            assert bad == int(np.sum(status))


def test_compact_values_equal_the_mxfp4_values():
    num, N, K = 1, 8, 512
    codes, e8 = _mx(num, N, K, -9, 4, seed=6)
    c2, e4, g, *_ = oracle.transcode(codes, e8, num, N, K)
    nib, rexp, status, bad = oracle.compact_scales(c2[0], e4[0], N, K)
    assert bad == 0
    scale = oracle.compact_decode(nib, rexp, N, K)
    e2m1 = oracle.decode_nvfp4(c2[0], np.full((N, K // 16), 0x38, np.uint8), 1.0, N, K)  # E4M3 0x38 = 1.0
    got = e2m1 * np.repeat(scale, 32, axis=1) * float(g[0])
    assert np.array_equal(got, oracle.decode_mxfp4(codes[0], e8[0], N, K))


def _sf_row(pairs):
    """One row of E4M3 scale bytes: a byte b stands for the pair (b, b)."""
    return np.array([x for p in pairs for x in (p if isinstance(p, tuple) else (p, p))], np.uint8)[None, :]


def test_compact_hand_example():
    # blocks: 2^0 (E4M3 0x38), 2^-3 (0x20), zero (codes +-0), 2^2 (0x48)
    codes = np.full((1, 64), 0x11, np.uint8)
    codes[0, 32:48] = 0x08
    nib, rexp, status, bad = oracle.compact_scales(codes, _sf_row([0x38, 0x20, 0x00, 0x48]), 1, 128)
    assert bad == 0 and status[0] == 0 and rexp[0] == 2
    assert list(nib[0]) == [0x52, 0x0F]  # n = 2, 5 | 15, 0
    assert list(oracle.compact_decode(nib, rexp, 1, 128)[0]) == [1.0, 0.125, 0.0, 4.0]


def test_compact_spread_and_subnormal_boundaries():
    codes = np.full((2, 64), 0x22, np.uint8)
    # row 0: 2^8 (0x78) and 2^-6 (0x08): spread 14, representable; row 1: 2^8 and 2^-7 (subnormal 0x04)
    sf = np.concatenate([_sf_row([0x78, 0x08, 0x78, 0x78]), _sf_row([0x78, 0x04, 0x78, 0x78])])
    nib, rexp, status, bad = oracle.compact_scales(codes, sf, 2, 128)
    assert list(status) == [0, 1] and bad == 1
    assert rexp[0] == 8 and nib[0, 0] == 0xE0
    assert rexp[1] == 0 and np.all(nib[1] == 0xFF)
    # subnormal powers of two are accepted: 2^-9 (0x01), 2^-8 (0x02), 2^-7 (0x04), 2^-6 (0x08)
    nib, rexp, status, _ = oracle.compact_scales(codes[:1], _sf_row([0x01, 0x02, 0x04, 0x08]), 1, 128)
    assert status[0] == 0 and rexp[0] == -6 and list(nib[0]) == [0x23, 0x01]


@pytest.mark.parametrize("pair,zero_codes", [((0x38, 0x30), True), ((0x39, 0x39), True), ((0x7F, 0x7F), True),
                                             ((0xB8, 0xB8), True), ((0x00, 0x00), False), ((0x00, 0x80), True)])
def test_compact_rejections(pair, zero_codes):
    # unequal halves, not a power of two, NaN, negative, zero scale over
    # non-zero codes; and +0 / -0 halves, which have equal value (accepted)
    codes = np.full((1, 64), 0x11, np.uint8)
    if zero_codes:
        codes[0, 0:16] = 0x00
    nib, rexp, status, bad = oracle.compact_scales(codes, _sf_row([pair, 0x38, 0x38, 0x38]), 1, 128)
    expect_ok = pair == (0x00, 0x80)
    assert status[0] == (0 if expect_ok else 1) and bad == (0 if expect_ok else 1)
    if expect_ok:
        assert rexp[0] == 0 and list(nib[0]) == [0x0F, 0x00]


# ---------------------------------------------------------------------------
# sigmoid / exp specification
# ---------------------------------------------------------------------------

def _ulp_diff(a: np.float32, b: float) -> float:
    return abs(float(a) - b) / float(np.spacing(np.float32(abs(b)) if b else np.float32(1e-45)))


def test_exp_and_sigmoid_within_2ulp():
    rng = np.random.default_rng(5)
    xs = np.concatenate([rng.uniform(-20, 20, 4000), rng.normal(0, 1, 2000), np.linspace(-87, 88, 500)])
    for x in xs.astype(np.float32):
        e = oracle.exp_spec(float(x))
        assert _ulp_diff(np.float32(e), math.exp(float(x))) <= 2.0, x
        s = oracle.sigmoid_spec(float(x))
        assert _ulp_diff(np.float32(s), 1.0 / (1.0 + math.exp(-float(x)))) <= 2.0, x
    assert oracle.sigmoid_spec(0.0) == 0.5


# ---------------------------------------------------------------------------
# router
# ---------------------------------------------------------------------------

def _route_bruteforce(logits, bias, ng, tg, k, rsf, renorm):
    T, E = logits.shape
    gsz = E // ng
    ids = np.zeros((T, k), np.int64)
    w = np.zeros((T, k), np.float32)
    for t in range(T):
        s = np.array([oracle.sigmoid_spec(float(v)) for v in logits[t]], np.float32)
        c = s + (bias if bias is not None else np.zeros(E, np.float32))
        c = c.astype(np.float32)
        score = []
        for g in range(ng):
            grp = sorted(c[g * gsz:(g + 1) * gsz], reverse=True)
            score.append(np.float32(grp[0]) + np.float32(grp[1]) if gsz > 1 else np.float32(grp[0]))
        # best subset of tg groups: enumerate all subsets, rank by (sorted scores desc, then indices)
        best = None
        for sub in itertools.combinations(range(ng), tg):
            key = sorted(((-score[g], g) for g in sub))
            # a subset is the top-tg set iff every member outranks every non-member
            others = [(-score[g], g) for g in range(ng) if g not in sub]
            if all(a < b for a in key for b in others):
                best = sub
        cand = [e for e in range(E) if e // gsz in best]
        order = sorted(cand, key=lambda e: (-c[e], e))[:k]
        ids[t] = order
        S = np.float32(0)
        for e in order:
            S = np.float32(S + s[e])
        for j, e in enumerate(order):
            w[t, j] = np.float32(np.float32(s[e] / S) * np.float32(rsf)) if renorm else np.float32(s[e] * np.float32(rsf))
    return ids, w


@pytest.mark.parametrize("E,ng,tg,k", [(16, 4, 2, 4), (32, 8, 4, 8), (12, 3, 2, 3), (8, 8, 3, 3), (8, 1, 1, 2)])
@pytest.mark.parametrize("ties", [False, True])
def test_route_bruteforce(E, ng, tg, k, ties):
    rng = np.random.default_rng(E * 7 + ng)
    T = 24
    if ties:  # few distinct values so that scores and groups tie
        logits = rng.integers(-2, 3, size=(T, E)).astype(np.float32)
    else:
        logits = rng.standard_normal((T, E)).astype(np.float32)
    bias = (rng.standard_normal(E) * 0.1).astype(np.float32) if not ties else None
    for renorm in (True, False):
        ids, w = oracle.route(logits, bias, ng, tg, k, 2.827, renorm)
        rid, rw = _route_bruteforce(logits, bias, ng, tg, k, 2.827, renorm)
        assert np.array_equal(ids, rid)
        assert np.array_equal(w.view(np.uint32), rw.view(np.uint32))


def test_route_nan_bias_ranks_like_minus_inf():
    # The pages never make the selection bias NaN; the reading is that a NaN
    # biased score counts as -inf.  -inf biases are ordinary values, which the
    # brute force ranks directly, so NaN entries must give exactly the -inf
    # routing, and a selection exists even when it has to take such experts.
    rng = np.random.default_rng(5)
    E, ng, tg = 16, 4, 2
    logits = rng.standard_normal((40, E)).astype(np.float32)
    bias = (rng.standard_normal(E) * 0.1).astype(np.float32)
    bad = [1, 5, 6, 7, 12, 13, 14, 15]  # one whole group, most of another, one more
    nan_b, inf_b = bias.copy(), bias.copy()
    nan_b[bad], inf_b[bad] = np.nan, -np.inf
    for k in (4, 8):  # k = 8: both kept groups whole, so -inf experts must be taken
        ids, w = oracle.route(logits, nan_b, ng, tg, k, 2.827)
        ids2, w2 = oracle.route(logits, inf_b, ng, tg, k, 2.827)
        assert np.array_equal(ids, ids2) and np.array_equal(w.view(np.uint32), w2.view(np.uint32))
        rid, rw = _route_bruteforce(logits, inf_b, ng, tg, k, 2.827, True)
        assert np.array_equal(ids, rid) and np.array_equal(w.view(np.uint32), rw.view(np.uint32))
        assert ids.min() >= 0 and ids.max() < E
        assert all(len(set(r)) == k for r in ids.tolist())
    # every bias NaN: all biased scores tie at -inf, so groups and experts go by index
    ids, _ = oracle.route(logits, np.full(E, np.nan, np.float32), ng, tg, 4, 2.827)
    assert np.array_equal(ids, np.tile(np.arange(4, dtype=np.int32), (40, 1)))
    # +inf and -inf in one group: its score (inf + -inf) counts as -inf, so the
    # group ranks as if both were -inf
    pm, mm = bias.copy(), bias.copy()
    pm[[0, 1]], mm[[0, 1]] = [np.inf, -np.inf], [-np.inf, -np.inf]
    pm[2:4], mm[2:4] = -np.inf, -np.inf
    a = oracle.route(logits, pm, ng, tg, 4, 2.827)[0]
    b = oracle.route(logits, mm, ng, tg, 4, 2.827)[0]
    assert not np.any(a // 4 == 0) and np.array_equal(a, b)


def test_route_single_group_is_plain_topk_and_weights_sum():
    rng = np.random.default_rng(99)
    logits = rng.standard_normal((64, 32)).astype(np.float32)
    ids, w = oracle.route(logits, None, 1, 1, 8, 2.827, True)
    s = np.vectorize(oracle.sigmoid_spec, otypes=[np.float32])(logits)
    ref = np.argsort(-s, axis=1, kind="stable")[:, :8]
    assert np.array_equal(ids, ref)
    assert np.allclose(w.sum(1), 2.827, rtol=3e-6)


# ---------------------------------------------------------------------------
# permutation
# ---------------------------------------------------------------------------

def test_permute_is_stable_grouping():
    rng = np.random.default_rng(1)
    logits = rng.standard_normal((50, 16)).astype(np.float32)
    ids, _ = oracle.route(logits, None, 4, 2, 4, 1.0)
    counts, offsets, rop, por = oracle.permute(ids, 16)
    pairs = sorted(range(ids.size), key=lambda p: (ids.reshape(-1)[p], p))
    assert list(por) == pairs
    assert np.array_equal(np.bincount(ids.reshape(-1), minlength=16), counts)
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(rop[por], np.arange(ids.size))


# ---------------------------------------------------------------------------
# quantiser
# ---------------------------------------------------------------------------

def _bits(x):
    return inputs.bf16_bits(np.asarray(x, np.float32))


def test_quantize_midpoints_with_unit_scale():
    # block max 6 -> scale E4M3(1.0) = 0x38; every other entry a golden ratio
    rows = [r for r in _rows("e2m1_rounding.txt") if abs(float(r[0])) <= 6.0]
    ratios = [float(r[0]) for r in rows]
    codes_ref = [int(r[1]) for r in rows]
    for i in range(0, len(ratios), 15):
        blk = [6.0] + ratios[i:i + 15]
        blk += [0.0] * (16 - len(blk))
        ref = [7] + codes_ref[i:i + 15] + [0] * (16 - 1 - len(codes_ref[i:i + 15]))
        c, s = oracle.quantize_f32(np.array([blk], np.float32))
        assert s[0, 0] == 0x38
        got = [(c[0, j // 2] >> (4 * (j % 2))) & 15 for j in range(16)]
        assert got == ref


def test_quantize_saturation_and_zero_block():
    x = np.zeros((2, 32), np.float32)
    x[0, 0] = 3.0e5  # >= 2688: scale saturates at 448, code saturates at 6
    x[0, 1] = -2688.0
    x[0, 2] = 1000.0
    c, s = oracle.quantize_f32(x)
    assert s[0, 0] == 0x7E
    assert c[0, 0] == (0x7 | (0xF << 4))
    assert s[0, 1] == 0 and np.all(c[1] == 0) and np.all(s[1] == 0)
    # 2688 is exactly representable: 6 x 448
    assert oracle.e2m1_value(0xF) * oracle.e4m3_value(s[0, 0]) == -2688.0


def test_e2m1_saturates_for_every_magnitude_above_six():
    # "sat": any |x| > 6 is +-6 (code 7 / 0xF), however large, infinities included
    for x in (6.0001, 7.0, 1e10, 2.0 ** 60, 1e30, 3.4e38, float("inf")):
        assert oracle.e2m1_rne_sat(x) == 0x7, x
        assert oracle.e2m1_rne_sat(-x) == 0xF, x
    # a block whose amax saturates the scale at 448 and whose quotients are ~2^90
    x = np.zeros((1, 16), np.float32)
    x[0, :4] = [2.0 ** 100, 2.0 ** 99, -(2.0 ** 98), 1.0]
    c, s = oracle.quantize_f32(x)
    assert s[0, 0] == 0x7E
    assert c[0, 0] == (0x7 | (0x7 << 4)) and c[0, 1] == 0xF  # codes 7, 7, 0xF, 0


def test_e2m1_keeps_the_sign_of_zero():
    # reading: the sign survives rounding to zero (-0 and small negatives give
    # code 0x8, as the hardware's satfinite conversion does); a block whose
    # scale is zero is all 0x0
    assert oracle.e2m1_rne_sat(0.0) == 0x0
    assert oracle.e2m1_rne_sat(-0.0) == 0x8
    assert oracle.e2m1_rne_sat(-0.2) == 0x8
    x = np.zeros((2, 16), np.float32)
    x[0, 0], x[0, 1], x[0, 2] = 6.0, -0.0, 0.0
    x[1, :] = -0.0
    c, s = oracle.quantize_f32(x)
    assert s[0, 0] == 0x38  # E4M3 1.0
    assert c[0, 0] == (0x7 | (0x8 << 4)) and c[0, 1] == 0x00
    assert s[1, 0] == 0 and np.all(c[1] == 0)


def test_quantize_roundtrip_of_representable_blocks():
    rng = np.random.default_rng(8)
    for _ in range(200):
        sfb = int(rng.integers(0x08, 0x70))
        sfv = oracle.e4m3_value(sfb)
        q = rng.integers(0, 16, 16)
        q[0] = 7  # block max = 6 * scale, so the scale is recovered exactly
        x = np.array([oracle.e2m1_value(int(v)) * sfv for v in q], np.float32)
        c, s = oracle.quantize_f32(x[None, :])
        assert s[0, 0] == sfb
        dec = [oracle.e2m1_value(int((c[0, j // 2] >> (4 * (j % 2))) & 15)) * sfv for j in range(16)]
        assert np.array_equal(np.array(dec, np.float32), x)


def test_quantize_scale_against_torch_fp8():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-6, 6, (64, 1)))).astype(np.float32)
    c, s = oracle.quantize_f32(x)
    amax = np.abs(x.reshape(64, 16, 16)).max(-1)
    ref = torch.from_numpy((amax / np.float32(6)).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(s, ref)


@pytest.mark.parametrize("gs", [0.37, 3.0, 1.0 / 64, 116.0])
def test_quantize_scale_with_a_global_against_torch_fp8(gs):
    # sf = E4M3((amax / 6) / gs): both divisions in IEEE FP32, the cast by torch
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-4, 4, (64, 1))) * gs).astype(np.float32)
    c, s = oracle.quantize_f32(x, gs)
    amax = np.abs(x.reshape(64, 16, 16)).max(-1)
    v = (amax / np.float32(6)).astype(np.float32) / np.float32(gs)
    assert np.all(v < 448)  # inside the cast's finite range
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(s, ref)


@pytest.mark.parametrize("j", [-5, -1, 3, 7])
def test_quantize_power_of_two_global_is_equivariant(j):
    # scaling the block and the global by the same 2^j changes neither a scale
    # byte nor a code: (amax 2^j / 6) / 2^j and x 2^j / (sf 2^j) are exact moves
    rng = np.random.default_rng(6 + j)
    x = (rng.standard_normal((32, 128)) * np.exp(rng.uniform(-3, 3, (32, 1)))).astype(np.float32)
    c1, s1 = oracle.quantize_f32(x, 1.0)
    cj, sj = oracle.quantize_f32(np.ldexp(x, j).astype(np.float32), 2.0 ** j)
    assert np.array_equal(s1, sj) and np.array_equal(c1, cj)


# ---------------------------------------------------------------------------
# GEMM exactness and the layer
# ---------------------------------------------------------------------------

def test_fp4_products_exact_in_fp32():
    rng = np.random.default_rng(0)
    lut = np.array([oracle.e2m1_value(c) for c in range(16)])
    for K in (16, 64, 4096):
        a = lut[rng.integers(0, 16, (8, K))]
        b = lut[rng.integers(0, 16, (8, K))]
        r64 = a @ b.T
        r32 = a.astype(np.float32) @ b.T.astype(np.float32)
        assert np.array_equal(r64, r32.astype(np.float64))
        assert np.all(np.mod(r64 * 4, 1) == 0)  # multiples of 0.25


def _np_decode(codes, sf, glob):
    """Independent numpy decode ([N, K/2] codes, [N, K/16] E4M3) via torch FP8."""
    lut = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])
    lo = lut[codes & 15]
    hi = lut[codes >> 4]
    vals = np.stack([lo, hi], -1).reshape(codes.shape[0], -1)
    s = torch.from_numpy(sf).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return vals * np.repeat(s, 16, axis=1) * float(glob)


@pytest.mark.parametrize("mode", [0, 1])
def test_layer_reduces_to_dense_swiglu(mode):
    rng = np.random.default_rng(21 + mode)
    T, H, I = 5, 64, 32
    gc, gs, _ = inputs.nvfp4_tensors(rng, 1, I, H)
    uc, us, _ = inputs.nvfp4_tensors(rng, 1, I, H)
    dc, ds, _ = inputs.nvfp4_tensors(rng, 1, H, I)
    wg = np.array([[0.5, 0.25, 2.0]], np.float32)
    x = inputs.activations(rng, T, H)
    logits = rng.standard_normal((T, 1)).astype(np.float32)
    out = oracle.moe_layer(mode, x, logits, None, gc, gs, uc, us, dc, ds, wg, 1.0, 1, 1, 1, 1.0)
    Wg = _np_decode(gc[0], gs[0], 0.5)
    Wu = _np_decode(uc[0], us[0], 0.25)
    Wd = _np_decode(dc[0], ds[0], 2.0)
    xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    if mode == 1:
        qc, qs = oracle.quantize_bf16(x)
        xf = _np_decode(qc, qs, 1.0)
    G = xf @ Wg.T
    U = xf @ Wu.T
    A = G / (1 + np.exp(-G)) * U
    if mode == 1:
        ac, as_ = oracle.quantize_f32(A.astype(np.float32))
        A = _np_decode(ac, as_, 1.0)
    else:
        A = torch.from_numpy(A.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    Y = A @ Wd.T
    assert np.allclose(out, Y, rtol=1e-12, atol=1e-12 * np.abs(Y).max())


@pytest.mark.parametrize("gs_in,gs_mid", [(0.37, 2.5), (116.0, 1.0), (1.0, 0.03125)])
def test_layer_separate_input_and_intermediate_scales(gs_in, gs_mid):
    # "Why a unit activation scale": calibrated per-layer scales, the down input's
    # capped at 2688, or unit.  Dense reduction (E=1, k=1, rsf=1) against the
    # quantiser pins: x quantised with gs_in, the SwiGLU output with gs_mid.
    rng = np.random.default_rng(41)
    T, H, I = 4, 64, 32
    gc, gs, _ = inputs.nvfp4_tensors(rng, 1, I, H)
    uc, us, _ = inputs.nvfp4_tensors(rng, 1, I, H)
    dc, ds, _ = inputs.nvfp4_tensors(rng, 1, H, I)
    wg = np.array([[0.5, 0.25, 2.0]], np.float32)
    x = inputs.activations(rng, T, H, outliers=True)
    logits = rng.standard_normal((T, 1)).astype(np.float32)
    out = oracle.moe_layer(1, x, logits, None, gc, gs, uc, us, dc, ds, wg, gs_in, 1, 1, 1, 1.0,
                           act_global_mid=gs_mid)
    qc, qs = oracle.quantize_bf16(x, gs_in)
    xf = _np_decode(qc, qs, gs_in)
    G = xf @ _np_decode(gc[0], gs[0], 0.5).T
    U = xf @ _np_decode(uc[0], us[0], 0.25).T
    A = G / (1 + np.exp(-G)) * U
    ac, as_ = oracle.quantize_f32(A.astype(np.float32), gs_mid)
    Y = _np_decode(ac, as_, gs_mid) @ _np_decode(dc[0], ds[0], 2.0).T
    assert np.allclose(out, Y, rtol=1e-12, atol=1e-12 * np.abs(Y).max())
    # the two scales are not interchangeable
    if gs_in != gs_mid:
        swapped = oracle.moe_layer(1, x, logits, None, gc, gs, uc, us, dc, ds, wg, gs_mid, 1, 1, 1, 1.0,
                                   act_global_mid=gs_in)
        assert not np.allclose(swapped, Y, rtol=1e-6)


def test_layer_combines_two_experts_with_routing_weights():
    rng = np.random.default_rng(33)
    T, H, I, E = 4, 32, 16, 2
    gc, gs, _ = inputs.nvfp4_tensors(rng, E, I, H)
    uc, us, _ = inputs.nvfp4_tensors(rng, E, I, H)
    dc, ds, _ = inputs.nvfp4_tensors(rng, E, H, I)
    wg = np.ones((E, 3), np.float32)
    x = inputs.activations(rng, T, H)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    both = oracle.moe_layer(0, x, logits, None, gc, gs, uc, us, dc, ds, wg, 1.0, 2, 2, 2, 2.827)
    ids, w = oracle.route(logits, None, 2, 2, 2, 2.827)
    xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    for t in range(T):
        acc = np.zeros(H)
        for j in range(2):
            e = ids[t, j]
            G = _np_decode(gc[e], gs[e], 1) @ xf[t]
            U = _np_decode(uc[e], us[e], 1) @ xf[t]
            A = G / (1 + np.exp(-G)) * U
            A = torch.from_numpy(A.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
            acc += float(w[t, j]) * (_np_decode(dc[e], ds[e], 1) @ A)
        assert np.allclose(both[t], acc, rtol=1e-12, atol=1e-12 * np.abs(acc).max())


# ---------------------------------------------------------------------------
# MXFP8 activations ("MiMo-V2.6-Flash-MOPD on one RTX PRO 6000", "Speed v5.2":
# E4M3 with a power-of-two scale per 32 values; OCP scale choice)
# ---------------------------------------------------------------------------

def _mx8_reference(x: np.ndarray):
    """Independent MXFP8 of FP32 rows with numpy frexp and torch's E4M3 cast."""
    M, K = x.shape
    blocks = x.astype(np.float64).reshape(M, K // 32, 32)
    amax = np.abs(blocks).max(-1)
    X = np.where(amax > 0, np.frexp(amax)[1] - 1 - 8, -127).clip(-127, 127)
    scaled = blocks * np.exp2(-X.astype(np.float64))[..., None]
    codes = torch.from_numpy(np.clip(scaled, -448, 448).reshape(M, K)).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.numpy(), (X + 127).astype(np.uint8)


def _mx8_decode(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    v = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return v * np.repeat(np.exp2(scales.astype(np.float64) - 127), 32, axis=1)


def test_mxfp8_matches_frexp_and_torch_e4m3():
    rng = np.random.default_rng(12)
    x = (rng.standard_normal((48, 256)) * np.exp(rng.uniform(-30, 30, (48, 1)))).astype(np.float32)
    x[3, 32:64] = 0.0                  # zero block
    x[4, 5] = 3.0e38                   # near the FP32 maximum
    x[5, 0:32] = 1e-42                 # FP32 subnormals
    x[6, 64:96] = np.float32(2.0 ** -3)  # power-of-two amax
    codes, scales = oracle.quantize_mxfp8_f32(x)
    rc, rs = _mx8_reference(x)
    assert np.array_equal(scales, rs)
    same = (codes == rc) | ((codes & 0x7F) == 0) & ((rc & 0x7F) == 0)  # +-0 either way
    assert same.all()
    assert scales[3, 1] == 0 and np.all(codes[3, 32:64] & 0x7F == 0)


def test_mxfp8_hand_values():
    x = np.zeros((1, 32), np.float32)
    x[0, :6] = [1.0, 0.3, -1.9, 2.0 ** -9, 1.875, 0.0]
    codes, scales = oracle.quantize_mxfp8_f32(x)
    # amax 1.9: X = 0 - 8, scale byte 119; elements x * 256
    assert scales[0, 0] == 119
    assert codes[0, 0] == 0x78          # 256 = 2^8
    assert codes[0, 1] == 0x6A          # 76.8 -> 80 = 1.25 * 2^6
    assert codes[0, 2] == 0xFE          # -486.4 saturates to -448
    assert codes[0, 3] == 0x30          # 2^-9 * 2^8 = 2^-1
    assert codes[0, 4] == 0x7E          # 480 saturates to 448
    assert codes[0, 5] == 0x00


def test_layer_w4a8_reduces_to_dense_swiglu():
    # mode 3: MXFP8 layer input and SwiGLU output, NVFP4 weights (E=1, k=1, rsf=1)
    rng = np.random.default_rng(25)
    T, H, I = 5, 64, 64
    gc, gs, _ = inputs.nvfp4_tensors(rng, 1, I, H)
    uc, us, _ = inputs.nvfp4_tensors(rng, 1, I, H)
    dc, ds, _ = inputs.nvfp4_tensors(rng, 1, H, I)
    wg = np.array([[0.5, 0.25, 2.0]], np.float32)
    x = inputs.activations(rng, T, H, outliers=True)
    logits = rng.standard_normal((T, 1)).astype(np.float32)
    out = oracle.moe_layer(3, x, logits, None, gc, gs, uc, us, dc, ds, wg, 1.0, 1, 1, 1, 1.0)
    xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(torch.float32).numpy()
    xc, xs = _mx8_reference(xf)
    xq = _mx8_decode(xc, xs)
    G = xq @ _np_decode(gc[0], gs[0], 0.5).T
    U = xq @ _np_decode(uc[0], us[0], 0.25).T
    A = G / (1 + np.exp(-G)) * U
    ac, as_ = _mx8_reference(A.astype(np.float32))
    Y = _mx8_decode(ac, as_) @ _np_decode(dc[0], ds[0], 2.0).T
    assert np.allclose(out, Y, rtol=1e-12, atol=1e-12 * np.abs(Y).max())
    # and it is not the W4A4 or W4A16 layer
    assert not np.allclose(out, oracle.moe_layer(1, x, logits, None, gc, gs, uc, us, dc, ds, wg, 1.0, 1, 1, 1, 1.0),
                           rtol=1e-6)
# ---------------------------------------------------------------------------
# router projection ("MiMo-V2.6-Flash-MOPD on one RTX PRO 6000", "What makes it
# fast": the router's matmul; routers kept in F32 per the mixed-quant GGUF
# page's precision table)
# ---------------------------------------------------------------------------
def _bf16_bits(a):
    return inputs.bf16_bits(np.asarray(a, np.float32))


def test_router_logits_one_hot_rows_copy_the_input():
    rng = np.random.default_rng(7)
    T, H, E = 5, 64, 48
    x = _bf16_bits(rng.standard_normal((T, H)).astype(np.float32) * 3)
    w = np.zeros((E, H), np.float32)
    w[np.arange(E), np.arange(E)] = 1.0
    logits, mag = oracle.router_logits(x, w)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(logits, xf[:, :E])
    assert np.array_equal(mag, np.abs(xf[:, :E]).astype(np.float64))


def test_router_logits_exact_integers():
    rng = np.random.default_rng(8)
    T, H, E = 7, 256, 16
    xi = rng.integers(-8, 9, size=(T, H))
    wi = rng.integers(-50, 51, size=(E, H))
    logits, mag = oracle.router_logits(_bf16_bits(xi), wi.astype(np.float32))
    ref = xi.astype(np.int64) @ wi.astype(np.int64).T  # |sum| < 2^24: exact in FP32
    assert np.array_equal(logits, ref.astype(np.float32))
    assert np.array_equal(mag, np.abs(xi)[:, None, :].__mul__(np.abs(wi)[None, :, :]).sum(-1).astype(np.float64))


def test_router_logits_match_float64_matmul():
    rng = np.random.default_rng(9)
    T, H, E = 6, 4096, 32
    x = _bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    w = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    logits, _ = oracle.router_logits(x, w)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = xf @ w.astype(np.float64).T
    # the only difference is the float64 summation order: at most one FP32 rounding apart
    ulp = np.spacing(np.abs(ref).astype(np.float32))
    assert np.all(np.abs(logits.astype(np.float64) - ref) <= ulp)


# ---------------------------------------------------------------------------
# the layer split at the down projection's input
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [0, 1, 3])
def test_layer_split_at_the_intermediate_reproduces_the_layer(mode):
    # The split oracle (SwiGLU output before the intermediate quantisation, then
    # the down projection and combine from given down inputs) is what the GPU
    # checks use to hold the two halves of the layer separately; requantising its
    # FP32 intermediate with the oracle's own quantiser and feeding it back must
    # give the whole-layer oracle bit for bit, in every mode.
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl, T=24)
    w = {}
    gl = []
    for name in ("gate", "up", "down"):
        c, e8 = d["mx"][name]
        nt, N, kh = c.shape
        c2, e4, g, st, _, _ = oracle.transcode(c, e8, nt, N, kh * 2)
        w[name + "_codes"], w[name + "_sf"] = c2.reshape(c.shape), e4
        gl.append(g)
    w["w_global"] = np.stack(gl, 1).astype(np.float32)
    g_in, g_mid = 0.75, 0.5
    toks = np.array([3, 0, 23, 11, 11, 7], np.int32)
    a32, ids, wts = oracle.moe_intermediate(mode, d["x"], d["logits"], None, w["gate_codes"], w["gate_sf"],
                                            w["up_codes"], w["up_sf"], w["w_global"], g_in, wl.n_group,
                                            wl.topk_group, wl.top_k, wl.rsf, True, toks)
    ri, rw = oracle.route(d["logits"][toks], None, wl.n_group, wl.topk_group, wl.top_k, wl.rsf)
    assert np.array_equal(ids, ri) and np.array_equal(wts.view(np.uint32), rw.view(np.uint32))
    n, k, I = a32.shape
    flat = a32.reshape(n * k, I)
    if mode == 1:
        c, s = oracle.quantize_f32(flat, g_mid)
        vals = oracle.decode_nvfp4(c, s, g_mid, n * k, I)
    elif mode == 3:
        c, s = oracle.quantize_mxfp8_f32(flat)
        vals = oracle.decode_mxfp8(c, s)
    else:
        bits = np.array([oracle.float_to_bf16(float(v)) for v in flat.reshape(-1)], np.uint32)
        vals = (bits << 16).view(np.float32).astype(np.float64).reshape(n * k, I)
    out = oracle.moe_down(vals.reshape(n, k, I), ids, wts, w["down_codes"], w["down_sf"], w["w_global"])
    ref = oracle.moe_layer(mode, d["x"], d["logits"], None, w["gate_codes"], w["gate_sf"], w["up_codes"],
                           w["up_sf"], w["down_codes"], w["down_sf"], w["w_global"], g_in, wl.n_group,
                           wl.topk_group, wl.top_k, wl.rsf, True, toks, act_global_mid=g_mid)
    assert np.array_equal(out.view(np.uint64), ref.view(np.uint64))


def test_intermediate_error_bound_covers_an_fp32_evaluation():
    # The bound the split checks allow flips within must hold for an FP32
    # evaluation of the same SwiGLU outputs: gate and up as float32 dot products
    # of the decoded operands (a plain float32 matmul, its own summation order),
    # SiLU and the product in float32.  At K = 256 a float32 sum errs by at most
    # 256 * 2^-24 = 2^-16 of the sum of magnitudes, so 2^-16 is the bound's
    # accumulation term here.
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl, T=16)
    w = {}
    gl = []
    for name in ("gate", "up", "down"):
        c, e8 = d["mx"][name]
        nt, N, kh = c.shape
        c2, e4, g, st, _, _ = oracle.transcode(c, e8, nt, N, kh * 2)
        w[name + "_codes"], w[name + "_sf"] = c2.reshape(c.shape), e4
        gl.append(g)
    w["w_global"] = np.stack(gl, 1).astype(np.float32)
    toks = np.arange(16, dtype=np.int32)
    a32, ids, wts, err = oracle.moe_intermediate(0, d["x"], d["logits"], None, w["gate_codes"], w["gate_sf"],
                                                 w["up_codes"], w["up_sf"], w["w_global"], 1.0, wl.n_group,
                                                 wl.topk_group, wl.top_k, wl.rsf, True, toks, acc_rel=2.0 ** -16)
    H, I = wl.H, wl.I
    x = (d["x"][toks].astype(np.uint32) << 16).view(np.float32)
    worst = 0.0
    for t in range(16):
        for j in range(wl.top_k):
            e = ids[t, j]
            wg = oracle.decode_nvfp4(w["gate_codes"][e], w["gate_sf"][e], w["w_global"][e, 0], I, H).astype(np.float32)
            wu = oracle.decode_nvfp4(w["up_codes"][e], w["up_sf"][e], w["w_global"][e, 1], I, H).astype(np.float32)
            g32 = wg @ x[t]
            u32 = wu @ x[t]
            a = (g32 / (np.float32(1) + np.exp(-g32))) * u32
            dev = np.abs(a.astype(np.float64) - a32[t, j])
            assert np.all(dev <= err[t, j]), (t, j, float((dev - err[t, j]).max()))
            worst = max(worst, float((dev / err[t, j]).max()))
    assert worst > 0.0
