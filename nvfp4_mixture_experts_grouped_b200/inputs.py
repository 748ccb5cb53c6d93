"""Seeded synthetic inputs shaped like the pages' workloads.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no transcode, routing, quantisation or GEMM).  The same
bytes feed the CUDA path and the CPU oracle.

Workloads (MiMo-V2.6-Flash MoE layer shapes: hidden 4096, expert
intermediate 2048, 256 routed experts in 8 groups, top-8, scaling 2.827 --
"MiMo-V2.6-Flash -- REAP-50", "Model Summary"; the 128-expert pruned variant
keeps 16 experts per group):

* ``tiny``      T=32, H=256, I=128, E=16, 4 groups x 4, keep 2, top-4; MXFP4
                weights with E8M0 exponents uniform in [-8, -3]; W4A4.
* ``transcode`` one layer of MXFP4 expert weights (256 experts x gate, up
                [2048, 4096] and down [4096, 2048]); per-expert exponent window
                of width w ~ U{0..17} placed at base ~ U{-20 .. 10-w}; plus one
                adversarial tensor whose spread is 18 octaves.
* ``decode``    T=16, H=4096, I=2048, E=256, 8x32 groups, keep 4, top-8; NVFP4
                weights: codes uniform over the 16 codes, E4M3 scale bytes
                uniform over the codes whose values lie in [2^-6, 2^2] (eight
                per octave: a discrete log-uniform draw), global 2^-4; W4A16.
* ``prefill``   as ``decode`` with T=8192 and 0.01% of the activations replaced
                by +-U(1e3, 3e5) outliers; W4A4.
* ``skewed``    T=65536, E=128 (8 groups x 16), otherwise as ``prefill``; router
                logits N(0,1) plus a per-expert Zipf(1.1) bias -1.1*ln(r_e), r a
                seeded permutation of 1..E.
* ``decode_pow2`` as ``decode``, but with the scale structure of a transcoded
                MXFP4 checkpoint: per 32 codes one E4M3 byte drawn uniformly
                from the zero-mantissa codes 0x08, 0x10, .., 0x48 (2^-6 .. 2^2),
                the same byte for both 16-code halves; W4A16 with compact
                scales.
* ``prefill_pow2`` as ``prefill`` (outliers included) with the weights of
                ``decode_pow2``; W4A8 (MXFP8 activations).

Activations are BF16 N(0,1) (drawn in float32, stored as BF16 bit patterns);
router logits are float32 N(0,1).  Seeds are 1234 + the workload's index.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    T: int
    H: int
    I: int
    E: int
    n_group: int
    topk_group: int
    top_k: int
    rsf: float
    mode: int  # 0 = W4A16, 1 = W4A4, 2 = W4A16 with compact scales, 3 = W4A8
    weights: str  # "mxfp4_tiny" | "nvfp4" | "nvfp4_pow2"
    outliers: bool = False
    zipf: bool = False

    @property
    def seed(self) -> int:
        return 1234 + self.index


WORKLOADS = {
    "tiny": Workload("tiny", 0, 32, 256, 128, 16, 4, 2, 4, 2.827, 1, "mxfp4_tiny"),
    "decode": Workload("decode", 2, 16, 4096, 2048, 256, 8, 4, 8, 2.827, 0, "nvfp4"),
    "prefill": Workload("prefill", 3, 8192, 4096, 2048, 256, 8, 4, 8, 2.827, 1, "nvfp4", outliers=True),
    "skewed": Workload("skewed", 4, 65536, 4096, 2048, 128, 8, 4, 8, 2.827, 1, "nvfp4", outliers=True, zipf=True),
    "decode_pow2": Workload("decode_pow2", 5, 16, 4096, 2048, 256, 8, 4, 8, 2.827, 2, "nvfp4_pow2"),
    "prefill_pow2": Workload("prefill_pow2", 6, 8192, 4096, 2048, 256, 8, 4, 8, 2.827, 3, "nvfp4_pow2",
                             outliers=True),
}

TRANSCODE_SEED = 1234 + 1


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> BF16 bit patterns (uint16), round to nearest even, via torch."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def activations(rng: np.random.Generator, T: int, H: int, outliers: bool = False) -> np.ndarray:
    """BF16 bit patterns [T, H]: N(0,1), optionally with 0.01% +-U(1e3, 3e5) entries."""
    x = rng.standard_normal((T, H), dtype=np.float32)
    if outliers:
        n = max(1, (T * H) // 10000)
        pos = rng.choice(T * H, size=n, replace=False)
        sign = np.where(rng.random(n) < 0.5, -1.0, 1.0).astype(np.float32)
        mag = rng.uniform(1e3, 3e5, size=n).astype(np.float32)
        x.reshape(-1)[pos] = sign * mag
    return bf16_bits(x)


def router_logits(rng: np.random.Generator, T: int, E: int, zipf: bool = False) -> np.ndarray:
    lg = rng.standard_normal((T, E), dtype=np.float32)
    if zipf:
        r = rng.permutation(E).astype(np.float64) + 1.0
        lg = (lg + (-1.1 * np.log(r)).astype(np.float32)[None, :]).astype(np.float32)
    return lg


def router_weights(rng: np.random.Generator, E: int, H: int) -> np.ndarray:
    """FP32 router rows [E, H] ~ N(0, 1/H): with N(0,1) hidden rows the logits are
    ~N(0,1), the scale of the logit recipe above."""
    return (rng.standard_normal((E, H), dtype=np.float32) / np.float32(np.sqrt(H))).astype(np.float32)


def random_codes(rng: np.random.Generator, shape) -> np.ndarray:
    """Packed E2M1 bytes: both nibbles uniform over all 16 codes."""
    return rng.integers(0, 256, size=shape, dtype=np.uint8)


def mxfp4_tensors(rng: np.random.Generator, num: int, N: int, K: int, exp_lo, exp_hi):
    """MXFP4 tensors [num, N, K]: codes [num, N, K/2], E8M0 [num, N, K/32].

    exp_lo/exp_hi are ints or per-tensor arrays: exponents uniform in [lo, hi]."""
    codes = random_codes(rng, (num, N, K // 2))
    lo = np.broadcast_to(np.asarray(exp_lo, np.int64), (num,)).reshape(num, 1, 1)
    hi = np.broadcast_to(np.asarray(exp_hi, np.int64), (num,)).reshape(num, 1, 1)
    u = rng.random((num, N, K // 32))
    ex = lo + np.floor(u * (hi - lo + 1)).astype(np.int64)
    return codes, (ex + 127).astype(np.uint8)


def nvfp4_tensors(rng: np.random.Generator, num: int, N: int, K: int):
    """NVFP4 tensors [num, N, K]: codes, E4M3 scale bytes in [0x08, 0x48] (values
    2^-6 .. 2^2), and the global scale 2^-4 per tensor."""
    codes = random_codes(rng, (num, N, K // 2))
    scales = rng.integers(0x08, 0x49, size=(num, N, K // 16), dtype=np.uint8)
    glob = np.full(num, 2.0 ** -4, np.float32)
    return codes, scales, glob


def nvfp4_pow2_tensors(rng: np.random.Generator, num: int, N: int, K: int):
    """NVFP4 tensors [num, N, K] whose two scales per 32 codes are one E4M3 byte
    drawn from the zero-mantissa codes 0x08 .. 0x48 (values 2^-6 .. 2^2); codes
    uniform; global 2^-4 per tensor."""
    codes = random_codes(rng, (num, N, K // 2))
    pick = rng.integers(1, 10, size=(num, N, K // 32), dtype=np.uint8) * np.uint8(8)
    scales = np.repeat(pick, 2, axis=2)
    glob = np.full(num, 2.0 ** -4, np.float32)
    return codes, scales, glob


def transcode_layer(rng: np.random.Generator, E: int = 256, H: int = 4096, I: int = 2048):
    """One MoE layer of MXFP4 expert weights plus one adversarial tensor.

    Returns dict with gate/up codes+e8m0 [E, I, H..], down [E, H, I..] and the
    adversarial tensor (shape [I, H]) whose exponents span exactly 18 octaves."""
    w = rng.integers(0, 18, size=E)
    base = np.array([rng.integers(-20, 10 - wi + 1) for wi in w])
    gate = mxfp4_tensors(rng, E, I, H, base, base + w)
    up = mxfp4_tensors(rng, E, I, H, base, base + w)
    down = mxfp4_tensors(rng, E, H, I, base, base + w)
    adv_codes, adv_e8m0 = mxfp4_tensors(rng, 1, I, H, -9, 9)
    # pin both ends of the 18-octave spread on non-zero blocks
    adv_codes[0, 0, :16] = 0x77
    adv_codes[0, 1, :16] = 0x77
    adv_e8m0[0, 0, 0] = 127 - 9
    adv_e8m0[0, 1, 0] = 127 + 9
    return {"gate": gate, "up": up, "down": down, "adversarial": (adv_codes, adv_e8m0), "window": (base, w)}


def moe_inputs(wl: Workload, T: int | None = None):
    """All inputs of one layer call for workload ``wl`` (optionally with another T).

    Weights are returned in the checkpoint ("linear") layout:
      gate/up codes [E, I, H/2], scales [E, I, H/16]; down codes [E, H, I/2],
      scales [E, H, I/16]; w_global [E, 3] (gate, up, down).
    For the tiny workload the weights are MXFP4 (``mx`` key) and must be
    transcoded first; the NVFP4 arrays are then None."""
    rng = np.random.default_rng(wl.seed)
    T = wl.T if T is None else T
    E, H, I = wl.E, wl.H, wl.I
    out = {"wl": wl, "T": T}
    if wl.weights == "mxfp4_tiny":
        out["mx"] = {
            "gate": mxfp4_tensors(rng, E, I, H, -8, -3),
            "up": mxfp4_tensors(rng, E, I, H, -8, -3),
            "down": mxfp4_tensors(rng, E, H, I, -8, -3),
        }
    else:
        gen = nvfp4_pow2_tensors if wl.weights == "nvfp4_pow2" else nvfp4_tensors
        gc, gs, gg = gen(rng, E, I, H)
        uc, us, ug = gen(rng, E, I, H)
        dc, ds, dg = gen(rng, E, H, I)
        out.update(gate_codes=gc, gate_sf=gs, up_codes=uc, up_sf=us, down_codes=dc, down_sf=ds,
                   w_global=np.stack([gg, ug, dg], axis=1).astype(np.float32))
    out["x"] = activations(rng, T, H, wl.outliers)
    out["logits"] = router_logits(rng, T, E, wl.zipf)
    return out
