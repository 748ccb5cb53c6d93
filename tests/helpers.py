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


def out_to_f64(out: torch.Tensor) -> np.ndarray:
    return out.float().cpu().numpy().astype(np.float64)
