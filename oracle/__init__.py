"""CPU oracle for the NVFP4 mixture-of-experts hot path (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it.

The arithmetic lives in ``nvfp4_oracle.c`` (plain C, float64 for the layer,
IEEE FP32 for the integer-producing decisions); this module only compiles it
with gcc and marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB = os.path.join(_HERE, "libnvfp4_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP over tokens for the layer)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB)
        L = _lib
        L.orc_e2m1_value.restype = ctypes.c_double
        L.orc_e2m1_value.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_value.restype = ctypes.c_double
        L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        L.orc_e8m0_value.restype = ctypes.c_double
        L.orc_e8m0_value.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_rne_satfinite.restype = ctypes.c_uint8
        L.orc_e4m3_rne_satfinite.argtypes = [ctypes.c_float]
        L.orc_e2m1_rne_sat.restype = ctypes.c_uint8
        L.orc_e2m1_rne_sat.argtypes = [ctypes.c_float]
        L.orc_exp_spec.restype = ctypes.c_float
        L.orc_exp_spec.argtypes = [ctypes.c_float]
        L.orc_sigmoid_spec.restype = ctypes.c_float
        L.orc_sigmoid_spec.argtypes = [ctypes.c_float]
        L.orc_float_to_bf16.restype = ctypes.c_uint16
        L.orc_float_to_bf16.argtypes = [ctypes.c_float]
        L.orc_transcode.restype = ctypes.c_int
        L.orc_num_threads.restype = ctypes.c_int
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


# --- scalar codecs -----------------------------------------------------------

def e2m1_value(code: int) -> float:
    return _load().orc_e2m1_value(code)


def e4m3_value(byte: int) -> float:
    return _load().orc_e4m3_value(byte)


def e8m0_value(byte: int) -> float:
    return _load().orc_e8m0_value(byte)


def e4m3_rne_satfinite(x: float) -> int:
    return _load().orc_e4m3_rne_satfinite(x)


def e2m1_rne_sat(x: float) -> int:
    return _load().orc_e2m1_rne_sat(x)


def exp_spec(y: float) -> float:
    return _load().orc_exp_spec(y)


def sigmoid_spec(x: float) -> float:
    return _load().orc_sigmoid_spec(x)


def float_to_bf16(x: float) -> int:
    return _load().orc_float_to_bf16(x)


def num_threads() -> int:
    return _load().orc_num_threads()


# --- tensors -------------------------------------------------------------------

def decode_mxfp4(codes: np.ndarray, e8m0: np.ndarray, N: int, K: int) -> np.ndarray:
    out = np.empty((N, K), np.float64)
    _load().orc_decode_mxfp4(_p(np.ascontiguousarray(codes)), _p(np.ascontiguousarray(e8m0)),
                             ctypes.c_int64(N), ctypes.c_int64(K), _p(out))
    return out


def decode_nvfp4(codes: np.ndarray, e4m3: np.ndarray, global_scale: float, N: int, K: int) -> np.ndarray:
    out = np.empty((N, K), np.float64)
    _load().orc_decode_nvfp4(_p(np.ascontiguousarray(codes)), _p(np.ascontiguousarray(e4m3)),
                             ctypes.c_float(global_scale), ctypes.c_int64(N), ctypes.c_int64(K), _p(out))
    return out


def compact_scales(codes: np.ndarray, e4m3: np.ndarray, rows: int, K: int):
    """NVFP4 rows -> compact scales.  Returns (nib [rows, K/64] u8, row_exp [rows]
    i8, status [rows] i32, number of rows that are not representable)."""
    codes = np.ascontiguousarray(codes, np.uint8)
    e4m3 = np.ascontiguousarray(e4m3, np.uint8)
    nib = np.empty((rows, K // 64), np.uint8)
    rexp = np.empty(rows, np.int8)
    status = np.empty(rows, np.int32)
    L = _load()
    L.orc_compact_scales.restype = ctypes.c_int64
    bad = L.orc_compact_scales(_p(codes), _p(e4m3), ctypes.c_int64(rows), ctypes.c_int64(K), _p(nib), _p(rexp),
                               _p(status))
    return nib, rexp, status, int(bad)


def compact_decode(nib: np.ndarray, row_exp: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Scale of every 32-code block [rows, K/32] (float64) of compact rows."""
    out = np.empty((rows, K // 32), np.float64)
    _load().orc_compact_decode(_p(np.ascontiguousarray(nib, np.uint8)), _p(np.ascontiguousarray(row_exp, np.int8)),
                               ctypes.c_int64(rows), ctypes.c_int64(K), _p(out))
    return out


def transcode(codes: np.ndarray, e8m0: np.ndarray, num_tensors: int, N: int, K: int):
    """Returns (codes_out, e4m3 [nt, N, K/16], global [nt] f32, status [nt] i32,
    report [blocks, zero_blocks, nonrepresentable_tensors, nan_tensors], worst)."""
    codes = np.ascontiguousarray(codes, np.uint8)
    e8m0 = np.ascontiguousarray(e8m0, np.uint8)
    codes_out = np.empty(num_tensors * N * K // 2, np.uint8)
    e4m3 = np.empty((num_tensors, N, K // 16), np.uint8)
    glob = np.empty(num_tensors, np.float32)
    status = np.empty(num_tensors, np.int32)
    report = np.zeros(4, np.int64)
    worst = _load().orc_transcode(_p(codes), _p(e8m0), ctypes.c_int64(num_tensors), ctypes.c_int64(N),
                                  ctypes.c_int64(K), _p(codes_out), _p(e4m3), _p(glob), _p(status), _p(report))
    return codes_out.reshape(num_tensors, N, K // 2), e4m3, glob, status, report, worst


def route(logits: np.ndarray, bias, n_group: int, topk_group: int, top_k: int, rsf: float,
          renormalize: bool = True):
    logits = np.ascontiguousarray(logits, np.float32)
    T, E = logits.shape
    ids = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    _load().orc_route(_p(logits), None if b is None else _p(b), ctypes.c_int(T), ctypes.c_int(E),
                      ctypes.c_int(n_group), ctypes.c_int(topk_group), ctypes.c_int(top_k), ctypes.c_float(rsf),
                      ctypes.c_int(int(renormalize)), _p(ids), _p(w))
    return ids, w


def router_logits(x_bits: np.ndarray, w: np.ndarray):
    """FP32 router logits of BF16 rows x_bits [T,H] (uint16) against FP32 router
    rows w [E,H], float64 dot products rounded once; also the float64 sums of
    |x_h w_h| (the scale of each logit's rounding error bound)."""
    x = np.ascontiguousarray(x_bits, np.uint16)
    wr = np.ascontiguousarray(w, np.float32)
    T, H = x.shape
    E = wr.shape[0]
    out = np.empty((T, E), np.float32)
    mag = np.empty((T, E), np.float64)
    _load().orc_router_logits(_p(x), _p(wr), ctypes.c_int(T), ctypes.c_int(H), ctypes.c_int(E), _p(out), _p(mag))
    return out, mag


def permute(topk_ids: np.ndarray, E: int):
    ids = np.ascontiguousarray(topk_ids, np.int32)
    T, k = ids.shape
    P = T * k
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    row_of_pair = np.empty(P, np.int32)
    pair_of_row = np.empty(P, np.int32)
    _load().orc_permute(_p(ids), ctypes.c_int(T), ctypes.c_int(k), ctypes.c_int(E), _p(counts), _p(offsets),
                        _p(row_of_pair), _p(pair_of_row))
    return counts, offsets, row_of_pair, pair_of_row


def quantize_bf16(x_bits: np.ndarray, gs: float = 1.0):
    """x_bits: uint16 BF16 bit patterns [M, K]. Returns codes [M, K/2], scales [M, K/16]."""
    x = np.ascontiguousarray(x_bits, np.uint16)
    M, K = x.shape
    codes = np.empty((M, K // 2), np.uint8)
    scales = np.empty((M, K // 16), np.uint8)
    _load().orc_quantize_bf16(_p(x), ctypes.c_int64(M), ctypes.c_int64(K), ctypes.c_float(gs), _p(codes),
                              _p(scales))
    return codes, scales


def quantize_f32(x: np.ndarray, gs: float = 1.0):
    x = np.ascontiguousarray(x, np.float32)
    M, K = x.shape
    codes = np.empty((M, K // 2), np.uint8)
    scales = np.empty((M, K // 16), np.uint8)
    _load().orc_quantize_f32(_p(x), ctypes.c_int64(M), ctypes.c_int64(K), ctypes.c_float(gs), _p(codes),
                             _p(scales))
    return codes, scales


def quantize_mxfp8_f32(x: np.ndarray):
    """MXFP8 of FP32 rows [M, K]: E4M3 codes [M, K] and E8M0 scales [M, K/32]."""
    x = np.ascontiguousarray(x, np.float32)
    M, K = x.shape
    codes = np.empty((M, K), np.uint8)
    scales = np.empty((M, K // 32), np.uint8)
    _load().orc_quantize_mxfp8_f32(_p(x), ctypes.c_int64(M), ctypes.c_int64(K), _p(codes), _p(scales))
    return codes, scales


def quantize_mxfp8_bf16(x_bits: np.ndarray):
    x = np.ascontiguousarray(x_bits, np.uint16)
    M, K = x.shape
    codes = np.empty((M, K), np.uint8)
    scales = np.empty((M, K // 32), np.uint8)
    _load().orc_quantize_mxfp8_bf16(_p(x), ctypes.c_int64(M), ctypes.c_int64(K), _p(codes), _p(scales))
    return codes, scales


def moe_layer(mode: int, x_bits, logits, bias, gate_codes, gate_sf, up_codes, up_sf, down_codes, down_sf,
              w_global, act_global: float, n_group: int, topk_group: int, top_k: int, rsf: float,
              renormalize: bool = True, tokens=None, act_global_mid=None) -> np.ndarray:
    """float64 layer output [len(tokens), H] (mode 0 = W4A16, 1 = W4A4, 3 = W4A8:
    MXFP8 activations, which takes no activation global).  act_global
    scales the layer input's quantisation, act_global_mid (default: the same) the
    down-projection input's."""
    x = np.ascontiguousarray(x_bits, np.uint16)
    T, H = x.shape
    E, I = gate_codes.shape[0], gate_codes.shape[1]
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tokens = np.ascontiguousarray(tokens, np.int32)
    out = np.empty((len(tokens), H), np.float64)
    arrs = [np.ascontiguousarray(a, np.uint8) for a in (gate_codes, gate_sf, up_codes, up_sf, down_codes, down_sf)]
    lg = np.ascontiguousarray(logits, np.float32)
    wg = np.ascontiguousarray(w_global, np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    mid = act_global if act_global_mid is None else act_global_mid
    _load().orc_moe_layer2(ctypes.c_int(mode), _p(x), _p(lg), None if b is None else _p(b), *[_p(a) for a in arrs],
                           _p(wg), ctypes.c_float(act_global), ctypes.c_float(mid), ctypes.c_int(T), ctypes.c_int(H),
                           ctypes.c_int(I), ctypes.c_int(E), ctypes.c_int(n_group), ctypes.c_int(topk_group),
                           ctypes.c_int(top_k), ctypes.c_float(rsf), ctypes.c_int(int(renormalize)), _p(tokens),
                           ctypes.c_int(len(tokens)), _p(out))
    return out


def moe_intermediate(mode: int, x_bits, logits, bias, gate_codes, gate_sf, up_codes, up_sf, w_global,
                     act_global: float, n_group: int, topk_group: int, top_k: int, rsf: float,
                     renormalize: bool = True, tokens=None, acc_rel: float | None = None):
    """The SwiGLU output before the intermediate quantisation, FP32 [n, top_k, I],
    with the tokens' routing ids / weights [n, top_k] (float64 arithmetic as the
    layer's, rounded once to FP32).  With acc_rel, also a bound [n, top_k, I] on
    the distance of an FP32 evaluation whose gate/up dot products err by at most
    acc_rel * sum |x w| (see orc_moe_intermediate)."""
    x = np.ascontiguousarray(x_bits, np.uint16)
    T, H = x.shape
    E, I = gate_codes.shape[0], gate_codes.shape[1]
    tokens = np.arange(T, dtype=np.int32) if tokens is None else np.ascontiguousarray(tokens, np.int32)
    n = len(tokens)
    a32 = np.empty((n, top_k, I), np.float32)
    ids = np.empty((n, top_k), np.int32)
    wts = np.empty((n, top_k), np.float32)
    arrs = [np.ascontiguousarray(a, np.uint8) for a in (gate_codes, gate_sf, up_codes, up_sf)]
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    err = None if acc_rel is None else np.empty((n, top_k, I), np.float32)
    _load().orc_moe_intermediate(ctypes.c_int(mode), _p(x), _p(np.ascontiguousarray(logits, np.float32)),
                                 None if b is None else _p(b), *[_p(a) for a in arrs],
                                 _p(np.ascontiguousarray(w_global, np.float32)), ctypes.c_float(act_global),
                                 ctypes.c_int(H), ctypes.c_int(I), ctypes.c_int(E), ctypes.c_int(n_group),
                                 ctypes.c_int(topk_group), ctypes.c_int(top_k), ctypes.c_float(rsf),
                                 ctypes.c_int(int(renormalize)), _p(tokens), ctypes.c_int(n), _p(a32), _p(ids),
                                 _p(wts), ctypes.c_double(acc_rel or 0.0), None if err is None else _p(err))
    return (a32, ids, wts) if err is None else (a32, ids, wts, err)


def moe_down(a: np.ndarray, ids: np.ndarray, wts: np.ndarray, down_codes, down_sf, w_global) -> np.ndarray:
    """float64 layer output [n, H] from down-projection inputs a [n, top_k, I]
    (float64 values) and the tokens' routing ids / weights [n, top_k]."""
    a = np.ascontiguousarray(a, np.float64)
    n, k, I = a.shape
    E, H = down_codes.shape[0], down_codes.shape[1]
    out = np.empty((n, H), np.float64)
    _load().orc_moe_down(_p(a), _p(np.ascontiguousarray(ids, np.int32)), _p(np.ascontiguousarray(wts, np.float32)),
                         _p(np.ascontiguousarray(down_codes, np.uint8)), _p(np.ascontiguousarray(down_sf, np.uint8)),
                         _p(np.ascontiguousarray(w_global, np.float32)), ctypes.c_int(H), ctypes.c_int(I),
                         ctypes.c_int(E), ctypes.c_int(k), ctypes.c_int(n), _p(out))
    return out


def decode_mxfp8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    M, K = codes.shape
    out = np.empty((M, K), np.float64)
    _load().orc_decode_mxfp8(_p(codes), _p(np.ascontiguousarray(scales, np.uint8)), ctypes.c_int64(M),
                             ctypes.c_int64(K), _p(out))
    return out
