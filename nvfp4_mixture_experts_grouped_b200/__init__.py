"""B200 (sm_100a) routed-expert MoE layer with NVFP4 expert weights.

Thin ctypes binding of ``libnvfp4moe.so`` (declared in ``include/nvfp4moe.h``).
Every function takes ``torch`` tensors that already live on the GPU and
passes raw device pointers and sizes to the C ABI; all arithmetic runs in the
library's CUDA kernels.  Before the call each tensor is checked for what a raw
pointer cannot carry -- it is on a CUDA device, contiguous and at least as
large as the header's layout for the given sizes -- so that a wrong argument
raises here instead of becoming an out-of-bounds access on the GPU.  PyTorch is used
for device memory and streams only.  There is no CPU fallback: if the shared
library cannot be loaded every call raises.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "W4A16", "W4A4", "NVFP4MoEError", "library_path", "load",
    "transcode_mxfp4_to_nvfp4", "nvfp4moe_transcode_workspace_size", "moe_route", "moe_router_topk",
    "moe_router_topk_workspace_size", "quantize_nvfp4",
    "moe_packed_weights_size", "moe_pack_weights", "moe_forward_workspace_size", "moe_forward",
    "moe_forward_ex", "moe_forward_routed", "nvfp4moe_check_device_status", "nvfp4moe_version", "moe_permute",
    "moe_permute_workspace_size", "nvfp4moe_set_trace_events", "moe_permute_noalloc", "W4A16C", "W4A8",
    "nvfp4_compact_scales", "quantize_mxfp8", "moe_forward_intermediate", "nvfp4moe_raise_device_error",
    "nvfp4moe_selftest_wait_timeout",
]

W4A16 = 0
W4A4 = 1
W4A16C = 2  # W4A16 on weights with compact (4.125-bit) scales
W4A8 = 3  # MXFP8 activations x FP4 weights (prefill)

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libnvfp4moe.so")
_lib = None

STATUS_NAMES = {
    0: "OK", 1: "ERR_INVALID_ARG", 2: "ERR_ALIGNMENT", 3: "ERR_UNSUPPORTED_SHAPE", 4: "ERR_NAN_SCALE",
    5: "ERR_NOT_REPRESENTABLE", 6: "ERR_WORKSPACE_TOO_SMALL", 7: "ERR_CUDA", 8: "ERR_TIMEOUT",
    9: "ERR_UNSUPPORTED_DEVICE",
}


class NVFP4MoEError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class TranscodeReport(ctypes.Structure):
    _fields_ = [("blocks", ctypes.c_int64), ("zero_blocks", ctypes.c_int64),
                ("nonrepresentable_tensors", ctypes.c_int64), ("nan_scale_tensors", ctypes.c_int64)]


class ExpertWeights(ctypes.Structure):
    _fields_ = [("gate_codes", ctypes.c_void_p), ("gate_sf", ctypes.c_void_p), ("up_codes", ctypes.c_void_p),
                ("up_sf", ctypes.c_void_p), ("down_codes", ctypes.c_void_p), ("down_sf", ctypes.c_void_p),
                ("w_global", ctypes.c_void_p), ("E", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32)]


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m nvfp4_mixture_experts_grouped_b200.build`")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    L.nvfp4moe_last_error_string.restype = ctypes.c_char_p
    L.nvfp4moe_version.restype = i32
    L.nvfp4moe_transcode_workspace_size.restype = sz
    L.nvfp4moe_transcode_workspace_size.argtypes = [i64]
    L.transcode_mxfp4_to_nvfp4.restype = ctypes.c_int
    L.transcode_mxfp4_to_nvfp4.argtypes = [vp, vp, i64, i64, i64, vp, vp, vp, vp, vp, sz, ctypes.POINTER(TranscodeReport),
                                           vp]
    L.nvfp4_compact_scales.restype = ctypes.c_int
    L.nvfp4_compact_scales.argtypes = [vp, vp, i64, i64, vp, vp, vp, vp, vp]
    L.moe_route.restype = ctypes.c_int
    L.moe_route.argtypes = [vp, vp, i32, i32, i32, i32, i32, f32, i32, vp, vp, vp]
    L.moe_router_topk_workspace_size.restype = sz
    L.moe_router_topk_workspace_size.argtypes = [i32]
    L.moe_router_topk.restype = ctypes.c_int
    L.moe_router_topk.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, i32, vp, vp, vp, vp, sz, vp]
    L.quantize_mxfp8.restype = ctypes.c_int
    L.quantize_mxfp8.argtypes = [vp, i64, i64, vp, vp, vp]
    L.quantize_nvfp4.restype = ctypes.c_int
    L.quantize_nvfp4.argtypes = [vp, i64, i64, f32, vp, vp, vp]
    L.moe_packed_weights_size.restype = sz
    L.moe_packed_weights_size.argtypes = [ctypes.c_int, i32, i32, i32]
    L.moe_pack_weights.restype = ctypes.c_int
    L.moe_pack_weights.argtypes = [ctypes.c_int, ctypes.POINTER(ExpertWeights), vp, vp]
    L.moe_forward_workspace_size.restype = sz
    L.moe_forward_workspace_size.argtypes = [ctypes.c_int, i32, i32, i32, i32, i32]
    L.moe_forward.restype = ctypes.c_int
    L.moe_forward.argtypes = [ctypes.c_int, vp, vp, vp, vp, f32, i32, i32, i32, i32, i32, i32, i32, f32, i32, vp, sz, vp,
                              i32, vp, vp, vp]
    L.moe_forward_ex.restype = ctypes.c_int
    L.moe_forward_ex.argtypes = [ctypes.c_int, vp, vp, vp, vp, f32, f32, i32, i32, i32, i32, i32, i32, i32, f32, i32,
                                 vp, sz, vp, i32, vp, vp, vp]
    L.moe_forward_routed.restype = ctypes.c_int
    L.moe_forward_routed.argtypes = [ctypes.c_int, vp, vp, vp, vp, f32, i32, i32, i32, i32, i32, vp, sz, vp, i32, vp]
    L.moe_permute_workspace_size.restype = sz
    L.moe_permute_workspace_size.argtypes = [i32, i32, i32, i32]
    L.moe_permute.restype = ctypes.c_int
    L.moe_permute.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, sz, vp]
    L.moe_permute_noalloc.restype = ctypes.c_int
    L.moe_permute_noalloc.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp]
    L.moe_forward_intermediate.restype = ctypes.c_int
    L.moe_forward_intermediate.argtypes = [ctypes.c_int, i32, i32, i32, i32, i32, vp, sz, vp, i32, vp, vp, vp]
    L.nvfp4moe_set_trace_events.restype = ctypes.c_int
    L.nvfp4moe_set_trace_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), i32]
    L.nvfp4moe_check_device_status.restype = ctypes.c_int
    L.nvfp4moe_check_device_status.argtypes = [vp]
    L.nvfp4moe_raise_device_error.restype = ctypes.c_int
    L.nvfp4moe_raise_device_error.argtypes = [i32, vp]
    L.nvfp4moe_selftest_wait_timeout.restype = ctypes.c_int
    L.nvfp4moe_selftest_wait_timeout.argtypes = [ctypes.c_int64, vp]
    _lib = L
    return L


def _on_device(t) -> bool:
    return t.is_cuda


def _arg(t, name: str, nbytes: int | None = None, optional: bool = False):
    """Device pointer of tensor ``t`` after the checks the C ABI cannot make: at
    least ``nbytes`` bytes, contiguous, on a CUDA device.  ``None`` passes only
    where the header allows NULL (``optional``)."""
    if t is None:
        if optional:
            return None
        raise NVFP4MoEError(1, f"{name} is required")
    if nbytes is not None and t.numel() * t.element_size() < nbytes:
        raise NVFP4MoEError(1, f"{name} holds {t.numel() * t.element_size()} bytes, needs {nbytes}")
    if not t.is_contiguous():
        raise NVFP4MoEError(1, f"{name} must be contiguous")
    if not _on_device(t):
        raise NVFP4MoEError(1, f"{name} must be a CUDA tensor (got {t.device})")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch

        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int):
    if status != 0:
        raise NVFP4MoEError(status, load().nvfp4moe_last_error_string().decode())


def nvfp4moe_version() -> int:
    return load().nvfp4moe_version()


def nvfp4moe_transcode_workspace_size(num_tensors: int) -> int:
    return load().nvfp4moe_transcode_workspace_size(num_tensors)


def transcode_mxfp4_to_nvfp4(codes_in, e8m0_in, num_tensors, N, K, codes_out, e4m3_out, global_scale_out,
                             tensor_status_out, workspace, report: bool = True, stream=None, raise_on_error=False):
    """Returns (status, report dict or None).  With report=True the call is synchronous."""
    rep = TranscodeReport()
    n = num_tensors * N * K
    st = load().transcode_mxfp4_to_nvfp4(
        _arg(codes_in, "codes_in", n // 2), _arg(e8m0_in, "e8m0_in", n // 32), num_tensors, N, K,
        _arg(codes_out, "codes_out", n // 2), _arg(e4m3_out, "e4m3_out", n // 16),
        _arg(global_scale_out, "global_scale_out", 4 * num_tensors),
        _arg(tensor_status_out, "tensor_status_out", 4 * num_tensors), _arg(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), ctypes.byref(rep) if report else None, _stream(stream))
    if st not in (0, 4, 5) or (raise_on_error and st != 0):
        _check(st)
    out = None
    if report:
        out = {f: getattr(rep, f) for f, _ in TranscodeReport._fields_}
    return st, out


def moe_route(logits, bias, n_group, topk_group, top_k, routed_scaling_factor, renormalize, topk_ids, topk_weights,
              stream=None):
    T, E = logits.shape
    _check(load().moe_route(_arg(logits, "logits", 4 * T * E), _arg(bias, "bias", 4 * E, optional=True), T, E,
                            n_group, topk_group, top_k, routed_scaling_factor, int(renormalize),
                            _arg(topk_ids, "topk_ids", 4 * T * top_k), _arg(topk_weights, "topk_weights", 4 * T * top_k),
                            _stream(stream)))


def moe_router_topk_workspace_size(T) -> int:
    return load().moe_router_topk_workspace_size(T)


def moe_router_topk(x_bf16, w_router, bias, n_group, topk_group, top_k, routed_scaling_factor, renormalize,
                    logits_out, topk_ids, topk_weights, workspace, stream=None):
    T, H = x_bf16.shape
    E = w_router.shape[0]
    _check(load().moe_router_topk(_arg(x_bf16, "x_bf16", 2 * T * H), _arg(w_router, "w_router", 4 * E * H),
                                  _arg(bias, "bias", 4 * E, optional=True), T, H, E, n_group, topk_group, top_k,
                                  routed_scaling_factor, int(renormalize), _arg(logits_out, "logits_out", 4 * T * E),
                                  _arg(topk_ids, "topk_ids", 4 * T * top_k),
                                  _arg(topk_weights, "topk_weights", 4 * T * top_k), _arg(workspace, "workspace"),
                                  workspace.numel() * workspace.element_size(), _stream(stream)))


def quantize_mxfp8(x, M, K, codes, e8m0_scales, stream=None):
    _check(load().quantize_mxfp8(_arg(x, "x", 2 * M * K), M, K, _arg(codes, "codes", M * K),
                                 _arg(e8m0_scales, "e8m0_scales", M * (K // 32)), _stream(stream)))


def quantize_nvfp4(x_bf16, gs, codes, e4m3_scales, stream=None):
    M, K = x_bf16.shape
    _check(load().quantize_nvfp4(_arg(x_bf16, "x_bf16", 2 * M * K), M, K, gs, _arg(codes, "codes", M * K // 2),
                                 _arg(e4m3_scales, "e4m3_scales", M * (K // 16)), _stream(stream)))


def moe_permute_workspace_size(T, E, top_k, pad) -> int:
    return load().moe_permute_workspace_size(T, E, top_k, pad)


def moe_permute(topk_ids, E, pad, counts_out, pad_offsets_out, row_of_pair_out, workspace, stream=None):
    T, k = topk_ids.shape
    _check(load().moe_permute(_arg(topk_ids, "topk_ids", 4 * T * k), T, E, k, pad, _arg(counts_out, "counts_out", 4 * E),
                              _arg(pad_offsets_out, "pad_offsets_out", 4 * (E + 1)),
                              _arg(row_of_pair_out, "row_of_pair_out", 4 * T * k), _arg(workspace, "workspace"),
                              workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_permute_noalloc(topk_ids, E, pad, counts_out, pad_offsets_out, row_of_pair_out, stream=None):
    """moe_permute for callers that cannot allocate device memory: the scratch is
    a fixed 1 MiB device array inside the library (see include/nvfp4moe.h)."""
    T, k = topk_ids.shape
    _check(load().moe_permute_noalloc(_arg(topk_ids, "topk_ids", 4 * T * k), T, E, k, pad,
                                      _arg(counts_out, "counts_out", 4 * E),
                                      _arg(pad_offsets_out, "pad_offsets_out", 4 * (E + 1)),
                                      _arg(row_of_pair_out, "row_of_pair_out", 4 * T * k), _stream(stream)))


def nvfp4_compact_scales(codes, e4m3_sf, rows, K, nib_out, row_exp_out, row_status_out, n_bad_out=None,
                         stream=None):
    _check(load().nvfp4_compact_scales(_arg(codes, "codes", rows * K // 2), _arg(e4m3_sf, "e4m3_sf", rows * (K // 16)),
                                       rows, K, _arg(nib_out, "nib_out", rows * (K // 64), optional=True),
                                       _arg(row_exp_out, "row_exp_out", rows, optional=True),
                                       _arg(row_status_out, "row_status_out", 4 * rows, optional=True),
                                       _arg(n_bad_out, "n_bad_out", 4, optional=True), _stream(stream)))


def moe_packed_weights_size(mode, E, H, I) -> int:
    return load().moe_packed_weights_size(mode, E, H, I)


def moe_pack_weights(mode, gate_codes, gate_sf, up_codes, up_sf, down_codes, down_sf, w_global, packed, stream=None):
    E, I = gate_codes.shape[0], gate_codes.shape[1]
    H = down_codes.shape[1]
    n = E * I * H  # elements of each projection
    ptrs = [_arg(gate_codes, "gate_codes", n // 2), _arg(gate_sf, "gate_sf", n // 16), _arg(up_codes, "up_codes", n // 2),
            _arg(up_sf, "up_sf", n // 16), _arg(down_codes, "down_codes", n // 2), _arg(down_sf, "down_sf", n // 16),
            _arg(w_global, "w_global", 4 * 3 * E)]
    w = ExpertWeights(*[q.value for q in ptrs], E, H, I)
    packed_ptr = _arg(packed, "packed", moe_packed_weights_size(mode, E, H, I))
    _check(load().moe_pack_weights(mode, ctypes.byref(w), packed_ptr, _stream(stream)))


def _layer_inputs(mode, x, router_logits, bias, packed_weights, T, H, I, E):
    """Checked pointers of the layer's inputs: x [T, H] BF16, router_logits
    [T, E] f32, bias [E] f32 or None, the packed weights of this mode."""
    return (_arg(x, "x", 2 * T * H), _arg(router_logits, "router_logits", 4 * T * E),
            _arg(bias, "bias", 4 * E, optional=True),
            _arg(packed_weights, "packed_weights", moe_packed_weights_size(mode, E, H, I)))


def moe_forward_workspace_size(mode, T, H, I, E, top_k) -> int:
    return load().moe_forward_workspace_size(mode, T, H, I, E, top_k)


def moe_forward(mode, x, router_logits, bias, packed_weights, act_global, T, H, I, E, n_group, topk_group, top_k,
                routed_scaling_factor, renormalize, workspace, out, topk_ids_out=None, topk_weights_out=None,
                stream=None):
    import torch

    out_f32 = 1 if out is not None and out.dtype == torch.float32 else 0
    _check(load().moe_forward(mode, *_layer_inputs(mode, x, router_logits, bias, packed_weights, T, H, I, E),
                              act_global, T, H, I, E, n_group, topk_group, top_k, routed_scaling_factor,
                              int(renormalize), _arg(workspace, "workspace"),
                              workspace.numel() * workspace.element_size(),
                              _arg(out, "out", (4 if out_f32 else 2) * T * H), out_f32,
                              _arg(topk_ids_out, "topk_ids_out", 4 * T * top_k, optional=True),
                              _arg(topk_weights_out, "topk_weights_out", 4 * T * top_k, optional=True),
                              _stream(stream)))


def moe_forward_ex(mode, x, router_logits, bias, packed_weights, act_global_in, act_global_mid, T, H, I, E, n_group,
                   topk_group, top_k, routed_scaling_factor, renormalize, workspace, out, topk_ids_out=None,
                   topk_weights_out=None, stream=None):
    import torch

    out_f32 = 1 if out is not None and out.dtype == torch.float32 else 0
    _check(load().moe_forward_ex(mode, *_layer_inputs(mode, x, router_logits, bias, packed_weights, T, H, I, E),
                                 act_global_in, act_global_mid, T, H, I, E, n_group, topk_group, top_k,
                                 routed_scaling_factor, int(renormalize), _arg(workspace, "workspace"),
                                 workspace.numel() * workspace.element_size(),
                                 _arg(out, "out", (4 if out_f32 else 2) * T * H), out_f32,
                                 _arg(topk_ids_out, "topk_ids_out", 4 * T * top_k, optional=True),
                                 _arg(topk_weights_out, "topk_weights_out", 4 * T * top_k, optional=True),
                                 _stream(stream)))


def moe_forward_routed(mode, x, topk_ids, topk_weights, packed_weights, act_global, T, H, I, E, top_k, workspace, out,
                       stream=None):
    import torch

    out_f32 = 1 if out is not None and out.dtype == torch.float32 else 0
    _check(load().moe_forward_routed(mode, _arg(x, "x", 2 * T * H), _arg(topk_ids, "topk_ids", 4 * T * top_k),
                                     _arg(topk_weights, "topk_weights", 4 * T * top_k),
                                     _arg(packed_weights, "packed_weights", moe_packed_weights_size(mode, E, H, I)),
                                     act_global, T, H, I, E, top_k, _arg(workspace, "workspace"),
                                     workspace.numel() * workspace.element_size(),
                                     _arg(out, "out", (4 if out_f32 else 2) * T * H), out_f32, _stream(stream)))


def moe_forward_intermediate(mode, T, H, I, E, top_k, workspace, pairs, codes_out, scales_out=None, stream=None):
    """The down projection's input rows of `pairs` (int32 t * top_k + j) from the
    last forward call made with `workspace`, in the checkpoint layout (see
    include/nvfp4moe.h for the per-mode shapes)."""
    n = pairs.numel()
    row_bytes = I // 2 if mode == W4A4 else I if mode == W4A8 else 2 * I
    scale_bytes = I // 16 if mode == W4A4 else I // 32 if mode == W4A8 else 0
    _check(load().moe_forward_intermediate(mode, T, H, I, E, top_k, _arg(workspace, "workspace"),
                                           workspace.numel() * workspace.element_size(), _arg(pairs, "pairs", 4 * n), n,
                                           _arg(codes_out, "codes_out", n * row_bytes),
                                           _arg(scales_out, "scales_out", n * scale_bytes, optional=scale_bytes == 0),
                                           _stream(stream)))


def nvfp4moe_set_trace_events(events) -> None:
    """events: None (tracing off) or 7 torch.cuda.Event(enable_timing=True) objects
    (each already created, e.g. recorded once)."""
    if events is None:
        _check(load().nvfp4moe_set_trace_events(None, 0))
        return
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _check(load().nvfp4moe_set_trace_events(arr, len(events)))


def nvfp4moe_check_device_status(stream=None):
    _check(load().nvfp4moe_check_device_status(_stream(stream)))


def nvfp4moe_raise_device_error(bits: int, stream=None):
    """Test hook: ORs `bits` into the device error word (see the header)."""
    _check(load().nvfp4moe_raise_device_error(int(bits), _stream(stream)))


def nvfp4moe_selftest_wait_timeout(limit_cycles: int, stream=None):
    """Test hook: a bounded wait on a barrier nothing arrives on (see the header)."""
    _check(load().nvfp4moe_selftest_wait_timeout(int(limit_cycles), _stream(stream)))
