"""The C ABI library: it loads, exports every function include/nvfp4moe.h
declares, and its host-side validation rejects bad arguments before touching
the GPU.  CPU only (no kernel is launched)."""
import ctypes
import os
import re

import pytest

import nvfp4_mixture_experts_grouped_b200 as moe

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "nvfp4moe.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w ]*?[\s\*]+([A-Za-z_]\w*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for n in ("transcode_mxfp4_to_nvfp4", "moe_route", "quantize_nvfp4", "moe_forward", "moe_pack_weights",
              "moe_permute", "moe_forward_routed", "moe_forward_ex", "nvfp4_compact_scales", "quantize_mxfp8"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = moe.load()
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_version_and_sizes():
    assert moe.nvfp4moe_version() >> 16 == 1
    assert moe.nvfp4moe_transcode_workspace_size(768) >= 32
    E, H, I = 256, 4096, 2048
    # W4A4 packed weights hold exactly the checkpoint bytes (codes + E4M3 scales + globals)
    exact = E * (2 * I * H + H * I) // 2 + E * (2 * I * H + H * I) // 16 + E * 3 * 4
    assert exact <= moe.moe_packed_weights_size(moe.W4A4, E, H, I) <= exact + 1024
    assert exact <= moe.moe_packed_weights_size(moe.W4A16, E, H, I) <= exact + 1024
    # compact scales: codes + one byte per 64 weights + one exponent byte per row + globals + a status word
    compact = E * (2 * I * H + H * I) // 2 + E * (2 * I * H + H * I) // 64 + E * (2 * I + H) + E * 3 * 4 + 16
    assert compact <= moe.moe_packed_weights_size(moe.W4A16C, E, H, I) <= compact + 2048
    bits = 8 * moe.moe_packed_weights_size(moe.W4A16C, E, H, I) / (E * 3 * I * H)
    assert 4.125 < bits < 4.13
    # W4A8: the 4-bit codes + an E8M0 scale per 32 + globals + a status word
    w8 = E * (2 * I * H + H * I) // 2 + E * (2 * I * H + H * I) // 32 + E * 3 * 4 + 16
    assert w8 <= moe.moe_packed_weights_size(moe.W4A8, E, H, I) <= w8 + 2048
    assert moe.moe_packed_weights_size(4, E, H, I) == 0  # unknown mode
    ws8 = moe.moe_forward_workspace_size(moe.W4A8, 8192, H, I, E, 8)
    assert ws8 > moe.moe_forward_workspace_size(moe.W4A4, 8192, H, I, E, 8)
    ws = moe.moe_forward_workspace_size(moe.W4A4, 8192, H, I, E, 8)
    assert ws > 8192 * 8 * H * 2  # holds the per-pair BF16 rows at least
    assert moe.moe_forward_workspace_size(moe.W4A4, -1, H, I, E, 8) == 0


def _status(call):
    return call


@pytest.mark.parametrize("args,expect", [
    # T, E, n_group, topk_group, top_k
    ((4, 0, 1, 1, 1), 3),
    ((4, 256, 7, 4, 8), 3),     # E % n_group
    ((4, 256, 8, 9, 8), 3),     # topk_group > n_group
    ((4, 256, 8, 4, 33), 3),    # top_k > 32
    ((4, 16, 4, 1, 5), 3),      # top_k > experts in the kept groups
    ((-1, 256, 8, 4, 8), 1),    # negative T
    ((4, 256, 64, 4, 8), 3),    # n_group > 32
])
def test_route_rejects_bad_shapes_before_launch(args, expect):
    lib = moe.load()
    T, E, ng, tg, k = args
    st = lib.moe_route(ctypes.c_void_p(16), None, T, E, ng, tg, k, 2.827, 1, ctypes.c_void_p(16),
                       ctypes.c_void_p(16), None)
    assert st == expect, lib.nvfp4moe_last_error_string()


def test_route_rejects_misaligned_pointer():
    lib = moe.load()
    st = lib.moe_route(ctypes.c_void_p(24), None, 4, 256, 8, 4, 8, 2.827, 1, ctypes.c_void_p(16),
                       ctypes.c_void_p(16), None)
    assert st == 2


def test_quantize_and_transcode_validation():
    lib = moe.load()
    assert lib.quantize_nvfp4(ctypes.c_void_p(16), 4, 24, 1.0, ctypes.c_void_p(16), ctypes.c_void_p(16), None) == 3
    assert lib.quantize_nvfp4(ctypes.c_void_p(16), 4, 32, 0.0, ctypes.c_void_p(16), ctypes.c_void_p(16), None) == 1
    assert lib.quantize_nvfp4(ctypes.c_void_p(16), 4, 32, float("nan"), ctypes.c_void_p(16), ctypes.c_void_p(16),
                              None) == 1
    p = ctypes.c_void_p(4096)
    # K not a multiple of 32
    assert lib.transcode_mxfp4_to_nvfp4(p, p, 1, 4, 48, p, p, p, p, p, 64, None, None) == 3
    # workspace too small
    assert lib.transcode_mxfp4_to_nvfp4(p, p, 1, 4, 64, p, p, p, p, p, 1, None, None) == 6
    # overlapping but unequal code buffers
    assert lib.transcode_mxfp4_to_nvfp4(p, p, 1, 4, 64, ctypes.c_void_p(4096 + 16), p, p, p, p, 64, None,
                                        None) == 1


def test_forward_validation():
    lib = moe.load()
    p = ctypes.c_void_p(4096)
    args = dict(T=4, H=4096, I=2048, E=256, ng=8, tg=4, k=8)

    def call(mode=1, ws_bytes=1 << 40, **kw):
        a = {**args, **kw}
        return lib.moe_forward(mode, p, p, None, p, 1.0, a["T"], a["H"], a["I"], a["E"], a["ng"], a["tg"], a["k"],
                               2.827, 1, p, ws_bytes, p, 0, None, None, None)

    assert call(mode=4) == 1  # unknown mode
    assert call(H=4000) == 3
    assert call(I=200) == 3
    assert call(ws_bytes=16) == 6
    assert lib.moe_forward(1, p, p, None, p, 0.0, 4, 4096, 2048, 256, 8, 4, 8, 2.827, 1, p, 1 << 40, p, 0, None,
                           None, None) == 1
    # T == 0 is a no-op even with null pointers
    assert lib.moe_forward(1, None, None, None, None, 1.0, 0, 4096, 2048, 256, 8, 4, 8, 2.827, 1, None, 0, None, 0,
                           None, None, None) == 0


def test_row_count_beyond_int32_indices_is_refused():
    # permuted rows are int32 indices: T * top_k (+ padding) above INT32_MAX is
    # refused before the workspace is looked at, however large it claims to be
    lib = moe.load()
    p = ctypes.c_void_p(4096)

    def forward(mode, T, ws_bytes):
        return lib.moe_forward(mode, p, p, None, p, 1.0, T, 4096, 2048, 256, 8, 4, 8, 2.827, 1, p, ws_bytes, p, 0,
                               None, None, None)

    big = (1 << 63) - 1
    assert forward(1, 1 << 28, big) == 3  # W4A4: 2^31 pairs
    assert forward(1, (1 << 28) - 64, big) == 3  # W4A4: below 2^31 pairs, above it with the 128-row padding
    assert forward(0, 1 << 28, big) == 3  # W4A16: 2^31 pairs, no padding
    assert forward(0, (1 << 28) - 1, 16) == 6  # 2^31 - 8 rows fit the indices: the small workspace is the error
    # moe_permute: the same bound on pairs plus padding
    assert lib.moe_permute(p, 1 << 28, 256, 8, 1, p, p, p, p, big, None) == 3
    assert lib.moe_permute(p, (1 << 28) - 64, 256, 8, 128, p, p, p, p, big, None) == 3
    assert lib.moe_permute(p, (1 << 28) - 1, 256, 8, 1, p, p, p, p, 16, None) == 6


@pytest.mark.parametrize("g_in,g_mid", [(0.0, 1.0), (1.0, 0.0), (1.0, -2.0), (float("nan"), 1.0),
                                        (1.0, float("inf"))])
def test_forward_ex_rejects_bad_activation_globals(g_in, g_mid):
    lib = moe.load()
    p = ctypes.c_void_p(4096)
    for mode in (0, 1):
        assert lib.moe_forward_ex(mode, p, p, None, p, g_in, g_mid, 4, 4096, 2048, 256, 8, 4, 8, 2.827, 1, p, 1 << 40,
                                  p, 0, None, None, None) == 1
    assert "act_global" in moe.load().nvfp4moe_last_error_string().decode()


def test_forward_ex_zero_tokens_is_a_no_op():
    lib = moe.load()
    assert lib.moe_forward_ex(1, None, None, None, None, 0.5, 2.0, 0, 4096, 2048, 256, 8, 4, 8, 2.827, 1, None, 0,
                              None, 0, None, None, None) == 0


def test_error_string_is_text():
    lib = moe.load()
    lib.moe_route(ctypes.c_void_p(16), None, 4, 0, 1, 1, 1, 1.0, 1, ctypes.c_void_p(16), ctypes.c_void_p(16), None)
    assert b"E=0" in lib.nvfp4moe_last_error_string()


@pytest.mark.parametrize("args,expect", [
    # T, H, E, n_group, topk_group, top_k, workspace bytes
    ((16, 4096, 254, 2, 1, 8, 64), 3),   # E % 4
    ((16, 4000, 256, 8, 4, 8, 64), 3),   # H % 256
    ((16, 128, 256, 8, 4, 8, 64), 3),    # H < 256
    ((16, 4096, 256, 7, 4, 8, 64), 3),   # E % n_group
    ((16, 4096, 256, 8, 4, 33, 64), 3),  # top_k > 32
    ((-2, 4096, 256, 8, 4, 8, 64), 1),   # negative T
    ((65535 * 128 + 1, 4096, 256, 8, 4, 8, 1 << 30), 1),  # T above the tiled projection's grid
    ((33, 4096, 256, 8, 4, 8, 8), 6),    # workspace below 4 bytes per 16 tokens
])
def test_router_topk_rejects_bad_arguments_before_launch(args, expect):
    T, H, E, ng, tg, k, wsb = args
    lib = moe.load()
    fake = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: validation fails first
    st = lib.moe_router_topk(fake, fake, None, T, H, E, ng, tg, k, ctypes.c_float(2.827), 1, fake, fake, fake, fake,
                             wsb, None)
    assert st == expect, moe.load().nvfp4moe_last_error_string()


def test_router_topk_zero_tokens_and_sizes():
    lib = moe.load()
    assert lib.moe_router_topk(None, None, None, 0, 4096, 256, 8, 4, 8, ctypes.c_float(1.0), 1, None, None, None,
                               None, 0, None) == 0
    assert moe.moe_router_topk_workspace_size(16) == 4
    assert moe.moe_router_topk_workspace_size(17) == 8
    assert moe.moe_router_topk_workspace_size(0) == 0


def test_compact_scales_validation():
    lib = moe.load()
    p = ctypes.c_void_p(4096)
    q = ctypes.c_void_p(4100)  # not 16-byte aligned
    assert lib.nvfp4_compact_scales(p, p, 8, 96, p, p, p, None, None) == 3   # K % 64
    assert lib.nvfp4_compact_scales(p, p, 8, 32, p, p, p, None, None) == 1   # K < 64
    assert lib.nvfp4_compact_scales(p, p, -1, 128, p, p, p, None, None) == 1
    assert lib.nvfp4_compact_scales(p, None, 8, 128, p, p, p, None, None) == 1
    assert lib.nvfp4_compact_scales(p, p, 8, 128, q, p, p, None, None) == 2
    assert lib.nvfp4_compact_scales(None, None, 0, 128, None, None, None, None, None) == 0  # no-op


def test_quantize_mxfp8_validation():
    lib = moe.load()
    p = ctypes.c_void_p(4096)
    assert lib.quantize_mxfp8(p, 4, 48, p, p, None) == 3    # K % 32
    assert lib.quantize_mxfp8(p, -1, 64, p, p, None) == 1
    assert lib.quantize_mxfp8(p, 4, 16, p, p, None) == 1    # K < 32
    assert lib.quantize_mxfp8(p, 4, 64, None, p, None) == 1
    assert lib.quantize_mxfp8(p, 4, 64, ctypes.c_void_p(4104), p, None) == 2
    assert lib.quantize_mxfp8(None, 0, 64, None, None, None) == 0


def test_forward_intermediate_validation():
    lib = moe.load()
    p = ctypes.c_void_p(4096)

    def call(mode=1, T=4, n=8, ws_bytes=1 << 40, ws=p, pairs=p, codes=p, scales=p):
        return lib.moe_forward_intermediate(mode, T, 4096, 2048, 256, 8, ws, ws_bytes, pairs, n, codes, scales, None)

    assert call(mode=4) == 1  # unknown mode
    assert call(n=-1) == 1
    assert call(ws=None) == 1
    assert call(scales=None) == 1  # W4A4 has scales
    assert call(ws_bytes=16) == 6
    # T == 0 or no pairs: nothing to read
    assert call(T=0, ws=None, pairs=None, codes=None, scales=None) == 0
    assert call(n=0, ws=None, pairs=None, codes=None, scales=None) == 0
