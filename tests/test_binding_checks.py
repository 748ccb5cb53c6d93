"""The Python binding's argument checks (CPU only): each tensor must be on a
CUDA device, contiguous and at least as large as include/nvfp4moe.h lays it out
for the sizes passed.  The library is replaced by a recorder, so no pointer is
ever used; the device test is switched off where sizes are under test."""
import pytest
import torch

import nvfp4_mixture_experts_grouped_b200 as moe

U8, I32, F32, BF16 = torch.uint8, torch.int32, torch.float32, torch.bfloat16


class _Recorder:
    """Stands in for the loaded library: size queries go to the real one, every
    other entry point records its call and returns OK."""

    def __init__(self, real):
        self.real, self.calls = real, []

    def __getattr__(self, name):
        if name.endswith("_size") or name == "nvfp4moe_last_error_string":
            return getattr(self.real, name)

        def call(*args):
            self.calls.append(name)
            return 0

        return call


@pytest.fixture
def recorder(monkeypatch):
    rec = _Recorder(moe.load())
    monkeypatch.setattr(moe, "load", lambda: rec)
    monkeypatch.setattr(moe, "_on_device", lambda t: True)
    return rec


def _z(n, dtype):
    return torch.zeros(n, dtype=dtype)


T, H, I, E, K_TOP, NG, TG = 5, 256, 128, 16, 4, 4, 2


def _cases():
    """(entry point, kwargs with correct sizes, names of the tensors whose size
    the check derives from the other arguments)."""
    P = T * K_TOP
    ws = _z(64, U8)
    packed = {m: _z(moe.load().moe_packed_weights_size(m, E, H, I), U8) for m in (moe.W4A4, moe.W4A16, moe.W4A8)}
    yield (moe.quantize_nvfp4, dict(x_bf16=torch.zeros((7, 64), dtype=BF16), gs=1.0, codes=_z(7 * 32, U8), e4m3_scales=_z(7 * 4, U8), stream=0),
           ["codes", "e4m3_scales"])
    yield (moe.quantize_mxfp8, dict(x=_z(7 * 64, BF16), M=7, K=64, codes=_z(7 * 64, U8), e8m0_scales=_z(14, U8),
                                    stream=0), ["x", "codes", "e8m0_scales"])
    yield (moe.moe_route, dict(logits=torch.zeros((T, E), dtype=F32), bias=_z(E, F32), n_group=NG, topk_group=TG,
                               top_k=K_TOP, routed_scaling_factor=2.827, renormalize=True, topk_ids=_z(P, I32),
                               topk_weights=_z(P, F32), stream=0), ["bias", "topk_ids", "topk_weights"])
    yield (moe.moe_router_topk, dict(x_bf16=torch.zeros((T, H), dtype=BF16), w_router=torch.zeros((E, H), dtype=F32),
                                     bias=None, n_group=NG, topk_group=TG, top_k=K_TOP, routed_scaling_factor=2.827,
                                     renormalize=True, logits_out=_z(T * E, F32), topk_ids=_z(P, I32),
                                     topk_weights=_z(P, F32), workspace=ws, stream=0),
           ["logits_out", "topk_ids", "topk_weights"])
    yield (moe.moe_permute, dict(topk_ids=torch.zeros((T, K_TOP), dtype=I32), E=E, pad=128, counts_out=_z(E, I32),
                                 pad_offsets_out=_z(E + 1, I32), row_of_pair_out=_z(P, I32), workspace=ws, stream=0),
           ["counts_out", "pad_offsets_out", "row_of_pair_out"])
    yield (moe.moe_permute_noalloc, dict(topk_ids=torch.zeros((T, K_TOP), dtype=I32), E=E, pad=128,
                                         counts_out=_z(E, I32), pad_offsets_out=_z(E + 1, I32),
                                         row_of_pair_out=_z(P, I32), stream=0),
           ["counts_out", "pad_offsets_out", "row_of_pair_out"])
    yield (moe.nvfp4_compact_scales, dict(codes=_z(9 * 128, U8), e4m3_sf=_z(9 * 16, U8), rows=9, K=256,
                                          nib_out=_z(9 * 4, U8), row_exp_out=_z(9, torch.int8),
                                          row_status_out=_z(9, I32), n_bad_out=_z(1, I32), stream=0),
           ["codes", "e4m3_sf", "nib_out", "row_exp_out", "row_status_out", "n_bad_out"])
    yield (moe.transcode_mxfp4_to_nvfp4, dict(codes_in=_z(3 * 8 * 64 // 2, U8), e8m0_in=_z(3 * 8 * 2, U8),
                                              num_tensors=3, N=8, K=64, codes_out=_z(3 * 8 * 32, U8),
                                              e4m3_out=_z(3 * 8 * 4, U8), global_scale_out=_z(3, F32),
                                              tensor_status_out=_z(3, I32), workspace=ws, report=False, stream=0),
           ["codes_in", "e8m0_in", "codes_out", "e4m3_out", "global_scale_out", "tensor_status_out"])
    n = E * I * H
    for mode in (moe.W4A4, moe.W4A16, moe.W4A8):
        yield (moe.moe_pack_weights, dict(mode=mode, gate_codes=torch.zeros((E, I, H // 2), dtype=U8),
                                          gate_sf=_z(n // 16, U8), up_codes=_z(n // 2, U8), up_sf=_z(n // 16, U8),
                                          down_codes=torch.zeros((E, H, I // 2), dtype=U8), down_sf=_z(n // 16, U8),
                                          w_global=_z(3 * E, F32), packed=packed[mode], stream=0),
               ["gate_sf", "up_codes", "up_sf", "down_sf", "w_global", "packed"])
        for out_dtype in (BF16, F32):
            common = dict(mode=mode, x=_z(T * H, BF16), packed_weights=packed[mode], T=T, H=H, I=I, E=E,
                          workspace=ws, out=_z(T * H, out_dtype), stream=0)
            layer = dict(common, router_logits=_z(T * E, F32), bias=_z(E, F32), n_group=NG, topk_group=TG,
                         top_k=K_TOP, routed_scaling_factor=2.827, renormalize=True, topk_ids_out=_z(P, I32),
                         topk_weights_out=_z(P, F32))
            sized = ["x", "router_logits", "bias", "packed_weights", "out", "topk_ids_out", "topk_weights_out"]
            yield (moe.moe_forward, dict(layer, act_global=1.0), sized)
            yield (moe.moe_forward_ex, dict(layer, act_global_in=1.0, act_global_mid=1.0), sized)
            yield (moe.moe_forward_routed, dict(common, topk_ids=_z(P, I32), topk_weights=_z(P, F32), act_global=1.0,
                                                top_k=K_TOP), ["x", "topk_ids", "topk_weights", "packed_weights", "out"])


CASES = list(_cases())


@pytest.mark.parametrize("i", range(len(CASES)))
def test_correct_sizes_pass_and_each_short_buffer_is_refused(recorder, i):
    fn, kw, sized = CASES[i]
    fn(**kw)
    assert len(recorder.calls) == 1
    for name in sized:
        t = kw[name]
        short = t.reshape(-1)[:-1]  # one element short
        with pytest.raises(moe.NVFP4MoEError, match=f"{name} holds"):
            fn(**dict(kw, **{name: short}))
    assert len(recorder.calls) == 1  # no refused call reached the library


def test_optional_tensors_may_be_none_and_required_ones_may_not(recorder):
    fn, kw, _ = CASES[[c[0] for c in CASES].index(moe.moe_forward)]
    fn(**dict(kw, bias=None, topk_ids_out=None, topk_weights_out=None))
    with pytest.raises(moe.NVFP4MoEError, match="out is required"):
        fn(**dict(kw, out=None))


def test_host_and_strided_tensors_are_refused(monkeypatch):
    rec = _Recorder(moe.load())
    monkeypatch.setattr(moe, "load", lambda: rec)
    x = torch.zeros((7, 64), dtype=BF16)
    c, s = _z(7 * 32, U8), _z(7 * 4, U8)
    with pytest.raises(moe.NVFP4MoEError, match="must be a CUDA tensor"):
        moe.quantize_nvfp4(x, 1.0, c, s, stream=0)
    monkeypatch.setattr(moe, "_on_device", lambda t: True)
    with pytest.raises(moe.NVFP4MoEError, match="must be contiguous"):
        moe.quantize_nvfp4(torch.zeros((64, 14), dtype=BF16).t()[:7], 1.0, c, s, stream=0)
    assert rec.calls == []
