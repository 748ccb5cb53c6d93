"""Guard bytes around everything the library writes (a stand-in for a memory
checker, which this pool does not run): the workspace and the output of
moe_forward sit inside larger buffers whose margins are filled with 0xFF, and
after the call every margin byte is still 0xFF.  The workspace itself also starts
full of 0xFF (NaN patterns in every float view of it): the outputs must be
bit-identical to those of a call on a zeroed workspace, so nothing the kernels
read from the workspace can be a byte they did not write first.  The same for
the transcode's outputs and workspace.  Then the error paths: a bounded wait
that runs out reports a timeout, and GEMM kernels that give up mid-flight leave
the context usable."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import nvfp4_mixture_experts_grouped_b200 as moe
from nvfp4_mixture_experts_grouped_b200 import inputs

from helpers import GpuLayer, bf16_tensor, dev, nvfp4_weights_from_inputs

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes of margin on each side


def guarded(nbytes: int, fill: int):
    big = torch.full((nbytes + 2 * GUARD,), fill, dtype=torch.uint8, device="cuda")
    return big, big[GUARD:GUARD + nbytes]


def margins_untouched(big: torch.Tensor) -> bool:
    return bool((big[:GUARD] == 0xFF).all() and (big[-GUARD:] == 0xFF).all())


@pytest.mark.parametrize("mode", [moe.W4A4, moe.W4A16, moe.W4A16C, moe.W4A8])
@pytest.mark.parametrize("T", [1, 37, 300])
def test_forward_writes_nothing_outside_its_buffers(mode, T):
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl, T=T)
    w = nvfp4_weights_from_inputs(d, False)  # a transcode: power-of-two scale pairs, valid for every mode
    layer = GpuLayer(mode, w, T, wl.n_group, wl.topk_group, wl.top_k)
    x, lg = bf16_tensor(d["x"]), dev(d["logits"])
    need = moe.moe_forward_workspace_size(mode, T, wl.H, wl.I, wl.E, wl.top_k)
    outs = []
    for fill in (0x00, 0xFF):
        ws_big, ws = guarded(need, fill)
        out_big = torch.full(((T + 2) * wl.H * 4,), 0xFF, dtype=torch.uint8, device="cuda")
        out = out_big[wl.H * 4:(T + 1) * wl.H * 4].view(torch.float32).view(T, wl.H)
        if fill == 0x00:
            ws_big[:GUARD] = 0xFF
            ws_big[-GUARD:] = 0xFF
        moe.moe_forward(mode, x, lg, None, layer.packed, 1.0, T, wl.H, wl.I, wl.E, wl.n_group, wl.topk_group,
                        wl.top_k, wl.rsf, True, ws, out)
        moe.nvfp4moe_check_device_status()
        torch.cuda.synchronize()
        assert margins_untouched(ws_big), "a kernel wrote outside the workspace"
        assert bool((out_big[:wl.H * 4] == 0xFF).all() and (out_big[(T + 1) * wl.H * 4:] == 0xFF).all()), \
            "a kernel wrote outside the output"
        assert torch.isfinite(out).all()
        outs.append(out.clone())
    # a workspace full of 0xFF gives the same bits as a zeroed one
    assert torch.equal(outs[0].view(torch.int32), outs[1].view(torch.int32))


def test_transcode_writes_nothing_outside_its_buffers():
    rng = np.random.default_rng(11)
    nt, N, K = 5, 256, 512
    codes, e8 = inputs.mxfp4_tensors(rng, nt, N, K, -12, 3)
    c, s = dev(codes), dev(e8)
    co_big, co = guarded(codes.nbytes, 0xFF)
    e4_big, e4 = guarded(nt * N * K // 16, 0xFF)
    g_big, g = guarded(nt * 4, 0xFF)
    st_big, st = guarded(nt * 4, 0xFF)
    wsn = moe.nvfp4moe_transcode_workspace_size(nt)
    ws_big, ws = guarded(wsn, 0xFF)
    status, rep = moe.transcode_mxfp4_to_nvfp4(c, s, nt, N, K, co, e4, g.view(torch.float32), st.view(torch.int32),
                                               ws, report=True)
    torch.cuda.synchronize()
    assert status == 0 and rep["blocks"] == nt * N * K // 32
    for big in (co_big, e4_big, g_big, st_big, ws_big):
        assert margins_untouched(big)
    assert torch.equal(co.cpu(), c.view(torch.uint8).reshape(-1).cpu())


# ---------------------------------------------------------------------------
# error paths: a bounded wait that runs out, and GEMM kernels that give up
# mid-flight; the failure is injected on the host's side and faults nothing
# ---------------------------------------------------------------------------
TIMEOUT = 8  # NVFP4MOE_ERR_TIMEOUT


def test_bounded_wait_runs_out_and_reports_timeout():
    moe.nvfp4moe_check_device_status()
    moe.nvfp4moe_selftest_wait_timeout(2_000_000)  # ~1 ms of SM clocks, then the wait gives up
    with pytest.raises(moe.NVFP4MoEError) as e:
        moe.nvfp4moe_check_device_status()
    assert e.value.status == TIMEOUT
    moe.nvfp4moe_check_device_status()  # the word was cleared: OK again


@pytest.mark.parametrize("mode", [moe.W4A4, moe.W4A8, moe.W4A16])
def test_gemm_error_path_leaves_the_context_usable(mode):
    # With the timeout bit raised before the call, every GEMM wait that is not
    # satisfied at once gives up and the kernels leave through their error paths
    # (draining the copies and MMAs they issued).  The status says so, and the
    # next call on the same context gives the bits of a clean call.
    wl = inputs.WORKLOADS["tiny"]
    T = 300
    d = inputs.moe_inputs(wl, T=T)
    w = nvfp4_weights_from_inputs(d, False)
    layer = GpuLayer(mode, w, T, wl.n_group, wl.topk_group, wl.top_k)
    x, lg = bf16_tensor(d["x"]), dev(d["logits"])
    ref, _, _ = layer.forward(x, lg, out_fp32=True)
    ref = ref.clone()
    moe.nvfp4moe_raise_device_error(1)
    out = torch.empty_like(ref)
    moe.moe_forward(mode, x, lg, None, layer.packed, 1.0, T, wl.H, wl.I, wl.E, wl.n_group, wl.topk_group, wl.top_k,
                    wl.rsf, True, layer.ws, out)
    with pytest.raises(moe.NVFP4MoEError) as e:
        moe.nvfp4moe_check_device_status()
    assert e.value.status == TIMEOUT
    again, _, _ = layer.forward(x, lg, out_fp32=True)
    assert torch.equal(again.view(torch.int32), ref.view(torch.int32))


def test_raise_device_error_rejects_unknown_bits():
    for bits in (0, 4, -1):
        with pytest.raises(moe.NVFP4MoEError):
            moe.nvfp4moe_raise_device_error(bits)
