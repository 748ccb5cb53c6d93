"""moe_permute_noalloc: the permutation for callers that cannot allocate device
memory (a plugin handed only its inputs and outputs, or a path where cudaMalloc
may not run).  Its scratch is a fixed device array inside the library, so it is
checked through the C ABI against moe_permute with a caller workspace, on
several calls in a row with different inputs (the array keeps the previous
call's contents, which must not leak into the next result).  This file sorts last so
that a run stopping at the first failure has already run every other test."""
import numpy as np
import pytest
import torch

import nvfp4_mixture_experts_grouped_b200 as moe

pytestmark = pytest.mark.gpu


def _ids(rng, T, E, k):
    return torch.from_numpy(np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)).cuda()


def _with_workspace(ids, E, pad):
    T, k = ids.shape
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    poff = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    rop = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.moe_permute_workspace_size(T, E, k, pad), dtype=torch.uint8, device="cuda")
    moe.moe_permute(ids, E, pad, counts, poff, rop, ws)
    return counts, poff, rop


def _no_alloc(ids, E, pad):
    T, k = ids.shape
    counts = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    poff = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    rop = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    moe.moe_permute_noalloc(ids, E, pad, counts, poff, rop)
    return counts, poff, rop


def test_no_alloc_permute_matches_workspace_entry_point_twice():
    rng = np.random.default_rng(2024)
    # calls in a row on the one scratch array, each finding the previous call's
    # contents there: a large request (the three-kernel path, which writes and
    # reads back per-chunk counts), a small one (the one-CTA path), then two more
    # large ones with other ids, expert counts and padding, so that the path that
    # reads back scratch it wrote also runs on stale contents
    cases = ((8192, 256, 8, 128), (300, 64, 6, 1), (4096, 256, 8, 128), (20000, 128, 3, 1))
    for T, E, k, pad in cases:
        assert moe.moe_permute_workspace_size(T, E, k, pad) <= (1 << 20)
    for T, E, k, pad in cases:
        ids = _ids(rng, T, E, k)
        ref = _with_workspace(ids, E, pad)
        got = _no_alloc(ids, E, pad)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)


def test_no_alloc_rejects_sizes_beyond_its_array():
    lib = moe.load()
    # 65536 tokens x 32 slots over 1024 experts needs far more than 1 MiB of scratch
    assert moe.moe_permute_workspace_size(65536, 1024, 32, 128) > (1 << 20)
    st = lib.moe_permute_noalloc(None, 65536, 1024, 32, 128, None, None, None, None)
    assert st == 3
    assert b"scratch" in lib.nvfp4moe_last_error_string()
