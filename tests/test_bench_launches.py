"""bench.py's per-step kernel-launch claim (gpu_launches) against the committed
ncu launch lists of the same workloads: the kernels a step launches, counted
from the recorded launches (weight packing and torch's own kernels excluded),
equal what launches_per_step derives from the library's dispatch rules."""
import os
import re

import pytest

import bench
from nvfp4_mixture_experts_grouped_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _launches(name):
    out = {}
    for line in open(os.path.join(ROOT, "profiles", name)):
        m = re.match(r"^(k_.+?)\s{2,}(\d+)\s", line)
        if m and "pack" not in m.group(1):
            out[m.group(1)] = int(m.group(2))
    return out


@pytest.mark.parametrize("profile,workload,gemm", [
    ("launches_prefill8k_w4a4.txt", "prefill", "k_w4a4_gemm<0, 0, 1>"),
    ("launches_decode16_w4a16.txt", "decode", "k_w16_gateup<0, 4>"),
])
def test_launches_per_step_match_the_recorded_launch_list(profile, workload, gemm):
    counts = _launches(profile)
    steps = counts[gemm]  # one gate/up GEMM per step
    per_step = sum(round(n / steps) for n in counts.values())
    wl = inputs.WORKLOADS[workload]
    assert per_step == bench.launches_per_step(wl.mode, wl.T, wl)
