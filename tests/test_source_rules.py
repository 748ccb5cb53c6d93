"""Source rules of the CUDA code that every later change must keep (CPU only):
no TMA or bulk copy carries the cluster-multicast qualifier (each copy lands in
the issuing CTA's own shared memory, so no path can read another GPU's memory
through a multicast load), and tensor-map copies are issued only through the
wrappers in tc_ptx.cuh, the one place to review their coordinates."""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "nvfp4_mixture_experts_grouped_b200", "csrc")
QUALIFIER = ".multi" + "cast"  # spelled in two pieces so this file names no such copy


def _sources():
    for path in sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))):
        yield path, open(path).read()


def test_no_bulk_or_tensor_copy_is_multicast():
    for path, src in _sources():
        for i, line in enumerate(src.splitlines(), 1):
            if "cp.async.bulk" in line or "cp.reduce.async.bulk" in line:
                assert QUALIFIER not in line, f"{os.path.basename(path)}:{i}: {line.strip()}"


def test_the_only_multicast_is_the_tcgen05_commit():
    for path, src in _sources():
        for i, line in enumerate(src.splitlines(), 1):
            if QUALIFIER in line:
                assert "tcgen05.commit" in line, f"{os.path.basename(path)}:{i}: {line.strip()}"


def test_tensor_map_copies_take_their_coordinates_from_the_wrappers():
    for path, src in _sources():
        if os.path.basename(path) == "tc_ptx.cuh":
            continue
        assert not re.search(r"cp\.async\.bulk\.tensor", src), os.path.basename(path)
