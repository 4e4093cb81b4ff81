"""Rules the kernel sources keep, checked by reading them (no GPU needed).

* No TMA or bulk load with cluster multicast: the multi-GPU path (one rank per GPU)
  must never issue one, and no kernel here needs one.
* Every mbarrier wait goes through the bounded helpers (a raw `mbarrier.try_wait` loop
  outside ptx.cuh could spin for ever when an arrival is lost).
* Kernels reach the legacy tensor-core path nowhere (`mma.sync`, `wmma`): contractions
  are tcgen05.
"""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "compressed_sparse_long_02_b200", "csrc")


def _sources():
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(CSRC, name)) as f:
                yield name, f.read()


def _code(text: str) -> str:
    """The source without // comments (string literals of inline PTX stay)."""
    return "\n".join(line.split("//", 1)[0] for line in text.splitlines())


def test_no_multicast_loads():
    for name, text in _sources():
        code = _code(text)
        for m in re.finditer(r'"[^"]*cp\.async\.bulk[^"]*"', code):
            assert "multicast" not in m.group(0), f"{name}: multicast bulk copy {m.group(0)}"


def test_mbarrier_waits_only_in_the_bounded_helpers():
    for name, text in _sources():
        if name == "ptx.cuh":
            continue
        assert "mbarrier.try_wait" not in _code(text), f"{name}: raw mbarrier wait outside the bounded helpers"


def test_tensor_core_path_is_tcgen05():
    for name, text in _sources():
        code = _code(text)
        assert "mma.sync" not in code and "wmma::" not in code, f"{name}: legacy tensor-core instruction"
