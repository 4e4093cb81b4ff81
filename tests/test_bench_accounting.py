"""The benchmark's algorithmic byte and FLOP counts, recounted independently.

Every roofline fraction `bench.py` reports divides these counts by a measured time, so a
wrong count would misreport every fraction.  Here each is rebuilt from the tensors a
call must touch (decode) or from a brute-force enumeration of the attended pairs
(prefill), on the workloads the benchmark runs.
"""
import numpy as np

import bench
from compressed_sparse_long_02_b200 import synth


def test_decode_bytes_from_tensor_shapes():
    wl = synth.WORKLOADS["csa_decode_128k"]
    tensors = {  # bytes per query of every tensor the decode step must read or write once
        "indexer keys (packed E2M1)": wl.E * wl.Di // 2,
        "indexer key scales (UE8M0 per 32)": wl.E * wl.Di // 32,
        "indexer query (float32)": wl.Hi * wl.Di * 4,
        "head weights (float32)": wl.Hi * 4,
        "selected entries (bf16)": wl.k * wl.D * 2,
        "window rows (bf16)": wl.W * wl.D * 2,
        "query (bf16)": wl.H * wl.D * 2,
        "output (bf16)": wl.H * wl.D * 2,
        "selected indices (int32)": wl.k * 4,
    }
    nb = bench.decode_bytes_per_query(wl)
    assert nb["step"] == sum(tensors.values())
    assert nb["step"] * wl.B == 114_434_048  # the 114.4 MB per step the benchmark reports
    attn = sum(v for k, v in tensors.items() if k.startswith(("selected", "window", "query (", "output")))
    assert nb["attention"] == attn


def _visible(t: np.ndarray, m: int, E: int) -> np.ndarray:
    return np.minimum((t + 1) // m, E)


def test_indexer_flops_by_enumeration():
    for name in ["csa_prefill_8k", "tiny"]:
        wl = synth.WORKLOADS[name]
        t = np.arange(wl.T)
        pairs = 0
        for q in range(wl.T):  # every (query, entry) pair the indexer scores
            pairs += sum(1 for j in range(wl.E) if m_pos(j, wl.m) <= q)
        assert pairs == int(_visible(t, wl.m, wl.E).sum())
        assert bench.indexer_flops(wl) == 2.0 * wl.Hi * wl.Di * pairs


def m_pos(j: int, m: int) -> int:
    """Position of compressed entry j: its last token."""
    return m * (j + 1) - 1


def test_attention_flops_by_enumeration():
    wl = synth.WORKLOADS["tiny"]
    keys = 0
    for q in range(wl.T):
        visible = sum(1 for j in range(wl.E) if m_pos(j, wl.m) <= q)
        selected = min(wl.k, visible)
        window = sum(1 for u in range(wl.T) if q - wl.W < u <= q)
        keys += selected + window
    assert bench.attention_flops(wl) == 4.0 * wl.H * wl.D * keys
