"""Seeded synthetic inputs for the CSA / HCA workloads.

This module only draws random numbers and rounds them once to the storage
dtype; it holds none of the layer's arithmetic.  Both the CUDA path (tests,
bench) and the CPU oracle take their inputs from here, so both see identical
bytes.

Workloads (shapes from the five configurations the pages' long-context setting
implies; see the CSA/HCA paragraphs of "Follow the white rabbit: DeepSeek V4's
architecture in 3D" and section 2.3 / section 4 of the "DeepSeek-V4: Towards
Highly Efficient Million-Token Context Intelligence" summary):

* ``tiny``            CSA prefill, T=512, C=D=128, fp32, 16 heads, 4 indexer heads of 64.
* ``csa_prefill_8k``  CSA prefill, T=8192, C=D=512, bf16, 64 heads, 64 indexer heads of 128.
* ``csa_decode_128k`` CSA decode, 32 sequences x 1 query at context 131072 (32768 entries).
* ``hca_prefill_64k`` HCA prefill, T=65536, m'=128 (512 entries), 64 heads of 512.
* ``csa_decode_1m``   CSA decode, 4 sequences x 1 query at context 1048576 (262144 entries).

Distribution convention: N(mu, var) names the variance (so "N(0, 1/128)" has
standard deviation 1/sqrt(128)).  Unstated distributions are readings: logits
N(0,1), slot bias N(0,0.1), head weights U(0,1), raw indexer keys N(0,1).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = ["Workload", "WORKLOADS", "prefill_inputs", "prefill_inputs_torch", "decode_inputs",
           "decode_inputs_torch", "to_dtype_np", "ProjShape", "PROJ", "proj_inputs", "proj_inputs_torch"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "csa_prefill" | "csa_decode" | "hca_prefill"
    seed: int
    dtype: str           # storage dtype of activations: "f32" | "bf16"
    C: int               # KV latent / head dim (C == D)
    H: int               # query heads
    rope_dims: int       # partial RoPE on the last rope_dims channels
    norm: bool           # RMSNorm on q, entries and window rows
    m: int               # tokens per compressed entry
    overlap: bool        # entry also pools the previous group (CSA)
    W: int               # sliding window of raw tokens
    T: int = 0           # tokens per sequence (prefill)
    B: int = 1           # sequences
    L: int = 0           # context length (decode)
    Hi: int = 0          # indexer heads
    Di: int = 0          # indexer head dim
    k: int = 0           # top-k entries per query
    boost_frac: float = 0.0   # decode 1M: fraction of entries whose raw indexer keys get +boost
    boost: float = 0.0
    q_var: float = 1.0   # variance of raw queries
    bias_var: float = 0.1
    eps: float = 1e-6
    theta: float = 10000.0

    @property
    def D(self) -> int:
        return self.C

    @property
    def E(self) -> int:
        """Compressed entries per sequence: floor(L/m) (decode) or floor(T/m) (prefill)."""
        n = self.L if self.kind == "csa_decode" else self.T
        return n // self.m

    @property
    def slots(self) -> int:
        return self.m * (2 if self.overlap else 1)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload(name="tiny", kind="csa_prefill", seed=0, dtype="f32", C=128, H=16,
                     rope_dims=32, norm=False, m=4, overlap=True, W=64, T=512, Hi=4, Di=64,
                     k=32, q_var=1.0 / 128.0),
    "csa_prefill_8k": Workload(name="csa_prefill_8k", kind="csa_prefill", seed=2, dtype="bf16",
                               C=512, H=64, rope_dims=64, norm=True, m=4, overlap=True, W=128,
                               T=8192, Hi=64, Di=128, k=512),
    "csa_decode_128k": Workload(name="csa_decode_128k", kind="csa_decode", seed=3, dtype="bf16",
                                C=512, H=64, rope_dims=64, norm=True, m=4, overlap=True, W=128,
                                B=32, L=131072, Hi=64, Di=128, k=1024),
    "hca_prefill_64k": Workload(name="hca_prefill_64k", kind="hca_prefill", seed=4, dtype="bf16",
                                C=512, H=64, rope_dims=64, norm=True, m=128, overlap=False, W=128,
                                T=65536),
    "csa_decode_1m": Workload(name="csa_decode_1m", kind="csa_decode", seed=5, dtype="bf16",
                              C=512, H=64, rope_dims=64, norm=True, m=4, overlap=True, W=128,
                              B=4, L=1048576, Hi=64, Di=128, k=1024, boost_frac=0.01, boost=3.0),
}


def to_dtype_np(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 samples once to the storage dtype.

    Returns float32 for "f32" and the raw uint16 bit pattern for "bf16"
    (round-to-nearest-even, as torch rounds)."""
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        import torch
        t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(torch.bfloat16)
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    raise ValueError(dtype)


def _normal(rng: np.random.Generator, shape, var: float = 1.0) -> np.ndarray:
    return rng.standard_normal(shape) * math.sqrt(var)


def prefill_inputs(wl: Workload, T: int | None = None, B: int | None = None) -> dict:
    """Host inputs of a prefill workload (CSA or HCA), drawn in float64 and rounded once.

    Keys: kv, z [B,T,C]; bias [slots,C] f32; q [B,T,H,C]; and for CSA the
    indexer inputs qi [B,T,Hi,Di], ki [B,T,Di], zi [B,T,Di], bias_i [slots,Di] f32,
    w [B,T,Hi] f32.  Activations are f32 or bf16 bit patterns (uint16)."""
    T = wl.T if T is None else T
    B = wl.B if B is None else B
    rng = np.random.default_rng(wl.seed)
    C, H = wl.C, wl.H
    out = {
        "kv": to_dtype_np(_normal(rng, (B, T, C)), wl.dtype),
        "z": to_dtype_np(_normal(rng, (B, T, C)), wl.dtype),
        "bias": _normal(rng, (wl.slots, C), wl.bias_var).astype(np.float32),
        "q": to_dtype_np(_normal(rng, (B, T, H, C), wl.q_var), wl.dtype),
    }
    if wl.kind == "csa_prefill":
        Hi, Di = wl.Hi, wl.Di
        out["qi"] = to_dtype_np(_normal(rng, (B, T, Hi, Di)), wl.dtype)
        out["ki"] = to_dtype_np(_normal(rng, (B, T, Di)), wl.dtype)
        out["zi"] = to_dtype_np(_normal(rng, (B, T, Di)), wl.dtype)
        out["bias_i"] = _normal(rng, (wl.slots, Di), wl.bias_var).astype(np.float32)
        out["w"] = rng.uniform(0.0, 1.0, (B, T, Hi)).astype(np.float32)
    return out


def prefill_inputs_torch(wl: Workload, device, T: int | None = None, replica: int = 0) -> dict:
    """Prefill inputs drawn directly on ``device`` (same keys, shapes and distributions as
    :func:`prefill_inputs`, torch dtypes) for the workloads too large to draw on the host."""
    import torch
    T = wl.T if T is None else T
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed * 7919 + 17 + replica)
    act = torch.float32 if wl.dtype == "f32" else torch.bfloat16

    def nrm(shape, var=1.0):
        return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * math.sqrt(var)).to(act)

    C, H = wl.C, wl.H
    out = {"kv": nrm((1, T, C)), "z": nrm((1, T, C)),
           "bias": torch.randn((wl.slots, C), generator=g, device=device) * math.sqrt(wl.bias_var),
           "q": nrm((1, T, H, C), wl.q_var)}
    if wl.kind == "csa_prefill":
        out["qi"] = nrm((1, T, wl.Hi, wl.Di))
        out["ki"] = nrm((1, T, wl.Di))
        out["zi"] = nrm((1, T, wl.Di))
        out["bias_i"] = torch.randn((wl.slots, wl.Di), generator=g, device=device) * math.sqrt(wl.bias_var)
        out["w"] = torch.rand((1, T, wl.Hi), generator=g, device=device)
    return out


def decode_inputs(wl: Workload, B: int | None = None, E: int | None = None, seed_offset: int = 0) -> dict:
    """Host inputs of a decode workload at reduced size (for the oracle-sized parity cases).

    Keys: entries [B,E,D] bf16 bits; ki [B,E,Di] f32 raw indexer keys (to be
    MXFP4-quantised); q [B,H,D] bf16; qi [B,Hi,Di] f32; w [B,Hi] f32;
    window [B,W,D] bf16; pos [B] int64 (query position = E*m - 1)."""
    B = wl.B if B is None else B
    E = wl.E if E is None else E
    rng = np.random.default_rng(wl.seed + 1000 * seed_offset)
    D, H, Hi, Di, W = wl.D, wl.H, wl.Hi, wl.Di, wl.W
    ki = _normal(rng, (B, E, Di))
    if wl.boost_frac > 0:
        n_boost = max(1, int(round(wl.boost_frac * E)))
        for b in range(B):
            sel = rng.choice(E, size=n_boost, replace=False)
            ki[b, sel, :] += wl.boost
    return {
        "entries": to_dtype_np(_normal(rng, (B, E, D)), "bf16"),
        "ki": ki.astype(np.float32),
        "q": to_dtype_np(_normal(rng, (B, H, D)), "bf16"),
        "qi": _normal(rng, (B, Hi, Di)).astype(np.float32),
        "w": rng.uniform(0.0, 1.0, (B, Hi)).astype(np.float32),
        "window": to_dtype_np(_normal(rng, (B, W, D)), "bf16"),
        "pos": np.full((B,), E * wl.m - 1, dtype=np.int64),
    }


def decode_inputs_torch(wl: Workload, device, B: int | None = None, E: int | None = None,
                        replica: int = 0) -> dict:
    """Full-size decode inputs drawn directly on ``device`` with a seeded torch generator.

    Same keys and dtypes as :func:`decode_inputs` but as torch tensors (bf16 /
    float32), for the workloads whose caches are too large to draw on the host.
    ``replica`` selects an independent draw (distinct seed)."""
    import torch
    B = wl.B if B is None else B
    E = wl.E if E is None else E
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed * 7919 + replica)
    D, H, Hi, Di, W = wl.D, wl.H, wl.Hi, wl.Di, wl.W
    ki = torch.randn((B, E, Di), generator=g, device=device, dtype=torch.float32)
    if wl.boost_frac > 0:
        n_boost = max(1, int(round(wl.boost_frac * E)))
        for b in range(B):
            sel = torch.randperm(E, generator=g, device=device)[:n_boost]
            ki[b, sel, :] += wl.boost
    return {
        "entries": torch.randn((B, E, D), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16),
        "ki": ki,
        "q": torch.randn((B, H, D), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16),
        "qi": torch.randn((B, Hi, Di), generator=g, device=device, dtype=torch.float32),
        "w": torch.rand((B, Hi), generator=g, device=device, dtype=torch.float32),
        "window": torch.randn((B, W, D), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16),
        "pos": torch.full((B,), E * wl.m - 1, dtype=torch.int32, device=device),
    }


# ----------------------------------------------------------------------------- output projection
@dataclasses.dataclass(frozen=True)
class ProjShape:
    """Grouped output projection after core attention (the pages name it, "DeepSeek-V4:
    Towards Highly Efficient ..." section 2.3, without sizes): H heads of D in G groups,
    R values per group, then d_model.  R and d_model are synthetic choices."""
    T: int
    H: int = 64
    D: int = 512
    G: int = 8
    R: int = 1024
    d_model: int = 4096
    seed: int = 6


PROJ = {"tiny": ProjShape(T=37, H=16, D=128, G=4, R=256, d_model=512),
        "csa_prefill_8k": ProjShape(T=8192)}


def proj_inputs(ps: ProjShape, T: int | None = None) -> dict:
    """Host inputs (bf16 bits): o [T, H, D] ~ N(0,1); A [G, R, (H/G) D] ~ N(0, 1/((H/G) D));
    Bm [d_model, G R] ~ N(0, 1/(G R)), so the intermediate and the output are ~N(0,1)."""
    T = ps.T if T is None else T
    rng = np.random.default_rng(ps.seed)
    Kg = (ps.H // ps.G) * ps.D
    return {"o": to_dtype_np(_normal(rng, (T, ps.H, ps.D)), "bf16"),
            "A": to_dtype_np(_normal(rng, (ps.G, ps.R, Kg), 1.0 / Kg), "bf16"),
            "Bm": to_dtype_np(_normal(rng, (ps.d_model, ps.G * ps.R), 1.0 / (ps.G * ps.R)), "bf16")}


def proj_inputs_torch(ps: ProjShape, device, T: int | None = None) -> dict:
    """The same shapes and distributions drawn on ``device`` (bf16 tensors)."""
    import torch
    T = ps.T if T is None else T
    g = torch.Generator(device=device)
    g.manual_seed(ps.seed * 7919 + 31)
    Kg = (ps.H // ps.G) * ps.D

    def nrm(shape, var=1.0):
        return (torch.randn(shape, generator=g, device=device) * math.sqrt(var)).to(torch.bfloat16)

    return {"o": nrm((T, ps.H, ps.D)), "A": nrm((ps.G, ps.R, Kg), 1.0 / Kg),
            "Bm": nrm((ps.d_model, ps.G * ps.R), 1.0 / (ps.G * ps.R))}
