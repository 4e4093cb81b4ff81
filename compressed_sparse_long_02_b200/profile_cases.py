"""One C-ABI call on seeded synthetic inputs, repeated a few times: the command line that
profiling captures (ncu) and timing runs share.

    python -m compressed_sparse_long_02_b200.profile_cases CASE [--reps N]

Cases (inputs larger than the 126 MB L2 where the call is memory-bound, so that DRAM
counters mean something, and a few GB on the device at most):

  pool_csa_64k      csa_compress, CSA (m=4, overlap), T=65536, C=512 bf16, entries + window rows
  pool_hca_64k      csa_compress, HCA (m'=128), T=65536, C=512 bf16, entries + window rows
  norm_rope_q_2k    csa_norm_rope of 2048 query rows x 64 heads x 512 (bf16)
  quantize_qi_8k    csa_quantize_mxfp4 of 8192 x 64 x 128 bf16 indexer queries
  decode_128k       the 128K decode step's indexer, top-k and attention calls (32 queries)
  attn_csa_4k       csa_sparse_attn_ex of 4096 raw prefill queries (k=512, W=128) over 1024 entries
  attn_hca_8k       hca_attn_ex of 8192 raw prefill queries over 64 entries + the 128-token window
  attn_hca_64k_tail hca_attn_ex of the last 1184 raw queries of a 65536-token prefill (503-512
                    entries + the window each: the persistent tile-resident path of the 64K layer)
  proj_2k           csa_grouped_out_proj of 2048 tokens (64 heads of 512, 8 groups, R=1024, 4096)
"""
from __future__ import annotations

import argparse
import sys

CASES = ["pool_csa_64k", "pool_hca_64k", "norm_rope_q_2k", "quantize_qi_8k", "decode_128k", "attn_csa_4k",
         "attn_hca_8k", "attn_hca_64k_tail", "proj_2k"]


def run(case: str, reps: int) -> None:
    import torch

    from . import binding as B
    from . import layer, synth
    dev = torch.device("cuda:0")
    B.lib()
    if case in ("pool_csa_64k", "pool_hca_64k"):
        wl = synth.WORKLOADS["csa_prefill_8k" if case == "pool_csa_64k" else "hca_prefill_64k"].replace(T=65536)
        g = torch.Generator(device=dev)
        g.manual_seed(wl.seed)
        kv = torch.randn((1, wl.T, wl.C), generator=g, device=dev).to(torch.bfloat16)
        z = torch.randn((1, wl.T, wl.C), generator=g, device=dev).to(torch.bfloat16)
        bias = torch.randn((wl.slots, wl.C), generator=g, device=dev) * wl.bias_var ** 0.5
        fn = lambda: B.csa_compress(kv, z, bias, m=wl.m, overlap=wl.overlap, norm=wl.norm, eps=wl.eps,
                                    rope_dims=wl.rope_dims, theta=wl.theta, want_window=True)
    elif case == "norm_rope_q_2k":
        wl = synth.WORKLOADS["csa_prefill_8k"]
        q = torch.randn((2048, 64, 512), device=dev).to(torch.bfloat16)
        pos = torch.arange(2048, dtype=torch.int32, device=dev)
        fn = lambda: B.csa_norm_rope(q, pos, norm=True, eps=wl.eps, rope_dims=wl.rope_dims, theta=wl.theta)
    elif case == "quantize_qi_8k":
        x = torch.randn((8192, 64, 128), device=dev).to(torch.bfloat16)
        fn = lambda: B.csa_quantize_mxfp4(x)
    elif case == "decode_128k":
        wl = synth.WORKLOADS["csa_decode_128k"]
        d = synth.decode_inputs_torch(wl, dev)
        kp, ks = B.csa_quantize_mxfp4(d["ki"])
        del d["ki"]
        cache = {"entries": d["entries"], "k_fp4": kp, "k_scale": ks, "window": d["window"],
                 "window_base": (d["pos"] - wl.W + 1).to(torch.int32),
                 "n_entries": torch.full((wl.B,), wl.E, dtype=torch.int32, device=dev)}
        step = {"q": d["q"], "qi": d["qi"], "w": d["w"], "pos": d["pos"]}
        fn = lambda: layer.csa_decode(wl, cache, step)
    elif case in ("attn_csa_4k", "attn_hca_8k"):
        T = 4096 if case == "attn_csa_4k" else 8192
        wl = synth.WORKLOADS["csa_prefill_8k" if case == "attn_csa_4k" else "hca_prefill_64k"].replace(T=T)
        t = synth.prefill_inputs_torch(wl, dev)
        r = (layer.csa_prefill if wl.kind == "csa_prefill" else layer.hca_prefill)(wl, t)
        pos = torch.arange(T, dtype=torch.int32, device=dev)
        seq = torch.zeros(T, dtype=torch.int32, device=dev)
        zero = torch.zeros(1, dtype=torch.int32, device=dev)
        ne = torch.tensor([wl.E], dtype=torch.int32, device=dev)
        if wl.kind == "csa_prefill":
            fn = lambda: B.csa_sparse_attn(r["q"], pos, seq, r["entries"], r["idx"], r["cnt"], r["window"], zero,
                                           W=wl.W, out=r["out"], prep=layer.q_prep(wl))
        else:
            fn = lambda: B.hca_attn(r["q"], pos, seq, r["entries"], ne, r["window"], zero, mprime=wl.m, W=wl.W,
                                    out=r["out"], prep=layer.q_prep(wl))
    elif case == "attn_hca_64k_tail":
        wl = synth.WORKLOADS["hca_prefill_64k"]
        n, T, W = 1184, wl.T, wl.W
        g = torch.Generator(device=dev)
        g.manual_seed(wl.seed + 7)
        q = torch.randn((n, wl.H, wl.D), generator=g, device=dev).to(torch.bfloat16)
        entries = torch.randn((1, wl.E, wl.D), generator=g, device=dev).to(torch.bfloat16)
        base = T - n - W + 1  # the window buffer holds tokens base .. T - 1
        window = torch.randn((1, T - base, wl.D), generator=g, device=dev).to(torch.bfloat16)
        pos = torch.arange(T - n, T, dtype=torch.int32, device=dev)
        seq = torch.zeros(n, dtype=torch.int32, device=dev)
        wb = torch.tensor([base], dtype=torch.int32, device=dev)
        ne = torch.tensor([wl.E], dtype=torch.int32, device=dev)
        out = torch.empty_like(q)
        fn = lambda: B.hca_attn(q, pos, seq, entries, ne, window, wb, mprime=wl.m, W=W, out=out,
                                prep=layer.q_prep(wl))
    elif case == "proj_2k":
        ps = synth.PROJ["csa_prefill_8k"]
        d = synth.proj_inputs_torch(ps, dev, T=2048)
        fn = lambda: B.csa_grouped_out_proj(d["o"], d["A"], d["Bm"])
    else:
        raise SystemExit(f"unknown case {case}; one of {', '.join(CASES)}")
    for _ in range(reps):
        fn()
    torch.cuda.synchronize()
    err = B.csa_get_device_error()
    if err != 0:
        raise SystemExit(f"device error word {err}")
    print(f"{case}: {reps} calls ok")


def main(argv=None) -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=CASES)
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args(argv)
    run(a.case, a.reps)


if __name__ == "__main__":
    main(sys.argv[1:])
