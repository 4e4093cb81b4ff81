"""The multi-process layout on CPU (two gloo ranks, world_size 2): the benchmark's harness
joins, synchronises and agrees on the max-over-ranks time that the throughput divides by;
and ranks that each run the decode step on their own sequences reproduce the one-process
result.  The data path has no collective: each rank's work is independent (weak scaling)."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import json, os, sys, time
sys.path.insert(0, os.environ["CSA_ROOT"])
import bench
d = bench.Dist()
rank = d.rank
d.barrier()
local = 10.0 * (rank + 1)          # rank 1 is the slowest
m = d.max(local)
d.barrier()
print(json.dumps({"rank": rank, "world": d.world, "max": m,
                  "value": 32 * d.world * 5 / (m / 1e3)}), flush=True)
d.close()
"""


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_two_gloo_ranks_agree_on_max_time(tmp_path):
    script = tmp_path / "worker.py"
    script.write_text(WORKER)
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, CSA_ROOT=ROOT, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2",
                   RANK=str(r), LOCAL_RANK=str(r), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        o, e = p.communicate(timeout=120)
        assert p.returncode == 0, e
        outs.append(json.loads(o.strip().splitlines()[-1]))
    assert {o["rank"] for o in outs} == {0, 1}
    for o in outs:
        assert o["world"] == 2 and o["max"] == 20.0
        assert abs(o["value"] - 32 * 2 * 5 / 0.02) < 1e-6


SHARD_WORKER = r"""
import json, os, sys
sys.path.insert(0, os.environ["CSA_ROOT"])
import numpy as np
import bench
import oracle
from compressed_sparse_long_02_b200 import synth
d = bench.Dist()
wl = synth.WORKLOADS["csa_decode_128k"].replace(k=16, W=8)
inp = synth.decode_inputs(wl, B=6, E=64)
kp, ks = oracle.mxfp4_quantize(inp["ki"])
qp, qs = oracle.mxfp4_quantize(inp["qi"])
seqs = np.arange(6)[d.rank::d.world]           # this rank's shard of the sequences
r = oracle.csa_decode(wl, inp["entries"], kp, ks, inp["q"], qp, qs, inp["w"], inp["window"], inp["pos"], seqs=seqs)
mine = {"seqs": seqs.tolist(), "idx": r["idx"].tolist(), "cnt": r["cnt"].tolist(),
        "out": r["out"].astype(np.float64).tobytes().hex()}
got = [None] * d.world
d.pg.all_gather_object(got, mine)              # the check only: the shards never exchange data
ok = True
if d.rank == 0:
    full = oracle.csa_decode(wl, inp["entries"], kp, ks, inp["q"], qp, qs, inp["w"], inp["window"], inp["pos"])
    seen = []
    for g in got:
        s = np.array(g["seqs"])
        seen += g["seqs"]
        out = np.frombuffer(bytes.fromhex(g["out"]), dtype=np.float64).reshape(len(s), wl.H, wl.D)
        ok &= np.array_equal(np.array(g["idx"]), full["idx"][s]) and np.array_equal(np.array(g["cnt"]), full["cnt"][s])
        ok &= np.array_equal(out, full["out"][s].astype(np.float64))
    ok &= sorted(seen) == list(range(6))
print(json.dumps({"rank": d.rank, "ok": bool(ok), "shard": seqs.tolist()}), flush=True)
d.close()
"""


def test_two_gloo_ranks_each_run_their_own_decode_shard(tmp_path):
    """Each rank runs the decode step (the oracle's indexer, top-k and attention) on its own
    sequences, with no exchange on the data path; the shards, gathered only to check them,
    reproduce the one-process result row for row and cover every sequence once."""
    script = tmp_path / "shard_worker.py"
    script.write_text(SHARD_WORKER)
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, CSA_ROOT=ROOT, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2",
                   RANK=str(r), LOCAL_RANK=str(r), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        o, e = p.communicate(timeout=300)
        assert p.returncode == 0, e
        outs.append(json.loads(o.strip().splitlines()[-1]))
    by_rank = {o["rank"]: o for o in outs}
    assert by_rank[0]["shard"] == [0, 2, 4] and by_rank[1]["shard"] == [1, 3, 5]
    assert by_rank[0]["ok"]
