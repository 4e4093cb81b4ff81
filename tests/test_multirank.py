"""The benchmark's multi-process harness on CPU: two gloo ranks (world_size 2) join,
synchronise, and agree on the max-over-ranks time that the throughput divides by.
The data path has no collective: each rank's work is independent (weak scaling)."""
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
