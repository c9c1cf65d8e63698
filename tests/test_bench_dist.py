"""The bench's multi-process plumbing on CPU: two ranks over gloo, launched the way a
launcher would (RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* in the environment).

The path shards as independent replicas (each rank denoises its own canvases), so the
only cross-rank steps are the barriers around the timed region and the max over ranks
of the device time; the whole-job value is world x units per rank / slowest rank.
"""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, os, sys
sys.path.insert(0, os.environ["REPO"])
import bench
from masked_discrete_diffusion_b200 import build

calls = []
build.build = lambda *a, **k: calls.append(1)
world, rank, local = bench.dist_setup("gloo")
bench.build_once(world, local)
# each rank reports its own time; everyone must see the slowest
ms = 100.0 + 50.0 * rank
ms_max = bench.max_over_ranks(ms, world)
value = bench.job_throughput(world, 256, 3, ms_max)
bench.barrier(world)
# the reference arm runs on rank 0 only: another rank returns at once, printing nothing
class A: steps = 1; warmup = 0; gpus = world
if rank != 0:
    bench.run_reference(A, None, world, rank)
print(json.dumps({"rank": rank, "world": world, "ms_max": ms_max, "value": value,
                  "built": len(calls)}), flush=True)
import torch.distributed as dist
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_gloo_max_over_ranks_and_value():
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), REPO=ROOT,
                   CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", CHILD], env=env, cwd=ROOT,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                      text=True))
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=120)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
        assert p.returncode == 0, e
        lines = [ln for ln in o.splitlines() if ln.startswith("{")]
        assert len(lines) == 1, o
        outs.append(json.loads(lines[0]))
    outs.sort(key=lambda d: d["rank"])
    for d in outs:
        assert d["world"] == 2
        assert d["ms_max"] == 150.0                      # the slowest rank's time
        assert abs(d["value"] - 2 * 256 * 3 / 0.150) < 1e-6
    # only local rank 0 builds; the other rank waited at the barrier
    assert [d["built"] for d in outs] == [1, 0]


def test_job_throughput_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_throughput(1, 256, 5, 1000.0) == 256 * 5
    assert bench.max_over_ranks(3.5, 1) == 3.5
