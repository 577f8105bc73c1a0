"""The bench's multi-rank host path on CPU: two `gloo` ranks as child processes.

With N GPUs the bench runs N independent replicas (no data-path collective); the
only cross-rank steps are the rendezvous, the barriers around the timed region and
the max over ranks of the timed duration.  This runs those helpers of bench.py with
world size 2 on the host."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, os, sys, time
sys.path.insert(0, {root!r})
import bench
rank, local, ws = bench.dist_setup("gloo")
bench.dist_barrier()
mine = 1.5 + 2.0 * rank          # a rank-dependent "duration"
got = bench.dist_max(mine)
bench.dist_barrier()
print(json.dumps({{"rank": rank, "local": local, "ws": ws, "max": got}}), flush=True)
import torch.distributed as dist
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_agree_on_max_time():
    port = _free_port()
    code = CHILD.format(root=ROOT)
    procs = []
    for rank in range(2):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2", RANK=str(rank),
                   LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=120)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    assert sorted(o["rank"] for o in outs) == [0, 1]
    for o in outs:
        assert o["ws"] == 2 and o["local"] == o["rank"]
        assert o["max"] == 3.5          # max over ranks of 1.5 and 3.5, seen by both


def test_single_rank_needs_no_process_group():
    code = ("import sys; sys.path.insert(0, %r); import bench; "
            "print(bench.dist_setup('gloo'), bench.dist_max(2.5)); bench.dist_barrier()") % ROOT
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip() == "(0, 0, 1) 2.5"
