"""The multi-rank host logic of bench.py on the CPU: two ranks over gloo.

The decode path shards by sequence with no collective in its data path; what more than one rank
adds is the timing rule (the slowest rank's time, known to every rank), the agreement on whether
to measure again, and a reference arm that only rank 0 runs and prints.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_WORKER = r"""
import os, sys, json, datetime
sys.path.insert(0, {root!r})
import torch.distributed as dist
import bench
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
t = bench.max_over_ranks([3.5, 7.25][rank], world)             # per-rank timings
flag = bench.max_over_ranks(1.0 if rank == 1 else 0.0, world)   # raised on rank 1 only
calm = bench.max_over_ranks(0.0, world)                          # raised nowhere
dist.barrier()
dist.destroy_process_group()
print(json.dumps(dict(rank=rank, t=t, flag=flag, calm=calm)), flush=True)
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_max_over_ranks_two_gloo_ranks():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                   CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", _WORKER.format(root=ROOT)], env=env, cwd=ROOT,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["t"] == 7.25          # every rank reports the slowest rank's time
        assert o["flag"] == 1.0        # one rank's rejected clocks make every rank measure again
        assert o["calm"] == 0.0


def test_max_over_ranks_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(2.5, 1) == 2.5


@pytest.mark.slow
def test_reference_arm_under_torchrun_prints_once_from_rank_0():
    """`bench.py --impl reference` launched like the multi-GPU runs (torchrun, two ranks): rank 0
    times the oracle and prints one JSON line; rank 1 exits 0 without work or output."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "smallem_fp32"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="1")
    res = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-3000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["n_gpus"] == 2
    assert line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
