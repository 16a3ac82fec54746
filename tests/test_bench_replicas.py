"""The multi-process host path of bench.py on CPU: two gloo ranks set up the
process group the way the GPU run does (from RANK / WORLD_SIZE / MASTER_*),
reduce their timings to the max over ranks, compute the whole-job value of
weak-scaled replicas, and leave the reference arm to rank 0 alone."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, os, sys
sys.path.insert(0, sys.argv[1])
import bench
world, rank, local = bench.dist_setup(2, backend="gloo")
ms = [1.0 + rank, 10.0 - rank, 3.0 * (rank + 1)]
got = bench.max_over_ranks(ms, world, device="cpu")
value = bench.replica_value(1_000_000_000, got[0], world)

class A:
    fmt = "base3"; M = 1; gpus = 2; steps = 1; warmup = 0; layers = 64; mode = "auto"
rc = bench.run_reference(A(), world, rank) if rank == 1 else 0
import torch.distributed as dist
dist.barrier()
dist.destroy_process_group()
print(json.dumps({"rank": rank, "world": world, "max": got, "value": value, "ref_rc": rc}))
"""


def test_two_gloo_ranks_reduce_max_and_gate_reference(tmp_path):
    script = tmp_path / "child.py"
    script.write_text(CHILD)
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(29511), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script), ROOT], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["world"] == 2
        assert o["max"] == [2.0, 10.0, 6.0]           # element-wise max over ranks
        assert o["value"] == pytest.approx(2 * 1.0 / 2e-3)  # 2 replicas x 1 GB per 2 ms
        assert o["ref_rc"] == 0                        # rank 1: the reference arm exits without work
