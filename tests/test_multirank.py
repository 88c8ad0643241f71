"""The benchmark's multi-rank plumbing on CPU: two gloo ranks (one process each, as torchrun starts them).
Each rank runs its own replica on its own seed, the job time is the slowest rank's, and the reference arm
does its work on rank 0 only."""
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = textwrap.dedent("""
    import json, os, sys, io, contextlib
    sys.path.insert(0, {root!r})
    import torch.distributed as dist
    import bench, mate_inputs as mi
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", init_method="env://")
    cfg = mi.CONFIGS["bf16_256x32x32"]
    seed = bench.replica_seed(cfg, rank)
    ms = bench.max_over_ranks(2.0 + rank, world, "cpu")      # rank 1 is the slow one
    seeds = [None] * world
    dist.all_gather_object(seeds, seed)
    class A:   # the reference arm's arguments
        config = "tiny_f32_4x8x8"; oracle_frames = 2; steps = 1; warmup = 0; gpus = world
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        rc = bench.reference_arm(A, rank)
    dist.barrier()
    dist.destroy_process_group()
    print(json.dumps({{"rank": rank, "ms": ms, "seeds": seeds, "value": bench.job_value(1000, world, ms),
                      "rc": rc, "printed": out.getvalue().strip()}}))
""")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks():
    pytest.importorskip("torch")
    import json
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        o, e = p.communicate(timeout=240)
        assert p.returncode == 0, e[-2000:]
        outs.append(json.loads(o.strip().splitlines()[-1]))
    outs.sort(key=lambda d: d["rank"])
    for d in outs:
        assert d["ms"] == 3.0                           # the slowest rank's time on every rank
        assert d["value"] == pytest.approx(1000 * 2 / 3.0e-3)
        assert len(set(d["seeds"])) == 2                # distinct replica inputs
        assert d["rc"] == 0
    line = json.loads(outs[0]["printed"])               # the reference arm prints on rank 0 only
    assert line["impl"] == "reference" and line["value"] > 0
    assert outs[1]["printed"] == ""
