"""Host logic of the N > 1 benchmark path on CPU: world_size-2 gloo ranks.

The timing reduction takes the maximum over ranks, every rank draws its own token
batches while sharing W, and under torchrun the reference arm runs on rank 0 only
(the other rank exits 0 without work).
"""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sys.path.insert(0, ROOT)
        import bench
        from workloads import synth
        got = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        cfg = bench.rank_config(synth.scaled_config("tiny_fwd"), rank)
        x = synth.batch_matrix(cfg, "X", 0)
        w = synth.operand_matrix(synth.scaled_config("tiny_fwd"), "W")
        xs = [torch.zeros_like(x) for _ in range(world)]
        ws = [torch.zeros_like(w) for _ in range(world)]
        dist.all_gather(xs, x)
        dist.all_gather(ws, w)
        out[rank] = (got, bool(torch.equal(xs[0], xs[1])), bool(torch.equal(ws[0], ws[1])))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_per_rank_batches():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in (0, 1):
        got, same_x, same_w = res[rank]
        assert got == 2.5                 # the maximum over ranks, on every rank
        assert not same_x                 # each rank its own tokens
        assert same_w                     # one shared weight


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--config", "tiny_fwd",
           "--ref-rows", "64", "--ref-cols", "128"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1                # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
