"""The multi-process host logic on CPU with two gloo ranks.

Batch images are independent in the forward and the backward (the input
gradient of image b only receives from image b), so ranks split the batch
with shard_range and exchange nothing on the data path.  This test runs two
ranks, each computing its shard with the fp64 oracle, gathers the shards on
the host and checks them against the whole batch, and checks the benchmark's
max-over-ranks timing reduction.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, result_q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        import synthetic_inputs as si
        from deformable_convolution_sampling_dcn_b200 import shard_range

        shape = si.CoreShape(B=5, H=7, W=6, G=2, C=4, dtype="f32", softmax=True)
        inp = si.core_inputs(shape, 21, with_grad_out=True)
        lo, hi = shard_range(shape.B, world, rank)
        mine = oracle.dcn_forward(inp["x"][lo:hi], inp["offset"][lo:hi], inp["mask"][lo:hi], G=2,
                                  softmax=True)
        gmine = oracle.dcn_backward(inp["x"][lo:hi], inp["offset"][lo:hi], inp["mask"][lo:hi],
                                    inp["grad_out"][lo:hi], G=2, softmax=True)["grad_x"]
        parts = [None] * world
        gparts = [None] * world
        dist.all_gather_object(parts, (lo, hi, mine))
        dist.all_gather_object(gparts, (lo, hi, gmine))
        slowest = bench.max_over_ranks(1.0 + rank, world)
        if rank == 0:
            full = oracle.dcn_forward(inp["x"], inp["offset"], inp["mask"], G=2, softmax=True)
            gfull = oracle.dcn_backward(inp["x"], inp["offset"], inp["mask"], inp["grad_out"], G=2,
                                        softmax=True)["grad_x"]
            cat = np.concatenate([p[2] for p in sorted(parts, key=lambda t: t[0])])
            gcat = np.concatenate([p[2] for p in sorted(gparts, key=lambda t: t[0])])
            result_q.put((np.array_equal(cat, full), np.array_equal(gcat, gfull), slowest,
                          [(p[0], p[1]) for p in parts]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_the_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world = 2
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    fwd_ok, bwd_ok, slowest, ranges = q.get(timeout=5)
    assert fwd_ok and bwd_ok
    assert slowest == 2.0
    assert ranges == [(0, 3), (3, 5)]


def test_reference_arm_under_two_ranks(tmp_path):
    """bench.py --impl reference launched as two ranks: rank 0 alone prints one
    JSON line, the other rank exits 0 without work."""
    import json
    import subprocess

    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
