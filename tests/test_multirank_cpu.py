"""Host logic of `bench.py --gpus N` with two ranks on the CPU (gloo backend, world size 2).

The path shards without an exchange step: every rank draws its own seeded tensors and the only
collective is the max over ranks of the timings.  These tests run that logic in two processes.
"""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        from fp4_microscaling_tensor_b200 import inputs
        # timings: element-wise max over ranks
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 0.5 * rank], "cpu")
        # each rank draws its own tensors: checksums differ across ranks
        x = inputs.workload5_tensor(bench.rank_layer(0, rank), 2, shape=(64, 256))
        chk = torch.tensor([float(x.float().sum())], dtype=torch.float64)
        allc = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(allc, chk)
        # the reference arm: only rank 0 prints
        buf = io.StringIO()
        args = bench.parse(["--impl", "reference", "--gpus", str(world), "--steps", "1",
                            "--warmup", "0"])
        if rank != 0:
            with redirect_stdout(buf):
                bench.run_reference(args)
        out[rank] = (got, [float(c) for c in allc], buf.getvalue())
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    port = free_port()
    with mp.get_context("spawn").Manager() as m:  # no fork of this (threaded) process
        out = m.dict()
        mp.spawn(worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        got, checks, printed = res[rank]
        assert got == [2.0, 10.0, 0.5]
        assert checks[0] != checks[1]
        assert printed == ""


def test_single_process_identity():
    assert bench.max_over_ranks([3.0, 4.0], "cpu") == [3.0, 4.0]
    assert bench.rank_layer(0, 0) != bench.rank_layer(0, 1)


def shard_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        import oracle
        from fp4_microscaling_tensor_b200 import dist as mxdist, inputs
        # one tensor, split by rows: each rank reduces its shard with the oracle, then combines
        x = inputs.student_t4_rowgain((64, 512), 5)
        shard = x[rank * 32:(rank + 1) * 32]
        xo = inputs.to_oracle(shard)
        g_local = oracle.global_scale(xo, oracle.UE5M3)
        g = mxdist.combine_g_bits(g_local)
        st = oracle.error_stats(xo, 32, 512, 32, oracle.UE5M3, g)
        out[rank] = (g, mxdist.combine_stats(st))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_row_sharded_tensor_combines_to_whole():
    import oracle
    from fp4_microscaling_tensor_b200 import inputs
    world = 2
    port = free_port()
    with mp.get_context("spawn").Manager() as m:  # no fork of this (threaded) process
        out = m.dict()
        mp.spawn(shard_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    x = inputs.student_t4_rowgain((64, 512), 5)
    xo = inputs.to_oracle(x)
    g_whole = oracle.global_scale(xo, oracle.UE5M3)
    whole = oracle.error_stats(xo, 64, 512, 32, oracle.UE5M3, g_whole)
    for rank in range(world):
        g, st = res[rank]
        assert g == g_whole
        for k in ("numel", "n_blocks", "n_zero_blocks", "n_scale_sat", "n_elem_sat"):
            assert st[k] == whole[k], k
        for k in ("sse_elem", "sse_max", "sse_zero"):
            assert abs(st[k] - whole[k]) <= 1e-12 * max(abs(whole[k]), 1e-300), k
