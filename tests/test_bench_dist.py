"""Host logic of bench.py's multi-rank path, on CPU with the gloo backend (world size 2).

Each rank of a multi-GPU run owns a shard of the weight rows of one tall matrix
(x replicated); the reported time is the maximum over ranks and the value is
the work of all ranks over that time.  The shard split and the reassembly of y
are checked with the CPU oracle standing in for the kernel.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    import datetime
    import torch.distributed as dist
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, lr, w = bench.dist_env()
        seconds = 0.5 + rank          # rank 1 is the slow one
        slowest = bench.max_over_ranks(seconds, w, device="cpu")
        value = bench.aggregate(100.0, w, slowest)
        dist.barrier()
        out.put((r, lr, w, slowest, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    got = sorted(q.get(timeout=10) for _ in range(world))
    for r, (rank, local_rank, w, slowest, value) in enumerate(got):
        assert (rank, local_rank, w) == (r, r, world)
        assert slowest == pytest.approx(1.5)          # the max, not the caller's own time
        assert value == pytest.approx(200.0 / 1.5)    # both ranks' work over the slowest time


def test_single_rank_helpers():
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.aggregate(10.0, 1, 2.0) == 5.0
    # every copy is used exactly once per cycle of n_copies launches
    n, per = 12, 3
    seen = [bench.rotation(n, per, step, j) for step in range(4) for j in range(per)]
    assert sorted(seen) == list(range(n))


def _shard_main(rank: int, world: int, port: int, rows: int, K: int, out):
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist
    import oracle
    from bit_quantized_gemm_quant_b200 import inputs
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # this rank's rows of the tall matrix, x replicated (the same seed on every rank)
        w = inputs.weights_fp32(rows, K, inputs.generator(bench.shard_seed(0, rank))).numpy()
        wq, d = oracle.q4_0_quantize(w)
        x = inputs.activations_bf16(3, K, inputs.generator(1)).view(torch.int16).numpy().view(np.uint16)
        y, _, _ = oracle.matmul_ref(x, oracle.q4_0_dequantize(wq, d), nthreads=1)
        shard = torch.from_numpy(np.ascontiguousarray(y))
        parts = [torch.empty_like(shard) for _ in range(world)]
        dist.all_gather(parts, shard)
        full = bench.assemble_shards(parts)
        out.put((rank, bench.shard_rows(rows, rank), full.numpy()))
    finally:
        dist.destroy_process_group()


def test_row_shards_reassemble_the_single_rank_product():
    """Two ranks, each with its shard of weight rows; the all-gathered y equals, bit
    for bit, the product of the whole tall matrix computed in one process."""
    import numpy as np
    import torch
    import oracle
    from bit_quantized_gemm_quant_b200 import inputs
    world, rows, K, port = 2, 48, 256, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_shard_main, args=(r, world, port, rows, K, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    got = sorted((q.get(timeout=10) for _ in range(world)), key=lambda t: t[0])
    w = np.concatenate([inputs.weights_fp32(rows, K, inputs.generator(bench.shard_seed(0, r))).numpy()
                        for r in range(world)])
    wq, d = oracle.q4_0_quantize(w)
    x = inputs.activations_bf16(3, K, inputs.generator(1)).view(torch.int16).numpy().view(np.uint16)
    y_ref, _, _ = oracle.matmul_ref(x, oracle.q4_0_dequantize(wq, d), nthreads=1)
    for r, (rank, (first, last), full) in enumerate(got):
        assert rank == r and (first, last) == (r * rows, (r + 1) * rows)
        assert full.shape == (3, world * rows)
        assert np.array_equal(full, y_ref)
