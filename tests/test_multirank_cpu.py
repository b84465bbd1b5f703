"""The multi-rank plumbing of bench.py, on CPU with the gloo backend (world size 2).

bench.py --gpus N splits one problem over the ranks: by rows of A (B
replicated, the default) or by column blocks of B (A replicated), and stitches
C with an all-gather; --parallel replicas gives every rank its own problem.
These tests check the partitions tile the problem exactly, that the stitched C
equals the oracle's full result (each rank computes its block with the oracle
as a stand-in for its GPU kernel, in the test only), the max-reduction of the
per-rank step times, and the per-rank seeds of the replicas.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import sys

    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        step_ms = [0.5, 0.8][rank]                      # rank 1 is the slowest
        slowest = bench.max_over_ranks(dist, step_ms, "cpu")
        value = bench.aggregate_throughput(world, 2 * 256 ** 3, slowest)
        dist.barrier()
        out.put((rank, slowest, value, bench.rank_seed(3, rank)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, v0, seed0), (r1, s1, v1, seed1) = results
    assert s0 == s1 == 0.8                              # every rank sees the max
    assert v0 == v1 == pytest.approx(2 * 2 * 256 ** 3 / 0.8e-3 / 1e12)
    assert seed0 != seed1                               # independent problems per rank


def test_rank_problems_are_independent_and_rank0_is_the_workload():
    import bench
    from tiled_dense_gemm_fp16_b200 import inputs
    name, M, N, K, A0, B0 = bench.workload_problem("square256", rank=0)
    (shape, A, B), = inputs.WORKLOADS["square256"].problems()
    assert (M, N, K) == shape and (A0 == A).all() and (B0 == B).all()
    _, _, _, _, A1, _ = bench.workload_problem("square256", rank=1)
    assert not (A1 == A0).all()


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    args = type("Args", (), {"workload": "square8192", "steps": 1, "warmup": 3, "gpus": 2})()
    assert bench.run_reference(args) == 0               # returns at once: no oracle run


def test_row_ranges_tile_m_exactly():
    import bench
    for M in (1, 2, 7, 37, 256, 3001, 8191, 8192):
        for world in (1, 2, 3, 4, 8):
            ranges = [bench.row_range(M, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == M
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [r1 - r0 for r0, r1 in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0


def _rows_worker(rank, world, port, out):
    import datetime
    import sys

    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import oracle
    from tiled_dense_gemm_fp16_b200 import inputs

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        M, N, K = 37, 24, 40                               # odd M: the blocks differ by one row
        A, B = inputs.operands(M, N, K, "int", seed=11)    # every rank draws the same problem
        r0, r1 = bench.row_range(M, world, rank)
        # Stand-in for the rank's GPU kernel (this test only): the oracle on the rank's rows.
        block = oracle.gemm_relu_f16(np.ascontiguousarray(A[r0:r1]), B)
        full = bench.gather_rows(dist, torch.from_numpy(block), M, world, rank)
        out.put((rank, r0, r1, full.numpy().view(np.uint16).copy()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_rows_and_stitch_c():
    import numpy as np

    import oracle
    from tiled_dense_gemm_fp16_b200 import inputs
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rows_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted((out.get(timeout=120) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    A, B = inputs.operands(37, 24, 40, "int", seed=11)
    want = oracle.gemm_relu_f16(A, B).view(np.uint16)
    assert [(r0, r1) for _, r0, r1, _ in results] == [(0, 18), (18, 37)]
    for _, _, _, full in results:                          # every rank holds the whole, stitched C
        assert full.shape == (37, 24)
        assert np.array_equal(full, want)


def test_col_ranges_tile_n_exactly_on_16_byte_boundaries():
    import bench
    for N in (1, 8, 9, 24, 43, 129, 5003, 8192, 12289):
        for world in (1, 2, 3, 4, 8):
            ranges = [bench.col_range(N, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == N
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            assert all(c0 % 8 == 0 and c1 >= c0 for c0, c1 in ranges)


def _cols_worker(rank, world, port, out):
    import datetime
    import sys

    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import oracle
    from tiled_dense_gemm_fp16_b200 import inputs

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        M, N, K = 37, 43, 40                               # odd N: blocks of 16 and 27 columns
        A, B = inputs.operands(M, N, K, "int", seed=12)    # every rank draws the same problem
        c0, c1 = bench.col_range(N, world, rank)
        # Stand-in for the rank's GPU kernel (this test only): the oracle on the rank's columns of B.
        block = oracle.gemm_relu_f16(A, np.ascontiguousarray(B[:, c0:c1]))
        full = bench.gather_cols(dist, torch.from_numpy(block), N, world, rank)
        out.put((rank, c0, c1, full.numpy().view(np.uint16).copy()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_columns_and_stitch_c():
    import numpy as np

    import oracle
    from tiled_dense_gemm_fp16_b200 import inputs
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cols_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted((out.get(timeout=120) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    A, B = inputs.operands(37, 43, 40, "int", seed=12)
    want = oracle.gemm_relu_f16(A, B).view(np.uint16)
    assert [(c0, c1) for _, c0, c1, _ in results] == [(0, 16), (16, 43)]
    for _, _, _, full in results:                          # every rank holds the whole, stitched C
        assert full.shape == (37, 43)
        assert np.array_equal(full, want)
