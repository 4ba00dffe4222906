"""The multi-rank path of bench.py on CPU: two gloo ranks, each timing its own independent
layer; the job time is the max over ranks and the value counts every rank's work."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import sys
    from datetime import timedelta

    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        local_ms = [12.5, 20.0][rank]                  # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, world, "cpu")
        q.put((rank, ms, bench.job_tflops(1e12, world, ms)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_count_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, value in got:
        assert ms == 20.0
        assert value == pytest.approx(2 * 1e12 / 20e-3 / 1e12)


def test_single_rank_is_unchanged():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.max_over_ranks(7.0, 1, "cpu") == 7.0
    assert bench.job_tflops(2e12, 1, 1000.0) == pytest.approx(2.0)


def _split_rank(rank, world, port, q):
    """One rank of a head-split layer: its heads of a small 4-head layer through the oracle,
    gathered over gloo and compared with the one-rank result on every rank."""
    import dataclasses
    import sys
    from datetime import timedelta

    import numpy as np
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import diffusion_transformer_ultra_b200 as ug
    from diffusion_transformer_ultra_b200.sharding import head_range, head_slice
    from oracle import hla_oracle as O
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        wl = dataclasses.replace(ug.WORKLOADS["tiny"], H=16, W=16, l=8, b=2, T=8, heads=4)
        g = O.Geometry(wl.H, wl.W, wl.l, wl.b, wl.rho, wl.T)
        qf, kf, vf = ug.make_qkv(wl)
        h0, h1 = head_range(wl.heads, world, rank)
        # every head belongs to exactly one rank
        ranges = [None] * world
        dist.all_gather_object(ranges, (h0, h1))
        owned = sorted(h for a, b in ranges for h in range(a, b))
        # this rank's heads, from its own head slices of the inputs
        mine, _ = O.forward(*(head_slice(x, h0, h1).double().numpy() for x in (qf, kf, vf)), g, wl.axes)
        mine = torch.from_numpy(np.ascontiguousarray(mine))
        parts = [None] * world
        dist.all_gather_object(parts, (h0, mine))
        # heads sit on axis 1 of the oracle's permuted output [B, heads, N_tot, D]
        joined = torch.cat([p for _, p in sorted(parts, key=lambda x: x[0])], dim=1)
        whole, _ = O.forward(*(x.double().numpy() for x in (qf, kf, vf)), g, wl.axes)
        q.put((rank, owned, bool(torch.equal(joined, torch.from_numpy(np.ascontiguousarray(whole))))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_head_split_over_two_gloo_ranks_reassembles_the_layer_bitwise():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, owned, equal in got:
        assert owned == [0, 1, 2, 3]
        assert equal


def test_head_range_partitions_any_head_count():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from diffusion_transformer_ultra_b200.sharding import head_range
    for heads in (1, 2, 5, 24, 25):
        for world in range(1, min(heads, 9) + 1):
            spans = [head_range(heads, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == heads
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        head_range(3, 4, 0)
    with pytest.raises(ValueError):
        head_range(24, 2, 2)
