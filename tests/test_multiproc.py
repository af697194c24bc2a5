"""The benchmark's multi-rank host logic on CPU with world_size 2 (gloo):
max-over-ranks timing, whole-job throughput, distinct per-rank streams."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    import bench
    import workloads as WL
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 100.0 + 50.0 * rank          # rank 1 is the slower one
        ms = bench.reduce_max(local_ms, world)
        value = bench.job_throughput(10, ms, world)
        g = WL.GradientStreams([(4, 5)], 2, 1.0, seed_base=bench.rank_seed_base(rank)).next_step()
        out.put((rank, ms, value, float(g[0][0].sum()), float(g[0][1].sum())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, v0, a0, b0), (r1, ms1, v1, a1, b1) = res
    assert ms0 == ms1 == 150.0                      # both ranks report the slowest time
    assert v0 == v1 == pytest.approx(2 * 10 / 0.150)
    assert len({a0, b0, a1, b1}) == 4               # four distinct gradient streams


def _exchange_worker(rank, world, port, out):
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle as O
    import workloads as WL
    from matrix_aware_sign_b200.distributed import exchange_packed, exchange_signs_int8
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shape = (37, 29)                      # 1073 entries: a ragged last word
        U = WL.synthetic_polar_outputs(shape, world, seed=5, dtype="f32", zero_fraction=0.05)
        signs = [O.sign_extract(u).reshape(-1) for u in U]   # every rank knows all, sends its own
        mine = torch.from_numpy(O.pack_bits(signs[rank]).view(np.int32))
        gathered = exchange_packed(mine).numpy().view(np.uint32)
        ok_gather = all(np.array_equal(gathered[k], O.pack_bits(signs[k])) for k in range(world))
        ok_vote = np.array_equal(O.vote_from_packed(list(gathered), world, signs[0].size),
                                 O.vote_from_signs(signs))
        total = exchange_signs_int8(torch.from_numpy(signs[rank].copy())).numpy()
        ok_sum = np.array_equal(total, np.sum(np.stack(signs).astype(np.int64), axis=0))
        out.put((rank, ok_gather, ok_vote, ok_sum))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_exchange_the_messages():
    """The pages' deployment (one worker per rank): the 1-bit messages are
    all-gathered in rank order and vote like the signs they carry; the int8
    signs all-reduce to their sum."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_exchange_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, True, True, True), (1, True, True, True)]
