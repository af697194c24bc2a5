"""The benchmark's multi-rank host logic on CPU with world_size 2 (gloo):
max-over-ranks timing, layer-set throughput, and the split of one layer set
by layer (every matrix with all its simulated workers on exactly one rank)."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 100.0 + 50.0 * rank          # rank 1 is the slower one
        ms = bench.reduce_max(local_ms, world)
        value = bench.layer_set_rate(10, ms)
        owned = {name: bench.rank_layers(name, 0, rank, world) for name in ("c5_gpt2l", "c2_resnet50", "c3_gpt2s")}
        everyone = [None] * world
        dist.all_gather_object(everyone, owned)
        out.put((rank, ms, value, everyone))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_split_one_layer_set_by_layer():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, v0, all0), (r1, ms1, v1, all1) = res
    assert ms0 == ms1 == 150.0                      # both ranks report the slowest time
    assert v0 == v1 == pytest.approx(10 / 0.150)     # one layer set, ten steps, in the slowest rank's time
    assert all0 == all1                             # every rank computes the same split

    import bench
    for name, _ in all0[0].items():
        shapes = bench.set_shapes(name)
        parts = [all0[r][name] for r in range(2)]
        owners = sorted(i for p in parts for i in p)
        assert owners == list(range(len(shapes)))   # every layer updated, and by exactly one rank
        costs = bench.set_costs(name, shapes)
        loads = [sum(costs[i] for i in p) for p in parts]
        # longest first onto the least loaded rank: the gap is at most the largest layer
        assert max(loads) - min(loads) <= max(costs)
        assert sum(loads) == pytest.approx(sum(costs))  # the ranks' work adds up to one step of the set


def test_partition_is_longest_first_and_deterministic():
    import bench
    costs = [5, 1, 4, 4, 3, 2, 2]
    parts = bench.partition_layers(costs, 3)
    # by hand: 0 (5) -> r0; 2 (4) -> r1; 3 (4) -> r2; 4 (3) -> r1 (tie 4/4, lower rank); 5 (2) -> r2;
    # 6 (2) -> r0 (load 5); 1 (1) -> r2 (loads 7, 7, 6)
    assert parts == [[0, 6], [2, 4], [1, 3, 5]]
    assert bench.partition_layers(costs, 1) == [list(range(7))]
    assert sorted(i for p in bench.partition_layers(costs, 10) for i in p) == list(range(7))


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
