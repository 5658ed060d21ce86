"""World-size-2 gloo runs on the CPU of the multi-rank host logic: slots split over
ranks, the ZigZagKV per-layer count exchange, and the benchmark's max-over-ranks
timing reduction. The per-slot counts come from the oracle (no GPU here)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, counts_all, n_layers, spl, L, avg, floor, ret):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import oracle as O
        from sparse_decode_attention_window_b200.sharding import slot_range, layer_count_sums, allreduce_layer_counts
        lo, hi = slot_range(len(counts_all), world, rank)
        local = torch.tensor(counts_all[lo:hi], dtype=torch.int32)
        sums = allreduce_layer_counts(layer_count_sums(local, lo, spl, n_layers))
        # the allocation from the reduced sums (one "head" per layer carrying the layer's sum)
        budgets = O.allocate_budgets(sums.numpy().reshape(n_layers, 1), L, avg, floor)
        # max over ranks of a per-rank time, as the benchmark reports it
        t = torch.tensor([1.0 + rank], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ret[rank] = (lo, hi, budgets.tolist(), float(t.item()))
    finally:
        dist.destroy_process_group()


def test_sharded_zigzag_allocation_matches_single_process():
    from workloads import get, make_inputs
    import oracle as O
    wl = get("zigzag").scaled(n_layers=4, L=1024, steps=0)
    inp = make_inputs(wl, "cpu")
    S = wl.n_slots
    counts = []
    for s in range(S):
        sc = O.window_scores(inp.q_win[s * wl.G:(s + 1) * wl.G], inp.k[s:s + 1], wl.L)[0]
        counts.append(O.mass_count(sc, wl.mass))
    ref = O.allocate_budgets(np.array(counts).reshape(wl.n_layers, wl.slots_per_layer), wl.L, wl.avg_budget,
                             wl.floor_budget)
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()               # its server process is spawned too: nothing forks
    ret = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, counts, wl.n_layers, wl.slots_per_layer, wl.L,
                                               wl.avg_budget, wl.floor_budget, ret)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert ret[0][0] == 0 and ret[1][1] == S and ret[0][1] == ret[1][0]
    for r in range(world):
        assert ret[r][2] == ref.tolist()
        assert ret[r][3] == 2.0


def test_slot_range_partitions():
    from sparse_decode_attention_window_b200.sharding import slot_range
    for n in (1, 7, 256):
        for world in (1, 2, 3, 8):
            spans = [slot_range(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
    with pytest.raises(ValueError):
        slot_range(4, 2, 2)
