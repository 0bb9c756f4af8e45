"""Multi-rank placement (hot prefixes replicated, cold on one rank), run as world_size-2 gloo
ranks on CPU: every rank computes the placement on its own, the ranks agree, every request is
served by exactly one rank, every rank holds the prefixes its requests read, cold prefixes
live on one rank and the FLOP load is balanced."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from prefix_shared_attention_b200.sharding import place, request_flops
from workloads import CONFIGS, make_table


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, name, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        tab = make_table(name)
        spec = CONFIGS[name]
        pl = place(tab.prefix_len, tab.req_prefix, tab.suffix_len, world, spec.H, spec.d)
        mine = pl.requests[rank]
        # Gather what every rank decided for itself.
        n = torch.tensor([len(mine)])
        ns = [torch.zeros(1, dtype=torch.long) for _ in range(world)]
        dist.all_gather(ns, n)
        buf = torch.full((int(max(x.item() for x in ns)),), -1, dtype=torch.long)
        buf[:len(mine)] = torch.from_numpy(mine)
        bufs = [torch.zeros_like(buf) for _ in range(world)]
        dist.all_gather(bufs, buf)
        load = torch.tensor([float(request_flops(tab.prefix_len, tab.req_prefix[mine], tab.suffix_len[mine],
                                                 spec.H, spec.d).sum())], dtype=torch.float64)
        loads = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(loads, load)
        if rank == 0:
            served = [b[:int(k.item())].numpy() for b, k in zip(bufs, ns)]
            out_q.put((served, [float(l.item()) for l in loads], [p.tolist() for p in pl.prefixes], pl.hot.tolist()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", ["item-as-prefix", "user-as-prefix", "long-user-history"])
def test_two_rank_placement(name):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, name, q)) for r in range(world)]
    for p in procs:
        p.start()
    served, loads, prefixes, hot = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    tab = make_table(name)
    allr = np.concatenate(served)
    assert np.array_equal(np.sort(allr), np.arange(tab.R)), "each request on exactly one rank"
    for k in range(world):
        need = np.unique(tab.req_prefix[served[k]][tab.req_prefix[served[k]] >= 0])
        assert set(need.tolist()) <= set(prefixes[k]), "a rank lacks a prefix its requests read"
    holders = {}
    for k in range(world):
        for p in prefixes[k]:
            holders[p] = holders.get(p, 0) + 1
    cold = [p for p, n in holders.items() if p not in hot]
    assert all(holders[p] == 1 for p in cold)
    assert max(loads) / (sum(loads) / world) < 1.05, loads


def test_hot_item_is_replicated():
    tab = make_table("item-as-prefix")
    pl = place(tab.prefix_len, tab.req_prefix, tab.suffix_len, 8, 8, 64)
    counts = np.bincount(tab.req_prefix, minlength=tab.P)
    hottest = int(np.argmax(counts))
    assert hottest in pl.hot.tolist()
    assert sum(hottest in p.tolist() for p in pl.prefixes) > 1
    assert pl.load.max() / pl.load.mean() < 1.05
