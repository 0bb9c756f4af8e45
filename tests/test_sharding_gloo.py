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


def _fetch_worker(rank, world, port, out_q):
    """One rank of a sharded pool: it holds the prefixes hash_owner gives it, fetches the ones its
    requests read from their owners (gloo send/recv standing in for the NVLink copy), builds its
    local batch and runs the oracle on it."""
    import oracle
    from prefix_shared_attention_b200.sharding import exchange_prefixes, hash_owner, local_table
    from workloads import host_tensors, random_table
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        tab, H, d = _fetch_table(), 2, 16
        x = host_tensors(tab, H, d, "bf16", 17)          # the same seeded data on every rank
        owner = hash_owner(tab.P, world)
        pl = place(tab.prefix_len, tab.req_prefix, tab.suffix_len, world, H, d, owner=owner, tolerance=0.0)
        po = tab.prefix_offsets
        owned = np.flatnonzero(owner == rank)
        rows = np.concatenate([np.arange(po[p], po[p + 1]) for p in owned]) if len(owned) else np.zeros(0, np.int64)
        ok_, ov_ = x["k_cache"][torch.from_numpy(rows)], x["v_cache"][torch.from_numpy(rows)]
        k_pool, v_pool, nbytes = exchange_prefixes(pl, rank, world, tab.prefix_len, owned, ok_, ov_)
        ltab, pids = local_table(pl, rank, tab)
        want = np.concatenate([np.arange(po[p], po[p + 1]) for p in pids]) if len(pids) else np.zeros(0, np.int64)
        pool_exact = bool(torch.equal(k_pool, x["k_cache"][torch.from_numpy(want)]) and
                          torch.equal(v_pool, x["v_cache"][torch.from_numpy(want)]))
        so = tab.suffix_offsets
        reqs = pl.requests[rank]
        srows = np.concatenate([np.arange(so[r], so[r + 1]) for r in reqs]) if len(reqs) else np.zeros(0, np.int64)
        sel = lambda t: t[torch.from_numpy(srows)]
        o, _ = oracle.bipartite_attention(sel(x["q"]), sel(x["k_suf"]), sel(x["v_suf"]), k_pool, v_pool,
                                          ltab.prefix_offsets, ltab.suffix_offsets, ltab.req_prefix)
        out_q.put((rank, reqs, o, pool_exact, nbytes, len(pl.fetch[rank])))
    finally:
        dist.destroy_process_group()


def _fetch_table():
    from workloads import RequestTable
    rng = np.random.default_rng(8)
    P = 7
    req = np.concatenate([np.zeros(9, np.int32), rng.integers(0, P, 15).astype(np.int32), [-1, -1]])
    return RequestTable(rng.integers(1, 200, P), req, rng.integers(1, 150, len(req)))


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_pool_with_fetch_equals_single_rank(world):
    """Hot prefix 0 (nine requests) replicated by fetching it from its owner, cold prefixes on
    hash owners with groups moved off an overloaded owner (and their prefixes fetched): the
    union of every rank's outputs equals the single-rank oracle output."""
    import oracle
    from workloads import host_tensors
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_fetch_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    tab = _fetch_table()
    x = host_tensors(tab, 2, 16, "bf16", 17)
    ref, _ = oracle.bipartite_attention(x["q"], x["k_suf"], x["v_suf"], x["k_cache"], x["v_cache"],
                                        tab.prefix_offsets, tab.suffix_offsets, tab.req_prefix)
    so = tab.suffix_offsets
    served = np.concatenate([r[1] for r in res])
    assert np.array_equal(np.sort(served), np.arange(tab.R)), "each request on exactly one rank"
    assert all(r[3] for r in res), "a rank's pool differs from the prefixes it should hold"
    assert sum(r[5] for r in res) > 0 and sum(r[4] for r in res) > 0, "no prefix was fetched"
    for rank, reqs, o, _, _, _ in res:
        row = 0
        for r in reqs:
            n = so[r + 1] - so[r]
            assert np.array_equal(o[row:row + n], ref[so[r]:so[r + 1]]), f"request {r} on rank {rank}"
            row += n
