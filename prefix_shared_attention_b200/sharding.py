"""Request placement across GPUs: hot prefixes replicated, cold prefixes on one owner.

Bat lead page, section "How Bat works" ("Keep the new item caches cheap by treating popular and
rare items differently"): hot item caches are replicated so any request finds them locally;
cold ones are sharded, each kept on one GPU, at the price of an occasional remote access.
Here the unit is a prefix group (the requests that read one cached prefix; a request with no
prefix is a group of its own).  Groups are placed longest-processing-time first on the least
loaded rank, by the FLOPs they cost.  A group heavier than half a rank's fair share is hot: its
requests are dealt out over several ranks and its prefix is replicated on each of them.

When the pool is already sharded (``owner[p]`` = the rank that holds prefix p's K/V, e.g. where
its prefix-side step ran), a cold group goes to its owner unless that would push the owner
past (1 + tolerance) of the fair share; it then goes to the least loaded rank, which fetches
the prefix from the owner before its forward (the remote access).  Hot prefixes are fetched
from their owner by every other rank that serves part of the group (the replication).

The attention itself needs no communication: every rank runs the forward on its own requests
against its local pool.  The only exchange is the prefix fetch, a set of point-to-point
copies (``exchange_prefixes``: NCCL send/recv between GPUs over NVLink, gloo between CPU
processes); the placement is host logic computed identically on every rank.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Callable, Dict, List, Optional, Tuple

import numpy as np


@dataclass
class Placement:
    requests: List[np.ndarray]      # per rank: request indices (ascending)
    prefixes: List[np.ndarray]      # per rank: prefix ids whose K/V must be resident (ascending)
    load: np.ndarray                # per rank: FLOPs
    hot: np.ndarray                 # prefix ids replicated on more than one rank
    owner: np.ndarray = None        # per prefix: rank holding it before the batch (-1: none)
    fetch: List[List[Tuple[int, int]]] = field(default_factory=list)   # per rank: (prefix, source rank)


def request_flops(prefix_len, req_prefix, suffix_len, H: int, d: int) -> np.ndarray:
    prefix_len = np.asarray(prefix_len, dtype=np.float64)
    req_prefix = np.asarray(req_prefix)
    Ls = np.asarray(suffix_len, dtype=np.float64)
    Lp = np.zeros_like(Ls)
    has = req_prefix >= 0
    Lp[has] = prefix_len[req_prefix[has]]
    return 4.0 * Ls * (Lp + Ls) * H * d


def hash_owner(P: int, world: int) -> np.ndarray:
    """A pool sharded without regard to load: prefix p on rank p mod world."""
    return np.arange(P, dtype=np.int64) % max(world, 1)


def place(prefix_len, req_prefix, suffix_len, world: int, H: int = 1, d: int = 1,
          hot_share: float = 0.5, owner: Optional[np.ndarray] = None, tolerance: float = 0.05) -> Placement:
    req_prefix = np.asarray(req_prefix)
    R = len(req_prefix)
    P = len(prefix_len)
    cost = request_flops(prefix_len, req_prefix, suffix_len, H, d)
    fair = cost.sum() / max(world, 1)
    own = np.full(P, -1, np.int64) if owner is None else np.asarray(owner, np.int64).copy()
    # Groups: one per referenced prefix, one per request without a prefix.
    groups = {}
    for r in range(R):
        key = int(req_prefix[r]) if req_prefix[r] >= 0 else -(r + 1)
        groups.setdefault(key, []).append(r)
    units = []   # (cost, prefix or -1, request list, hot)
    for key, reqs in groups.items():
        reqs = np.array(reqs, dtype=np.int64)
        c = float(cost[reqs].sum())
        p = key if key >= 0 else -1
        if p >= 0 and c > hot_share * fair and len(reqs) > 1:
            # Hot: cut into pieces of about a quarter of the fair share, each placed on its own.
            n_pieces = int(min(len(reqs), max(2, np.ceil(c / (0.25 * fair)))))
            order = reqs[np.argsort(-cost[reqs], kind="stable")]
            pieces = [[] for _ in range(n_pieces)]
            pc = np.zeros(n_pieces)
            for r in order:                       # LPT inside the group
                i = int(np.argmin(pc))
                pieces[i].append(r)
                pc[i] += cost[r]
            units += [(pc[i], p, np.array(pieces[i], dtype=np.int64), True) for i in range(n_pieces) if pieces[i]]
        else:
            units.append((c, p, reqs, False))
    units.sort(key=lambda u: (-u[0], u[1]))
    load = np.zeros(world)
    req_lists = [[] for _ in range(world)]
    pre_sets = [set() for _ in range(world)]
    for c, p, reqs, is_hot in units:
        k = int(np.argmin(load))
        if p >= 0 and not is_hot and own[p] >= 0 and load[own[p]] + c <= (1.0 + tolerance) * fair:
            k = int(own[p])                       # cold group on the rank that already holds its prefix
        load[k] += c
        req_lists[k].append(reqs)
        if p >= 0:
            pre_sets[k].add(p)
    reps = {}
    for k in range(world):
        for p in pre_sets[k]:
            reps[p] = reps.get(p, 0) + 1
    hot = np.array(sorted(p for p, n in reps.items() if n > 1), dtype=np.int64)
    prefixes = [np.array(sorted(s), dtype=np.int64) for s in pre_sets]
    # A prefix that no rank holds yet is built where it is needed (its prefix-side step runs
    # there, on every rank of a hot group): no fetch.  One that a rank already holds is fetched
    # from it by every other rank that needs it.
    fetch = [[(int(p), int(own[p])) for p in prefixes[k] if 0 <= own[p] != k] for k in range(world)]
    for k in range(world):
        for p in prefixes[k]:
            if own[p] < 0 and p not in set(hot.tolist()):
                own[p] = k
    return Placement([np.sort(np.concatenate(l)) if l else np.zeros(0, np.int64) for l in req_lists],
                     prefixes, load, hot, own, fetch)


def local_table(pl: Placement, rank: int, table):
    """This rank's batch: its requests (in ascending global order) over a local pool holding
    pl.prefixes[rank] in that order.  Returns (RequestTable, global prefix ids of the pool)."""
    from workloads import RequestTable
    reqs = pl.requests[rank]
    pids = pl.prefixes[rank]
    remap = np.full(max(table.P, 1), -1, np.int64)
    remap[pids] = np.arange(len(pids))
    rp = table.req_prefix[reqs]
    local = np.where(rp >= 0, remap[np.clip(rp, 0, None)], -1)
    assert (local[rp >= 0] >= 0).all(), "a request's prefix is missing from its rank's pool"
    return RequestTable(table.prefix_len[pids], local.astype(np.int32), table.suffix_len[reqs],
                        table.kind[reqs]), pids


def torch_copy_rows(k_src, v_src, ranges, k_dst, v_dst):
    """Row copies [(src_row0, rows, dst_row0)] between [T, H, d] tensors (torch slicing)."""
    for s0, n, d0 in ranges:
        k_dst[d0:d0 + n].copy_(k_src[s0:s0 + n])
        v_dst[d0:d0 + n].copy_(v_src[s0:s0 + n])


def bat_copy_rows(k_src, v_src, ranges, k_dst, v_dst):
    """The same copies by the library's K/V pack kernel (bat_prefix_kv_build), one launch per
    run of source-contiguous ranges."""
    import prefix_shared_attention_b200 as bat
    i = 0
    while i < len(ranges):
        j = i + 1
        while j < len(ranges) and ranges[j][0] == ranges[j - 1][0] + ranges[j - 1][1]:
            j += 1
        run = ranges[i:j]
        so = np.array([r[0] for r in run] + [run[-1][0] + run[-1][1]], np.int64)
        do = np.array([r[2] for r in run], np.int64)
        bat.bat_prefix_kv_build(k_src, v_src, so, do, k_dst, v_dst)
        i = j


def exchange_prefixes(pl: Placement, rank: int, world: int, prefix_len, owned_ids, owned_k, owned_v,
                      copy_rows: Callable = torch_copy_rows, group=None):
    """Builds this rank's local pool (pl.prefixes[rank] in order) from the prefixes it owns and
    those it fetches from their owners.

    owned_ids: global ids of the prefixes this rank holds before the exchange (those it owns and
    those it builds itself), in the row order of owned_k/owned_v ([rows, H, d] tensors, on this
    rank's device).  For every (destination, source) pair the
    source packs the requested prefixes' K and V rows into one buffer each, in ascending prefix
    order, and sends them; the destination receives them and copies them into place.  Every rank
    posts its sends and receives in the same order (ascending peer), as point-to-point
    collectives require.  Returns (k_pool, v_pool, bytes received)."""
    import torch
    import torch.distributed as dist
    prefix_len = np.asarray(prefix_len, np.int64)
    owned_ids = np.asarray(owned_ids, np.int64)
    own_row = {int(p): int(r) for p, r in zip(owned_ids, np.concatenate([[0], np.cumsum(prefix_len[owned_ids])])[:-1])}
    shape = tuple(owned_k.shape[1:])
    dev, dt = owned_k.device, owned_k.dtype
    pids = pl.prefixes[rank]
    pool_row = np.concatenate([[0], np.cumsum(prefix_len[pids])]).astype(np.int64)
    pos = {int(p): int(r) for p, r in zip(pids, pool_row[:-1])}
    k_pool = torch.empty((int(pool_row[-1]),) + shape, dtype=dt, device=dev)
    v_pool = torch.empty_like(k_pool)
    fetched = {int(p) for p, _ in pl.fetch[rank]}
    missing = [int(p) for p in pids if int(p) not in own_row and int(p) not in fetched]
    assert not missing, f"rank {rank} neither holds nor fetches prefixes {missing[:8]}"
    # Local prefixes: copy from the owned buffers.
    local = [(own_row[int(p)], int(prefix_len[p]), pos[int(p)]) for p in pids if int(p) not in fetched]
    if local:
        copy_rows(owned_k, owned_v, local, k_pool, v_pool)
    ops, recv = [], []
    for peer in range(world):
        if peer == rank:
            continue
        # What `peer` fetches from me, and what I fetch from `peer`, both in ascending prefix order.
        give = sorted(p for p, src in pl.fetch[peer] if src == rank)
        take = sorted(p for p, src in pl.fetch[rank] if src == peer)
        if give:
            n = int(prefix_len[give].sum())
            kb = torch.empty((n,) + shape, dtype=dt, device=dev)
            vb = torch.empty_like(kb)
            ranges, r0 = [], 0
            for p in give:
                ranges.append((own_row[p], int(prefix_len[p]), r0))
                r0 += int(prefix_len[p])
            copy_rows(owned_k, owned_v, ranges, kb, vb)
            ops += [dist.P2POp(dist.isend, kb, peer, group), dist.P2POp(dist.isend, vb, peer, group)]
        if take:
            n = int(prefix_len[take].sum())
            kb = torch.empty((n,) + shape, dtype=dt, device=dev)
            vb = torch.empty_like(kb)
            ops += [dist.P2POp(dist.irecv, kb, peer, group), dist.P2POp(dist.irecv, vb, peer, group)]
            recv.append((take, kb, vb))
    nbytes = 0
    if ops:
        for w in dist.batch_isend_irecv(ops):
            w.wait()
    for take, kb, vb in recv:
        ranges, r0 = [], 0
        for p in take:
            ranges.append((r0, int(prefix_len[p]), pos[p]))
            r0 += int(prefix_len[p])
        copy_rows(kb, vb, ranges, k_pool, v_pool)
        nbytes += 2 * kb.numel() * kb.element_size()
    return k_pool, v_pool, nbytes
