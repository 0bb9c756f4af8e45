"""Request placement across GPUs: hot prefixes replicated, cold prefixes on one GPU.

Bat lead page, section "Why it works" (and "How Bat works"): hot item caches are replicated so
any request finds them locally, cold ones are sharded so each lives in one place.  Here the
unit is a prefix group (the requests that read one cached prefix; a request with no prefix
is a group of its own).  Groups are placed longest-processing-time first on the least loaded
rank, by the FLOPs they cost.  A group heavier than half a rank's fair share is hot: its
requests are dealt out over several ranks and its prefix K/V is replicated on each of them.

The attention itself needs no communication between ranks: every rank runs the forward on
its own requests against its local copy of the prefixes they read.  This module only decides
the placement (host logic, identical on every rank, so no collective is needed either).
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import List

import numpy as np


@dataclass
class Placement:
    requests: List[np.ndarray]      # per rank: request indices (ascending)
    prefixes: List[np.ndarray]      # per rank: prefix ids whose K/V must be resident
    load: np.ndarray                # per rank: FLOPs
    hot: np.ndarray                 # prefix ids replicated on more than one rank


def request_flops(prefix_len, req_prefix, suffix_len, H: int, d: int) -> np.ndarray:
    prefix_len = np.asarray(prefix_len, dtype=np.float64)
    req_prefix = np.asarray(req_prefix)
    Ls = np.asarray(suffix_len, dtype=np.float64)
    Lp = np.zeros_like(Ls)
    has = req_prefix >= 0
    Lp[has] = prefix_len[req_prefix[has]]
    return 4.0 * Ls * (Lp + Ls) * H * d


def place(prefix_len, req_prefix, suffix_len, world: int, H: int = 1, d: int = 1,
          hot_share: float = 0.5) -> Placement:
    req_prefix = np.asarray(req_prefix)
    R = len(req_prefix)
    cost = request_flops(prefix_len, req_prefix, suffix_len, H, d)
    fair = cost.sum() / max(world, 1)
    # Groups: one per referenced prefix, one per request without a prefix.
    groups = {}
    for r in range(R):
        key = int(req_prefix[r]) if req_prefix[r] >= 0 else -(r + 1)
        groups.setdefault(key, []).append(r)
    units = []   # (cost, prefix or -1, request list)
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
            units += [(pc[i], p, np.array(pieces[i], dtype=np.int64)) for i in range(n_pieces) if pieces[i]]
        else:
            units.append((c, p, reqs))
    units.sort(key=lambda u: (-u[0], u[1]))
    load = np.zeros(world)
    req_lists = [[] for _ in range(world)]
    pre_sets = [set() for _ in range(world)]
    for c, p, reqs in units:
        k = int(np.argmin(load))
        load[k] += c
        req_lists[k].append(reqs)
        if p >= 0:
            pre_sets[k].add(p)
    reps = {}
    for k in range(world):
        for p in pre_sets[k]:
            reps[p] = reps.get(p, 0) + 1
    hot = np.array(sorted(p for p, n in reps.items() if n > 1), dtype=np.int64)
    return Placement([np.sort(np.concatenate(l)) if l else np.zeros(0, np.int64) for l in req_lists],
                     [np.array(sorted(s), dtype=np.int64) for s in pre_sets], load, hot)
