"""Seeded synthetic workloads for bipartite prefix-shared attention.

This module only *generates inputs*: request tables (which cached prefix each
request reads, and how long every block is) and N(0,1) tensors for Q, K and V.
It holds none of the attention arithmetic, so both the fp64 oracle and the
CUDA library can be fed from it without sharing any of the method's code.

Shapes follow the serving mix of "Bat: Efficient Generative Recommender
Serving with Bipartite Attention" (section "This paper's idea": a user block
or an item block is the cached prefix; section "Why it works": a hot item is
shared by many users).  The pages print no dataset, so the five named
configurations below are synthetic stand-ins:

* ``tiny``              H=2,  d=32,  fp32, 1 user prefix of 16 tokens, 4 requests x 8 suffix tokens.
* ``user-as-prefix``    H=8,  d=64,  bf16, 64 users x 256 cached tokens, 8 requests/user x 128 item tokens.
* ``item-as-prefix``    H=8,  d=64,  bf16, 4096 items x 32 cached tokens, 8192 requests, each one
                        Zipf(1.1)-drawn item plus 512 fresh user tokens.
* ``long-user-history`` H=16, d=128, bf16, 16 prefixes x 8192 tokens, 16 requests/prefix x 256 tokens.
* ``mixed``             H=16, d=128, bf16, 32768 requests: half user-prefix (2048 users x 8 requests),
                        half item-prefix (Zipf(1.1) over 16384 items); every block length is
                        uniform in [64, 2048].

Token-major layout: every tensor is ``[T, H, d]`` with d contiguous.  Request
``r`` owns suffix rows ``[suffix_offsets[r], suffix_offsets[r+1])``; prefix
``p`` owns cache rows ``[prefix_offsets[p], prefix_offsets[p+1])``;
``req_prefix[r] == -1`` means the request has no cached prefix.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

__all__ = [
    "CONFIGS",
    "WorkloadSpec",
    "RequestTable",
    "make_table",
    "split_launches",
    "random_table",
    "prefix_side_table",
    "host_tensors",
    "device_tensors",
    "zipf_ranks",
    "GBLA_LONG_HISTORY",
    "gbla_tensors",
]


@dataclass(frozen=True)
class WorkloadSpec:
    name: str
    H: int
    d: int
    dtype: str  # "fp32" or "bf16"
    seed: int
    description: str


CONFIGS: Dict[str, WorkloadSpec] = {
    s.name: s
    for s in [
        WorkloadSpec("tiny", 2, 32, "fp32", 0,
                     "1 user prefix of 16 tokens, 4 requests each with 8 item suffix tokens"),
        WorkloadSpec("user-as-prefix", 8, 64, "bf16", 1,
                     "64 users x 256 cached user tokens; 8 requests/user x 128 item tokens"),
        WorkloadSpec("item-as-prefix", 8, 64, "bf16", 2,
                     "4096 items x 32 cached item tokens; 8192 requests, Zipf(1.1) item + 512 user tokens"),
        WorkloadSpec("long-user-history", 16, 128, "bf16", 3,
                     "16 prefixes x 8192 user tokens; 16 requests/prefix x 256 item tokens"),
        WorkloadSpec("mixed", 16, 128, "bf16", 4,
                     "32768 requests, half user-prefix (2048 users x 8), half item-prefix "
                     "(Zipf(1.1) over 16384 items); block lengths uniform in [64, 2048]"),
    ]
}


@dataclass
class RequestTable:
    """Ragged request -> prefix index table (host arrays)."""

    prefix_len: np.ndarray          # int64 [P]   cached tokens of each prefix
    req_prefix: np.ndarray          # int32 [R]   prefix id of each request, -1 = none
    suffix_len: np.ndarray          # int64 [R]   suffix tokens of each request
    kind: Optional[np.ndarray] = None  # int8 [R]  0 = user block is the prefix, 1 = item block
    note: Dict[str, object] = field(default_factory=dict)

    def __post_init__(self):
        self.prefix_len = np.ascontiguousarray(self.prefix_len, dtype=np.int64)
        self.req_prefix = np.ascontiguousarray(self.req_prefix, dtype=np.int32)
        self.suffix_len = np.ascontiguousarray(self.suffix_len, dtype=np.int64)
        if self.kind is None:
            self.kind = np.zeros(len(self.req_prefix), dtype=np.int8)
        assert self.req_prefix.shape == self.suffix_len.shape

    @property
    def P(self) -> int:
        return int(self.prefix_len.shape[0])

    @property
    def R(self) -> int:
        return int(self.req_prefix.shape[0])

    @property
    def prefix_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.prefix_len)]).astype(np.int64)

    @property
    def suffix_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.suffix_len)]).astype(np.int64)

    @property
    def T_suf(self) -> int:
        return int(self.suffix_len.sum())

    @property
    def T_cache(self) -> int:
        return int(self.prefix_len.sum())

    def referenced_prefixes(self) -> np.ndarray:
        rp = self.req_prefix[self.req_prefix >= 0]
        return np.unique(rp)

    def prefix_len_of_request(self) -> np.ndarray:
        out = np.zeros(self.R, dtype=np.int64)
        m = self.req_prefix >= 0
        out[m] = self.prefix_len[self.req_prefix[m]]
        return out

    def compact(self, idx: np.ndarray) -> "RequestTable":
        """Requests ``idx`` over a cache holding only the prefixes they reference (ids remapped)."""
        idx = np.asarray(idx, dtype=np.int64)
        rp = self.req_prefix[idx]
        used = np.unique(rp[rp >= 0])
        remap = np.full(max(self.P, 1), -1, np.int64)
        remap[used] = np.arange(len(used))
        return RequestTable(self.prefix_len[used], np.where(rp >= 0, remap[np.clip(rp, 0, None)], -1),
                            self.suffix_len[idx], self.kind[idx], dict(self.note))

    def subset(self, idx: np.ndarray) -> "RequestTable":
        """Requests ``idx`` (in that order) over the same prefix cache."""
        idx = np.asarray(idx, dtype=np.int64)
        return RequestTable(self.prefix_len, self.req_prefix[idx], self.suffix_len[idx],
                            self.kind[idx], dict(self.note))


def zipf_ranks(rng: np.random.Generator, n_items: int, s: float, size: int) -> np.ndarray:
    """Finite Zipf draw by inverse CDF: rank k in [1, n_items] with P(k) proportional to k**-s."""
    w = np.arange(1, n_items + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(size)
    return np.searchsorted(cdf, u, side="right").clip(0, n_items - 1) + 1


def make_table(name: str) -> RequestTable:
    """The request table of a named configuration (seeded, deterministic)."""
    spec = CONFIGS[name]
    rng = np.random.default_rng(spec.seed)
    if name == "tiny":
        return RequestTable(np.array([16]), np.zeros(4, np.int32), np.full(4, 8))
    if name == "user-as-prefix":
        P, per = 64, 8
        return RequestTable(np.full(P, 256), np.repeat(np.arange(P), per), np.full(P * per, 128))
    if name == "item-as-prefix":
        n_items, R = 4096, 8192
        perm = rng.permutation(n_items)
        ranks = zipf_ranks(rng, n_items, 1.1, R)
        return RequestTable(np.full(n_items, 32), perm[ranks - 1], np.full(R, 512),
                            np.ones(R, np.int8))
    if name == "long-user-history":
        P, per = 16, 16
        return RequestTable(np.full(P, 8192), np.repeat(np.arange(P), per), np.full(P * per, 256))
    if name == "mixed":
        n_users, per_user, n_items, n_item_req = 2048, 8, 16384, 16384
        lo, hi = 64, 2048
        user_len = rng.integers(lo, hi + 1, n_users)
        item_len = rng.integers(lo, hi + 1, n_items)
        perm = rng.permutation(n_items)
        item_of_req = perm[zipf_ranks(rng, n_items, 1.1, n_item_req) - 1]
        # Only the items some request references are materialised in the cache.
        ref_items, item_req_local = np.unique(item_of_req, return_inverse=True)
        prefix_len = np.concatenate([user_len, item_len[ref_items]])
        req_prefix = np.concatenate([np.repeat(np.arange(n_users), per_user),
                                     n_users + item_req_local])
        suffix_len = rng.integers(lo, hi + 1, n_users * per_user + n_item_req)
        kind = np.concatenate([np.zeros(n_users * per_user, np.int8), np.ones(n_item_req, np.int8)])
        order = rng.permutation(len(req_prefix))
        t = RequestTable(prefix_len, req_prefix[order], suffix_len[order], kind[order])
        t.note["referenced_items"] = int(len(ref_items))
        return t
    raise KeyError(name)


def split_launches(table: RequestTable, n_launches: int) -> List[RequestTable]:
    """Request-disjoint equal chunks (the table's request order is already shuffled)."""
    R = table.R
    bounds = [(R * i) // n_launches for i in range(n_launches + 1)]
    return [table.subset(np.arange(bounds[i], bounds[i + 1])) for i in range(n_launches)]


def prefix_side_table(table: "RequestTable") -> "RequestTable":
    """The prefix-side batch of a workload: every prefix some request reads becomes one
    request with no cached prefix whose own tokens are the prefix's tokens (lengths only)."""
    used = table.referenced_prefixes()
    return RequestTable(np.zeros(0, np.int64), np.full(len(used), -1, np.int32), table.prefix_len[used])


def random_table(rng: np.random.Generator, P: int, R: int, max_prefix: int, max_suffix: int,
                 p_none: float = 0.1, min_suffix: int = 1) -> RequestTable:
    """Small ragged table for parity tests: random lengths, some requests with no prefix,
    some prefixes referenced by nobody."""
    prefix_len = rng.integers(0, max_prefix + 1, P) if P else np.zeros(0, np.int64)
    req_prefix = rng.integers(0, max(P, 1), R).astype(np.int32)
    if P == 0:
        req_prefix[:] = -1
    else:
        req_prefix[rng.random(R) < p_none] = -1
    suffix_len = rng.integers(min_suffix, max_suffix + 1, R)
    return RequestTable(prefix_len, req_prefix, suffix_len)


def _torch_dtype(dtype: str):
    import torch
    return {"fp32": torch.float32, "bf16": torch.bfloat16}[dtype]


def host_tensors(table: RequestTable, H: int, d: int, dtype: str, seed: int):
    """N(0,1) tensors on the host, drawn in fp32 and rounded (RNE) to ``dtype``.

    Returns a dict of CPU torch tensors: q, k_suf, v_suf ``[T_suf, H, d]`` and
    k_cache, v_cache ``[T_cache, H, d]``.
    """
    import torch
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    td = _torch_dtype(dtype)
    out = {}
    for key, T in (("q", table.T_suf), ("k_suf", table.T_suf), ("v_suf", table.T_suf),
                   ("k_cache", table.T_cache), ("v_cache", table.T_cache)):
        out[key] = torch.randn((T, H, d), generator=g, dtype=torch.float32).to(td)
    return out


def device_tensors(table: RequestTable, H: int, d: int, dtype: str, seed: int, device="cuda",
                   which=("q", "k_suf", "v_suf", "k_cache", "v_cache"), rows=None):
    """Same distribution as :func:`host_tensors`, drawn on the device by a seeded generator
    (for sizes the host cannot generate quickly).  ``rows`` overrides the row count of the
    suffix tensors (used when several launches share one buffer)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    td = _torch_dtype(dtype)
    out = {}
    for key in which:
        T = table.T_cache if key.endswith("cache") else (rows if rows is not None else table.T_suf)
        t = torch.empty((T, H, d), dtype=td, device=device)
        # Draw in bounded chunks so the fp32 staging buffer stays small.
        flat = t.view(-1)
        chunk = 1 << 28
        for s in range(0, flat.numel(), chunk):
            n = min(chunk, flat.numel() - s)
            flat[s:s + n].copy_(torch.randn(n, generator=g, device=device, dtype=torch.float32))
        out[key] = t
    return out


def gather_requests(table: RequestTable, tensors: dict, reqs, out=None):
    """Compact copy of the rows that requests ``reqs`` read, moved to the host.

    Returns ``(sub_table, host_tensors, rows)``: a table over just those requests and the
    prefixes they reference, their q/k_suf/v_suf rows and the referenced prefix rows (CPU
    torch tensors in the original dtype), and the original suffix row index of every row of
    the compact suffix tensors (so outputs can be gathered the same way).  ``out``, when
    given, is gathered into ``host_tensors['out']``.  Pure data movement.
    """
    import torch
    reqs = np.asarray(reqs, dtype=np.int64)
    so, po = table.suffix_offsets, table.prefix_offsets
    rows = np.concatenate([np.arange(so[r], so[r + 1]) for r in reqs]) if len(reqs) else np.zeros(0, np.int64)
    used = np.unique(table.req_prefix[reqs][table.req_prefix[reqs] >= 0])
    remap = {int(p): i for i, p in enumerate(used)}
    crow = np.concatenate([np.arange(po[p], po[p + 1]) for p in used]) if len(used) else np.zeros(0, np.int64)
    sub = RequestTable(table.prefix_len[used], np.array([remap.get(int(table.req_prefix[r]), -1) for r in reqs]),
                       table.suffix_len[reqs], table.kind[reqs])

    def take(t, idx):
        ii = torch.from_numpy(idx).to(t.device)
        return t.index_select(0, ii).cpu()

    host = {k: take(tensors[k], rows) for k in ("q", "k_suf", "v_suf")}
    host["k_cache"] = take(tensors["k_cache"], crow)
    host["v_cache"] = take(tensors["v_cache"], crow)
    if out is not None:
        host["out"] = take(out, rows)
    return sub, host, rows


# GBLA (gated bidirectional linear attention, the second workload): a batch of long user
# histories.  The GBLA page quotes its single-layer speed at a history length of 32768; the
# batch and head count are this build's choice (8 histories, 8 heads of width 128).
GBLA_LONG_HISTORY = {"name": "gbla-long-history", "seq_lens": [32768] * 8, "H": 8, "d": 128, "seed": 5,
                     "description": "8 user histories x 32768 tokens, H=8, d=128, bf16 (q, k, v, z N(0,1); "
                                    "gate logits N(0, 2^2); conv taps N(0, 0.6^2); norm weight 1 + N(0, 0.2^2))"}


def gbla_tensors(seq_lens, H: int, seed: int, device="cpu", d: int = 128):
    """Seeded inputs of the GBLA layer: q, k, v, z bf16 [T, H, d] ~ N(0,1); key-gate logits a bf16
    [T, H] ~ N(0, 2^2); causal-convolution taps cq, ck, cv fp32 [H, 4, d] ~ N(0, 0.6^2); norm weight
    g fp32 [H, d] ~ 1 + N(0, 0.2^2).  Returns (dict, seq_offsets)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    T = int(sum(seq_lens))
    rn = lambda *shape: torch.randn(*shape, generator=g, device=device)
    x = {"q": rn(T, H, d).bfloat16(), "k": rn(T, H, d).bfloat16(), "v": rn(T, H, d).bfloat16(),
         "z": rn(T, H, d).bfloat16(), "a": (2.0 * rn(T, H)).bfloat16(),
         "cq": 0.6 * rn(H, 4, d), "ck": 0.6 * rn(H, 4, d), "cv": 0.6 * rn(H, 4, d), "g": 1.0 + 0.2 * rn(H, d)}
    so = np.concatenate([[0], np.cumsum(np.asarray(seq_lens, np.int64))]).astype(np.int64)
    return x, so
