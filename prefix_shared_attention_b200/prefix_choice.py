"""Hotness-aware choice of each query's prefix block under a cache-memory budget.

Bat lead page, section "How Bat works" ("Make the whole serving system revolve around that
flexible choice"): a scheduler decides, under memory limits, which block of each query (the
user's or the item's) becomes the cached prefix; section "Why it works" ("Hotness-aware
scheduling turns the flexibility into hits"): caching a block pays when many queries reuse
it, so hot items and busy users are the ones worth caching.  The pages give no policy, cost
model or thresholds; the ones below follow from the attention this library computes.

Cost model (algorithmic FLOPs of the attention layer, the library's own counts; every term
is multiplied by 4*H*d).  A query is a (user block of u tokens, item block of i tokens) pair.

* cached prefix X of length x used by a query whose other block has s tokens: the query's
  own tokens attend over [X ; own]: s * (x + s)  (the forward's per-request count);
* caching X: its own tokens' outputs, the prefix-side step, are computed once: x * x;
* no cached block: the query computes both blocks itself, one of them as its own prefix:
  u*u + i*(u + i) = u*u + u*i + i*i (the same for either order).

So a query that reads cached X instead of computing everything itself saves exactly x*x, and
caching X costs x*x once: X pays off when two or more queries read it.  Cache memory of X is
its K and V: 2 * x * H * d * elt bytes.  The choice is a budgeted facility-location problem
(each query takes the cached block that saves it most, i.e. the longer one); it is solved
greedily by saving per byte, with lazy re-evaluation (the savings of the remaining blocks
only shrink as blocks are added), then unused blocks are dropped.  The result is never worse
than the conventional user-as-prefix policy under the same budget: both are computed and the
cheaper one is returned.

The token count (tokens whose own projections and outputs are computed: each cached block
once plus every query's non-cached tokens) is reported beside the FLOPs: the rest of a model
layer scales with it.  All figures are synthetic (seeded inputs).
"""

from __future__ import annotations

import heapq
from dataclasses import dataclass

import numpy as np

NONE, USER, ITEM = -1, 0, 1


@dataclass
class Choice:
    cached_users: np.ndarray   # bool [n_users]
    cached_items: np.ndarray   # bool [n_items]
    prefix_kind: np.ndarray    # int8 [Q]: USER, ITEM or NONE (no cached block)
    attn_flops: float          # total algorithmic attention FLOPs (prefix-side + per-query)
    prefix_side_flops: float   # part of attn_flops spent on the cached blocks' own tokens
    tokens: int                # tokens computed: cached blocks once + each query's own
    cache_bytes: float         # K/V bytes of the cached blocks (per layer)
    policy: str


def _query_cost(u, i, kind):
    """Per-query attention cost in units of 4*H*d (vectorised over queries)."""
    u = np.asarray(u, np.float64)
    i = np.asarray(i, np.float64)
    return np.where(kind == USER, i * (u + i), np.where(kind == ITEM, u * (u + i), u * u + u * i + i * i))


def assign(user_len, item_len, q_user, q_item, cached_users, cached_items):
    """Each query takes the cached block that saves it most (the longer one; the user on a tie)."""
    u = np.asarray(user_len, np.float64)[q_user]
    i = np.asarray(item_len, np.float64)[q_item]
    cu = np.asarray(cached_users, bool)[q_user]
    ci = np.asarray(cached_items, bool)[q_item]
    kind = np.full(len(q_user), NONE, np.int8)
    kind[ci] = ITEM
    kind[cu & (~ci | (u >= i))] = USER
    return kind


def evaluate(user_len, item_len, q_user, q_item, cached_users, cached_items, H, d, elt=2, policy="given"):
    """Costs of a cached set: queries assigned by `assign`, the cached blocks' prefix-side step
    counted once for every cached block."""
    user_len = np.asarray(user_len, np.int64)
    item_len = np.asarray(item_len, np.int64)
    cached_users = np.asarray(cached_users, bool)
    cached_items = np.asarray(cached_items, bool)
    kind = assign(user_len, item_len, q_user, q_item, cached_users, cached_items)
    u = user_len[q_user].astype(np.float64)
    i = item_len[q_item].astype(np.float64)
    unit = 4.0 * H * d
    ps = float((user_len[cached_users].astype(np.float64) ** 2).sum() + (item_len[cached_items].astype(np.float64) ** 2).sum())
    per_q = float(_query_cost(u, i, kind).sum())
    own = np.where(kind == USER, i, np.where(kind == ITEM, u, u + i))
    tokens = int(user_len[cached_users].sum() + item_len[cached_items].sum() + own.sum())
    nbytes = 2.0 * (user_len[cached_users].sum() + item_len[cached_items].sum()) * H * d * elt
    return Choice(cached_users, cached_items, kind, unit * (ps + per_q), unit * ps, tokens, nbytes, policy)


def _greedy(user_len, item_len, q_user, q_item, budget_bytes, H, d, elt, allow_users, allow_items):
    """Lazy greedy by saving per byte over the allowed candidate blocks, then dropping blocks
    that no longer pay (read by fewer than two queries)."""
    nu, ni = len(user_len), len(item_len)
    lens = np.concatenate([np.asarray(user_len, np.float64), np.asarray(item_len, np.float64)])
    Q = len(q_user)
    # Candidate c in [0, nu) is a user, [nu, nu+ni) an item; its queries:
    qs_of = [[] for _ in range(nu + ni)]
    for q in range(Q):
        qs_of[int(q_user[q])].append(q)
        qs_of[nu + int(q_item[q])].append(q)
    qs_of = [np.array(v, np.int64) for v in qs_of]
    save = np.zeros(Q)          # current saving of each query (x*x of the block it reads)
    row_bytes = 2.0 * H * d * elt

    def gain(c):
        x2 = lens[c] ** 2
        return float(np.maximum(x2 - save[qs_of[c]], 0.0).sum()) - x2

    heap = []
    for c in range(nu + ni):
        if (c < nu and not allow_users) or (c >= nu and not allow_items) or len(qs_of[c]) < 2:
            continue
        g = gain(c)
        if g > 0:
            heapq.heappush(heap, (-g / (lens[c] * row_bytes), c))
    chosen = np.zeros(nu + ni, bool)
    used = 0.0
    while heap:
        neg, c = heapq.heappop(heap)
        cost_b = lens[c] * row_bytes
        if used + cost_b > budget_bytes:
            continue
        g = gain(c)
        if g <= 0:
            continue
        dens = g / cost_b
        if heap and dens < -heap[0][0] - 1e-12:
            heapq.heappush(heap, (-dens, c))     # stale: re-queue with its current density
            continue
        chosen[c] = True
        used += cost_b
        save[qs_of[c]] = np.maximum(save[qs_of[c]], lens[c] ** 2)
    # Drop blocks that no query prefers any more, or that only one query reads (they cost
    # their prefix-side step and save no more than it).
    while True:
        kind = assign(user_len, item_len, q_user, q_item, chosen[:nu], chosen[nu:])
        cnt = np.zeros(nu + ni, np.int64)
        np.add.at(cnt, np.asarray(q_user)[kind == USER], 1)
        np.add.at(cnt, nu + np.asarray(q_item)[kind == ITEM], 1)
        drop = chosen & (cnt < 2)
        if not drop.any():
            break
        chosen &= ~drop
    return chosen[:nu], chosen[nu:]


def user_as_prefix(user_len, item_len, q_user, q_item, budget_bytes, H, d, elt=2):
    """The conventional policy: only user blocks are cached (the most profitable per byte
    first, within the budget); every query with a cached user reads it."""
    cu, ci = _greedy(user_len, item_len, q_user, q_item, budget_bytes, H, d, elt, True, False)
    return evaluate(user_len, item_len, q_user, q_item, cu, ci, H, d, elt, "user-as-prefix")


def choose(user_len, item_len, q_user, q_item, budget_bytes, H, d, elt=2):
    """Hotness-aware choice: user or item blocks cached within `budget_bytes`, each query reading
    the cached block that saves it most; never worse than `user_as_prefix` at the same budget."""
    cu, ci = _greedy(user_len, item_len, q_user, q_item, budget_bytes, H, d, elt, True, True)
    mine = evaluate(user_len, item_len, q_user, q_item, cu, ci, H, d, elt, "hotness-aware")
    base = user_as_prefix(user_len, item_len, q_user, q_item, budget_bytes, H, d, elt)
    return mine if mine.attn_flops <= base.attn_flops else base


def synthetic_queries(seed=4, n_users=2048, per_user=8, n_items=16384, s=1.1, lo=64, hi=2048):
    """Queries shaped like the mixed serving batch: every user issues `per_user` queries, each
    pairing the user's block with one item drawn Zipf(s) over `n_items`; every block length is
    uniform in [lo, hi]."""
    from workloads import zipf_ranks
    rng = np.random.default_rng(seed)
    user_len = rng.integers(lo, hi + 1, n_users)
    item_len = rng.integers(lo, hi + 1, n_items)
    perm = rng.permutation(n_items)
    q_user = np.repeat(np.arange(n_users), per_user)
    q_item = perm[zipf_ranks(rng, n_items, s, n_users * per_user) - 1]
    return user_len, item_len, q_user, q_item


def reduction_table(H=16, d=128, elt=2, budgets=(0.25, 0.5, 1.0, 2.0), **kw):
    """Attention FLOPs and tokens of the hotness-aware choice against user-as-prefix, at cache
    budgets given as fractions of the bytes that caching every user would take."""
    user_len, item_len, q_user, q_item = synthetic_queries(**kw)
    all_users = 2.0 * float(np.sum(user_len)) * H * d * elt
    rows = []
    for f in budgets:
        b = f * all_users
        base = user_as_prefix(user_len, item_len, q_user, q_item, b, H, d, elt)
        mine = choose(user_len, item_len, q_user, q_item, b, H, d, elt)
        rows.append({"budget_frac_of_all_users": f, "budget_gb": b / 1e9,
                     "user_as_prefix_tflop": base.attn_flops / 1e12, "hotness_aware_tflop": mine.attn_flops / 1e12,
                     "flop_reduction": 1.0 - mine.attn_flops / base.attn_flops,
                     "token_reduction": 1.0 - mine.tokens / base.tokens,
                     "cached_users": int(mine.cached_users.sum()), "cached_items": int(mine.cached_items.sum()),
                     "queries_item_prefix": int((mine.prefix_kind == ITEM).sum()),
                     "queries_user_prefix": int((mine.prefix_kind == USER).sum()),
                     "queries_no_prefix": int((mine.prefix_kind == NONE).sum())})
    return rows


def to_request_table(choice: Choice, user_len, item_len, q_user, q_item):
    """The forward's batch for a choice: cached blocks become the prefixes (users first, then
    items); each query becomes one request whose own tokens are its non-cached block.  A query
    with no cached block reads its user block as a prefix built for it alone (computed, not
    kept).  Returns (RequestTable, prefix_src, suffix_src): for every prefix and every request,
    (kind, index) of the block it holds (kind USER or ITEM)."""
    from workloads import RequestTable
    cu = np.flatnonzero(choice.cached_users)
    ci = np.flatnonzero(choice.cached_items)
    pid_u = {int(x): k for k, x in enumerate(cu)}
    pid_i = {int(x): len(cu) + k for k, x in enumerate(ci)}
    prefix_src = [(USER, int(x)) for x in cu] + [(ITEM, int(x)) for x in ci]
    req_prefix, suffix_src = [], []
    for q in range(len(q_user)):
        k = int(choice.prefix_kind[q])
        if k == USER:
            req_prefix.append(pid_u[int(q_user[q])])
            suffix_src.append((ITEM, int(q_item[q])))
        elif k == ITEM:
            req_prefix.append(pid_i[int(q_item[q])])
            suffix_src.append((USER, int(q_user[q])))
        else:
            req_prefix.append(len(prefix_src))
            prefix_src.append((USER, int(q_user[q])))
            suffix_src.append((ITEM, int(q_item[q])))
    ln = lambda src: [int(user_len[x]) if kk == USER else int(item_len[x]) for kk, x in src]
    tab = RequestTable(np.array(ln(prefix_src), np.int64), np.array(req_prefix, np.int32),
                       np.array(ln(suffix_src), np.int64))
    return tab, prefix_src, suffix_src


def main():
    import json
    for r in reduction_table():
        print(json.dumps(r))


if __name__ == "__main__":
    main()
