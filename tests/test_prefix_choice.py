"""Hotness-aware prefix choice (prefix_shared_attention_b200/prefix_choice.py): its FLOP accounting,
checked through the forward's own batch (request tables and the pinned work metrics), its
result against exhaustive search over every cached set on tiny instances, the budget, and
hand-built cases whose answer is known.  CPU only."""

import itertools

import numpy as np
import pytest

from prefix_shared_attention_b200 import prefix_choice as pc
from prefix_shared_attention_b200.metrics import algorithmic_flops
from workloads import RequestTable

H, D, ELT = 2, 64, 2
ROW = 2 * H * D * ELT   # cache bytes per cached token (K and V)


def flops_via_batches(ch, user_len, item_len, q_user, q_item):
    """The FLOPs of running a choice as the library would: the forward over the request table
    (each request's own tokens over [prefix ; own]) plus the prefix-side step of every prefix
    in it (its tokens over itself), both counted by the work metrics."""
    tab, prefix_src, _ = pc.to_request_table(ch, user_len, item_len, q_user, q_item)
    fwd = algorithmic_flops(tab.prefix_len, tab.req_prefix, tab.suffix_len, H, D)
    side = RequestTable(np.zeros(0), np.full(tab.P, -1), tab.prefix_len)
    return fwd + algorithmic_flops(side.prefix_len, side.req_prefix, side.suffix_len, H, D)


def random_instance(rng, nu, ni, nq, lo=1, hi=40):
    user_len = rng.integers(lo, hi + 1, nu)
    item_len = rng.integers(lo, hi + 1, ni)
    q_user = rng.integers(0, nu, nq)
    q_item = rng.integers(0, ni, nq)
    return user_len, item_len, q_user, q_item


def exhaustive(user_len, item_len, q_user, q_item, budget, users_only=False):
    """Cheapest cached set by enumeration (each query reads its cached block that saves most)."""
    nu, ni = len(user_len), len(item_len)
    best = None
    for mask in range(1 << (nu + (0 if users_only else ni))):
        cu = np.array([(mask >> k) & 1 for k in range(nu)], bool)
        ci = np.array([(mask >> (nu + k)) & 1 for k in range(ni)], bool) if not users_only else np.zeros(ni, bool)
        if (user_len[cu].sum() + item_len[ci].sum()) * ROW > budget:
            continue
        c = pc.evaluate(user_len, item_len, q_user, q_item, cu, ci, H, D, ELT)
        if best is None or c.attn_flops < best.attn_flops:
            best = c
    return best


@pytest.mark.parametrize("seed", range(6))
def test_accounting_matches_the_forward_batches(seed):
    rng = np.random.default_rng(seed)
    user_len, item_len, q_user, q_item = random_instance(rng, 5, 6, 14)
    for budget in (0, 20 * ROW, 10**9):
        for f in (pc.choose, pc.user_as_prefix):
            ch = f(user_len, item_len, q_user, q_item, budget, H, D, ELT)
            assert ch.attn_flops == pytest.approx(flops_via_batches(ch, user_len, item_len, q_user, q_item), rel=1e-12)
            assert ch.cache_bytes <= budget
            # Every cached block is read by at least two queries.
            tab, _, _ = pc.to_request_table(ch, user_len, item_len, q_user, q_item)
            n_cached = int(ch.cached_users.sum() + ch.cached_items.sum())
            reads = np.bincount(tab.req_prefix, minlength=tab.P)[:n_cached]
            assert (reads >= 2).all()


@pytest.mark.parametrize("seed", range(12))
def test_against_exhaustive_search(seed):
    rng = np.random.default_rng(100 + seed)
    nu, ni = int(rng.integers(1, 5)), int(rng.integers(1, 5))
    user_len, item_len, q_user, q_item = random_instance(rng, nu, ni, int(rng.integers(3, 16)))
    budget = float(rng.integers(0, 120)) * ROW
    opt = exhaustive(user_len, item_len, q_user, q_item, budget)
    opt_u = exhaustive(user_len, item_len, q_user, q_item, budget, users_only=True)
    mine = pc.choose(user_len, item_len, q_user, q_item, budget, H, D, ELT)
    base = pc.user_as_prefix(user_len, item_len, q_user, q_item, budget, H, D, ELT)
    assert opt.attn_flops <= mine.attn_flops + 1e-6
    assert opt_u.attn_flops <= base.attn_flops + 1e-6
    assert mine.attn_flops <= base.attn_flops + 1e-6
    # The greedy is not optimal in general (budgeted facility location), but on these sizes
    # it stays close to the optimum.
    assert mine.attn_flops <= 1.25 * opt.attn_flops


def test_no_budget_means_no_cache():
    rng = np.random.default_rng(7)
    user_len, item_len, q_user, q_item = random_instance(rng, 4, 4, 10)
    ch = pc.choose(user_len, item_len, q_user, q_item, 0, H, D, ELT)
    assert not ch.cached_users.any() and not ch.cached_items.any()
    u, i = user_len[q_user].astype(float), item_len[q_item].astype(float)
    assert ch.attn_flops == pytest.approx(4 * H * D * float((u * u + u * i + i * i).sum()))


def test_hot_long_item_becomes_the_prefix():
    # Ten users with one query each, all on one long item: caching the item saves 9 * 512^2;
    # no user is worth caching (one query each).
    user_len, item_len = np.full(10, 30), np.array([512, 20])
    q_user, q_item = np.arange(10), np.zeros(10, np.int64)
    ch = pc.choose(user_len, item_len, q_user, q_item, 10**9, H, D, ELT)
    assert ch.cached_items.tolist() == [True, False] and not ch.cached_users.any()
    assert (ch.prefix_kind == pc.ITEM).all()
    base = pc.user_as_prefix(user_len, item_len, q_user, q_item, 10**9, H, D, ELT)
    assert not base.cached_users.any()
    # Exact saving: nine extra reads of the item's 512 tokens.
    assert base.attn_flops - ch.attn_flops == pytest.approx(4 * H * D * 9 * 512.0**2)


def test_busy_user_becomes_the_prefix_and_the_budget_binds():
    # One user with eight queries over distinct items, one with two: only the first fits.
    user_len, item_len = np.array([300, 200]), np.arange(10) + 5
    q_user = np.array([0] * 8 + [1] * 2)
    q_item = np.arange(10)
    ch = pc.choose(user_len, item_len, q_user, q_item, 300 * ROW, H, D, ELT)
    assert ch.cached_users.tolist() == [True, False] and not ch.cached_items.any()
    assert (ch.prefix_kind[:8] == pc.USER).all() and (ch.prefix_kind[8:] == pc.NONE).all()


def test_query_reads_the_longer_cached_block():
    user_len, item_len = np.array([100, 100, 100]), np.array([400, 50])
    q_user = np.array([0, 0, 0, 1, 2])
    q_item = np.array([0, 1, 0, 0, 1])
    kind = pc.assign(user_len, item_len, q_user, q_item, np.array([True, False, False]), np.array([True, True]))
    assert kind.tolist() == [pc.ITEM, pc.USER, pc.ITEM, pc.ITEM, pc.ITEM]


def test_synthetic_reduction_is_reported_and_positive():
    rows = pc.reduction_table(n_users=256, n_items=2048, budgets=(0.5, 1.0))
    for r in rows:
        assert 0.0 < r["flop_reduction"] < 1.0
        assert r["hotness_aware_tflop"] <= r["user_as_prefix_tflop"]
