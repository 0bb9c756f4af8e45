"""Pins for the fp64 oracle, none of which re-types the oracle's own formula.

* brute force: explicit per-element loops over the definition (math.exp, no numpy);
* hand-derived worked examples in tests/golden/hand_derived.json;
* closed forms (zero keys, one key, equal values, vanishing scale);
* the four invariants named for the method (prefix/suffix role swap, token
  permutation, log-sum-exp split, empty prefix);
* a library routine for the empty-prefix case (torch scaled_dot_product_attention, fp64, CPU);
* planted mistakes: each plausible bug, planted in the oracle, fails at least one pin.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle
import oracle.attention as oa
from workloads import RequestTable, host_tensors, make_table, random_table

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_derived.json")


# ----------------------------------------------------------------------------------------
# helpers

def brute_force(q, k_suf, v_suf, k_cache, v_cache, prefix_offsets, suffix_offsets, req_prefix,
                scale=None):
    """Element-by-element definition: for every suffix row, list the keys it sees
    (prefix rows, then its own suffix rows), score, exponentiate, normalise, sum."""
    T, H, d = q.shape
    dv = v_suf.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.full((T, H, dv), np.nan)
    lse = np.full((H, T), np.nan)
    for r in range(len(req_prefix)):
        rows = range(int(suffix_offsets[r]), int(suffix_offsets[r + 1]))
        p = int(req_prefix[r])
        pre = range(int(prefix_offsets[p]), int(prefix_offsets[p + 1])) if p >= 0 else range(0)
        for h in range(H):
            keys = [(k_cache[j, h], v_cache[j, h]) for j in pre] + [(k_suf[j, h], v_suf[j, h]) for j in rows]
            for i in rows:
                scores = []
                for kv in keys:
                    acc = 0.0
                    for c in range(d):
                        acc += float(q[i, h, c]) * float(kv[0][c])
                    scores.append(scale * acc)
                top = max(scores)
                w = [math.exp(s - top) for s in scores]
                z = sum(w)
                for c in range(dv):
                    out[i, h, c] = sum(w[j] * float(keys[j][1][c]) for j in range(len(keys))) / z
                lse[h, i] = top + math.log(z)
    return out, lse


def as64(t):
    return t.double().numpy()


def tiny_inputs():
    tab = make_table("tiny")
    x = host_tensors(tab, 2, 32, "fp32", 0)
    return tab, {k: as64(v) for k, v in x.items()}


def run_oracle(tab, x, **kw):
    return oracle.bipartite_attention(x["q"], x["k_suf"], x["v_suf"], x["k_cache"], x["v_cache"],
                                      tab.prefix_offsets, tab.suffix_offsets, tab.req_prefix, **kw)


def run_brute(tab, x, **kw):
    return brute_force(x["q"], x["k_suf"], x["v_suf"], x["k_cache"], x["v_cache"],
                       tab.prefix_offsets, tab.suffix_offsets, tab.req_prefix, **kw)


def small_random(seed, P=3, R=5, max_prefix=9, max_suffix=7, H=2, d=4):
    rng = np.random.default_rng(seed)
    tab = random_table(rng, P, R, max_prefix, max_suffix)
    x = host_tensors(tab, H, d, "fp32", seed)
    return tab, {k: as64(v) for k, v in x.items()}


# ----------------------------------------------------------------------------------------
# brute force

def test_tiny_config_matches_brute_force():
    tab, x = tiny_inputs()
    o, l = run_oracle(tab, x)
    ob, lb = run_brute(tab, x)
    assert np.isfinite(o).all()
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l, lb, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("seed", range(6))
def test_random_ragged_tables_match_brute_force(seed):
    tab, x = small_random(seed)
    o, l = run_oracle(tab, x)
    ob, lb = run_brute(tab, x)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l, lb, rtol=1e-12, atol=1e-13)


def test_explicit_scale_matches_brute_force():
    tab, x = small_random(11)
    o, l = run_oracle(tab, x, scale=0.73)
    ob, lb = run_brute(tab, x, scale=0.73)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l, lb, rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------------------
# hand-derived worked examples

@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_hand_derived_examples(case):
    a = {k: np.array(case[k], dtype=np.float64) for k in ("q", "k_suf", "v_suf", "k_cache", "v_cache")}
    o, l = oracle.bipartite_attention(a["q"], a["k_suf"], a["v_suf"], a["k_cache"], a["v_cache"],
                                      np.array(case["prefix_offsets"]), np.array(case["suffix_offsets"]),
                                      np.array(case["req_prefix"]), scale=case["scale"])
    np.testing.assert_allclose(o, np.array(case["out"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, np.array(case["lse"]), rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------------------
# closed forms

def test_zero_keys_give_mean_of_values():
    tab, x = small_random(3)
    x["k_suf"][:] = 0.0
    x["k_cache"][:] = 0.0
    o, l = run_oracle(tab, x)
    for r in range(tab.R):
        s0, s1 = tab.suffix_offsets[r], tab.suffix_offsets[r + 1]
        p = tab.req_prefix[r]
        for h in range(2):
            vals = list(x["v_suf"][s0:s1, h])
            if p >= 0:
                vals = list(x["v_cache"][tab.prefix_offsets[p]:tab.prefix_offsets[p + 1], h]) + vals
            mean = np.mean(vals, axis=0)
            for i in range(s0, s1):
                np.testing.assert_allclose(o[i, h], mean, rtol=1e-12, atol=1e-13)
                assert abs(l[h, i] - math.log(len(vals))) < 1e-12


def test_single_key_returns_its_value():
    tab = RequestTable(np.zeros(1), np.array([-1, 0]), np.array([1, 1]))
    x = host_tensors(tab, 3, 8, "fp32", 5)
    x = {k: as64(v) for k, v in x.items()}
    o, l = run_oracle(tab, x)
    np.testing.assert_allclose(o, x["v_suf"], rtol=0, atol=1e-14)
    expect = np.einsum("thd,thd->ht", x["q"], x["k_suf"]) / math.sqrt(8)
    np.testing.assert_allclose(l, expect, rtol=1e-13, atol=1e-13)


def test_equal_values_return_that_value():
    tab, x = small_random(4)
    row = np.linspace(-1.0, 2.0, x["v_suf"].shape[2])
    x["v_suf"][:] = row
    x["v_cache"][:] = row
    o, _ = run_oracle(tab, x)
    valid = ~np.isnan(o)
    np.testing.assert_allclose(o[valid].reshape(-1, row.size), np.broadcast_to(row, (valid.sum() // row.size, row.size)),
                               rtol=1e-13, atol=1e-13)


def test_vanishing_scale_gives_uniform_mean():
    tab, x = small_random(5)
    o, _ = run_oracle(tab, x, scale=1e-14)
    x["k_suf"][:] = 0.0
    x["k_cache"][:] = 0.0
    o0, _ = run_oracle(tab, x)   # zero keys: exact uniform mean
    np.testing.assert_allclose(o, o0, rtol=1e-10, atol=1e-11)


# ----------------------------------------------------------------------------------------
# invariant (1): which block is the prefix does not change the outputs

def _pair_case(seed, n_pairs=3, H=2, d=8):
    rng = np.random.default_rng(seed)
    ul = rng.integers(1, 9, n_pairs)   # user block lengths
    il = rng.integers(1, 9, n_pairs)   # item block lengths
    tok = {}
    for key in ("q", "k", "v"):
        tok[key] = [rng.standard_normal((ul[i] + il[i], H, d)) for i in range(n_pairs)]  # [U ; I] tokens
    return ul, il, tok


def _run_as(prefix_is_user, ul, il, tok):
    """Build a cache of one block per pair and a request per pair whose suffix is the other block."""
    n = len(ul)
    pre = [slice(0, ul[i]) if prefix_is_user else slice(ul[i], ul[i] + il[i]) for i in range(n)]
    suf = [slice(ul[i], ul[i] + il[i]) if prefix_is_user else slice(0, ul[i]) for i in range(n)]
    cat = lambda key, sl: np.concatenate([tok[key][i][sl[i]] for i in range(n)], axis=0)
    tab = RequestTable(np.array([s.stop - s.start for s in pre]), np.arange(n),
                       np.array([s.stop - s.start for s in suf]))
    o, l = oracle.bipartite_attention(cat("q", suf), cat("k", suf), cat("v", suf), cat("k", pre), cat("v", pre),
                                      tab.prefix_offsets, tab.suffix_offsets, tab.req_prefix)
    return tab, o, l


@pytest.mark.parametrize("seed", range(4))
def test_invariant_role_swap(seed):
    ul, il, tok = _pair_case(seed)
    tab_u, o_u, l_u = _run_as(True, ul, il, tok)    # user block cached, item tokens are the suffix
    tab_i, o_i, l_i = _run_as(False, ul, il, tok)   # item block cached, user tokens are the suffix
    d = tok["q"][0].shape[2]
    for i in range(len(ul)):
        # Monolithic bidirectional attention over the whole request, both token orders.
        for order in ("UI", "IU"):
            idx = np.arange(ul[i] + il[i]) if order == "UI" else np.r_[ul[i]:ul[i] + il[i], 0:ul[i]]
            for h in range(tok["q"][i].shape[1]):
                Q, K, V = (tok[k][i][idx, h] for k in ("q", "k", "v"))
                mono, mono_l = oracle.attend(Q, K, V, 1 / math.sqrt(d))
                back = np.empty_like(mono)
                back[idx] = mono
                back_l = np.empty_like(mono_l)
                back_l[idx] = mono_l
                item_rows = slice(tab_u.suffix_offsets[i], tab_u.suffix_offsets[i + 1])
                user_rows = slice(tab_i.suffix_offsets[i], tab_i.suffix_offsets[i + 1])
                np.testing.assert_allclose(o_u[item_rows, h], back[ul[i]:], rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(o_i[user_rows, h], back[:ul[i]], rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(l_u[h, item_rows], back_l[ul[i]:], rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(l_i[h, user_rows], back_l[:ul[i]], rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------------------
# invariant (2): permuting tokens inside a block permutes outputs identically

@pytest.mark.parametrize("seed", range(4))
def test_invariant_token_permutation(seed):
    tab, x = small_random(100 + seed, P=2, R=4, max_prefix=10, max_suffix=9)
    o, l = run_oracle(tab, x)
    rng = np.random.default_rng(seed)
    # Permute the cached rows inside every prefix: outputs unchanged.
    perm_c = np.arange(tab.T_cache)
    for p in range(tab.P):
        a, b = tab.prefix_offsets[p], tab.prefix_offsets[p + 1]
        perm_c[a:b] = a + rng.permutation(b - a)
    # Permute the suffix rows inside every request (q, k, v together): outputs permute alike.
    perm_s = np.arange(tab.T_suf)
    for r in range(tab.R):
        a, b = tab.suffix_offsets[r], tab.suffix_offsets[r + 1]
        perm_s[a:b] = a + rng.permutation(b - a)
    y = dict(x)
    y["k_cache"], y["v_cache"] = x["k_cache"][perm_c], x["v_cache"][perm_c]
    y["q"], y["k_suf"], y["v_suf"] = x["q"][perm_s], x["k_suf"][perm_s], x["v_suf"][perm_s]
    o2, l2 = run_oracle(tab, y)
    np.testing.assert_allclose(o2, o[perm_s], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l2, l[:, perm_s], rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------------------
# invariant (3): the log-sum-exp merge of a split equals the monolithic softmax

@pytest.mark.parametrize("chunks", [1, 2, 3, 5, 12])
def test_invariant_split_merge(chunks):
    tab, x = small_random(7, P=3, R=6, max_prefix=11, max_suffix=6)
    o, l = run_oracle(tab, x)
    os_, ls_ = oracle.bipartite_attention_split(x["q"], x["k_suf"], x["v_suf"], x["k_cache"], x["v_cache"],
                                                tab.prefix_offsets, tab.suffix_offsets, tab.req_prefix,
                                                prefix_chunks=chunks)
    np.testing.assert_allclose(os_, o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ls_, l, rtol=1e-12, atol=1e-13)


def test_merge_of_disjoint_halves_matches_brute_force():
    rng = np.random.default_rng(8)
    Q, K, V = rng.standard_normal((4, 6)), rng.standard_normal((9, 6)), rng.standard_normal((9, 5))
    parts = [oracle.attend(Q, K[:4], V[:4], 0.5), oracle.attend(Q, K[4:], V[4:], 0.5),
             oracle.attend(Q, K[:0], V[:0], 0.5)]
    o, l = oracle.merge_partials(parts)
    tab = RequestTable(np.array([4]), np.array([0]), np.array([4]))
    # Brute force over the same 9 keys: 4 "prefix" + 5 more rows appended as extra suffix keys
    # cannot be expressed with 4 queries, so compare with a direct loop here.
    for i in range(4):
        s = [0.5 * float(Q[i] @ K[j]) for j in range(9)]
        top = max(s)
        w = [math.exp(t - top) for t in s]
        z = sum(w)
        np.testing.assert_allclose(o[i], sum(w[j] * V[j] for j in range(9)) / z, rtol=1e-12)
        assert abs(l[i] - (top + math.log(z))) < 1e-12


# ----------------------------------------------------------------------------------------
# invariant (4): an empty prefix is plain attention (library routine as the witness)

def test_invariant_empty_prefix_is_plain_attention():
    import torch
    rng = np.random.default_rng(9)
    tab = random_table(rng, 2, 5, 6, 8, p_none=1.0)     # every request has req_prefix = -1
    x = {k: as64(v) for k, v in host_tensors(tab, 3, 16, "fp32", 9).items()}
    o, _ = run_oracle(tab, x)
    for r in range(tab.R):
        a, b = tab.suffix_offsets[r], tab.suffix_offsets[r + 1]
        t = lambda k: torch.from_numpy(np.ascontiguousarray(x[k][a:b].transpose(1, 0, 2)))[None]
        ref = torch.nn.functional.scaled_dot_product_attention(t("q"), t("k_suf"), t("v_suf"), is_causal=False)
        np.testing.assert_allclose(o[a:b], ref[0].numpy().transpose(1, 0, 2), rtol=1e-12, atol=1e-13)


def test_prefix_of_length_zero_equals_no_prefix():
    tab, x = small_random(10, P=2, R=5)
    tab0 = RequestTable(np.zeros(tab.P, np.int64), tab.req_prefix, tab.suffix_len)
    none = RequestTable(tab.prefix_len, np.full(tab.R, -1), tab.suffix_len)
    x0 = dict(x)
    x0["k_cache"] = x["k_cache"][:0]
    x0["v_cache"] = x["v_cache"][:0]
    a, la = run_oracle(tab0, x0)
    b, lb = run_oracle(none, x)
    np.testing.assert_allclose(a, b, rtol=0, atol=0)
    np.testing.assert_allclose(la, lb, rtol=0, atol=0)


# ----------------------------------------------------------------------------------------
# prefix-side step: each prefix's tokens attend over that prefix's tokens only

def _prefix_inputs(seed, lens, H=2, d=8):
    rng = np.random.default_rng(seed)
    T = int(sum(lens))
    so = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    x = {k: rng.standard_normal((T, H, d)) for k in ("q", "k", "v")}
    return so, x


@pytest.mark.parametrize("seed", range(4))
def test_prefix_side_matches_brute_force(seed):
    lens = [0, 1, 5, 9, 3][seed:] + [7]
    so, x = _prefix_inputs(seed, lens)
    o, l = oracle.prefix_side_attention(x["q"], x["k"], x["v"], so)
    # The element-by-element definition, with every prefix as a request that has no cached
    # prefix and its own tokens as the suffix.
    tab = RequestTable(np.zeros(0, np.int64), np.full(len(lens), -1), np.array(lens))
    empty = x["k"][:0]
    bo, bl = brute_force(x["q"], x["k"], x["v"], empty, empty, tab.prefix_offsets, so, tab.req_prefix)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l, bl, rtol=1e-12, atol=1e-13)


def test_prefix_side_matches_library_attention():
    import torch
    so, x = _prefix_inputs(11, [4, 17, 1, 30], H=3, d=16)
    o, _ = oracle.prefix_side_attention(x["q"], x["k"], x["v"], so)
    for p in range(len(so) - 1):
        a, b = so[p], so[p + 1]
        t = lambda k: torch.from_numpy(np.ascontiguousarray(x[k][a:b].transpose(1, 0, 2)))[None]
        ref = torch.nn.functional.scaled_dot_product_attention(t("q"), t("k"), t("v"), is_causal=False)
        np.testing.assert_allclose(o[a:b], ref[0].numpy().transpose(1, 0, 2), rtol=1e-12, atol=1e-13)


def test_prefix_side_token_permutation_and_isolation():
    so, x = _prefix_inputs(12, [6, 9])
    o, _ = oracle.prefix_side_attention(x["q"], x["k"], x["v"], so)
    perm = np.concatenate([np.random.default_rng(3).permutation(6), 6 + np.arange(9)])
    xp = {k: v[perm] for k, v in x.items()}
    op, _ = oracle.prefix_side_attention(xp["q"], xp["k"], xp["v"], so)
    np.testing.assert_allclose(op, o[perm], rtol=1e-12, atol=1e-13)
    # A prefix does not see another prefix's tokens: changing prefix 1 leaves prefix 0 alone.
    x2 = {k: v.copy() for k, v in x.items()}
    x2["k"][6:] += 5.0
    x2["v"][6:] -= 3.0
    o2, _ = oracle.prefix_side_attention(x2["q"], x2["k"], x2["v"], so)
    np.testing.assert_array_equal(o2[:6], o[:6])
    assert not np.allclose(o2[6:], o[6:])


def test_requests_subset_and_empty_suffix():
    tab = RequestTable(np.array([3]), np.array([0, 0, -1]), np.array([2, 0, 3]))
    x = {k: as64(v) for k, v in host_tensors(tab, 1, 4, "fp32", 12).items()}
    o, l = run_oracle(tab, x, requests=[2])
    assert np.isnan(o[:2]).all() and np.isfinite(o[2:]).all()
    full, _ = run_oracle(tab, x)
    np.testing.assert_allclose(o[2:], full[2:], rtol=0, atol=0)


# ----------------------------------------------------------------------------------------
# planted mistakes: each must be caught by at least one pin above

def _pins_pass():
    """Run a compact set of the pins; True when all hold."""
    try:
        tab, x = small_random(21)
        o, l = run_oracle(tab, x)
        ob, lb = run_brute(tab, x)
        np.testing.assert_allclose(o, ob, rtol=1e-9, atol=1e-10)
        np.testing.assert_allclose(l, lb, rtol=1e-9, atol=1e-10)
        os_, ls_ = oracle.bipartite_attention_split(x["q"], x["k_suf"], x["v_suf"], x["k_cache"], x["v_cache"],
                                                    tab.prefix_offsets, tab.suffix_offsets, tab.req_prefix,
                                                    prefix_chunks=3)
        np.testing.assert_allclose(os_, ob, rtol=1e-9, atol=1e-10)
        np.testing.assert_allclose(ls_, lb, rtol=1e-9, atol=1e-10)
        for case in json.load(open(GOLDEN))["cases"]:
            test_hand_derived_examples(case)
        return True
    except AssertionError:
        return False


def _mut_attend(kind):
    orig = oa.attend

    def f(Q, K, V, scale):
        Q, K, V = (np.asarray(a, dtype=np.float64) for a in (Q, K, V))
        if K.shape[0] == 0:
            return orig(Q, K, V, scale)
        S = scale * (Q @ K.T)
        if kind == "sign":
            S = -S
        if kind == "scale_inverted":
            S = S / scale / scale
        mx = S.max(axis=1, keepdims=True)
        E = np.exp(S - mx)
        if kind == "softmax_axis":
            E = E / E.sum(axis=0, keepdims=True)
            return E @ V, (mx + np.log(E.sum(axis=1, keepdims=True)))[:, 0]
        l = E.sum(axis=1, keepdims=True)
        O = (E @ (K[:, :V.shape[1]] if kind == "k_for_v" else V))
        if kind != "no_normalise":
            O = O / l
        lse = (mx + np.log(l))[:, 0]
        if kind == "lse_no_shift":
            lse = np.log(l)[:, 0]
        return O, lse
    return f


def _mut_keys(kind):
    def f(k_suf, v_suf, k_cache, v_cache, po, so, rp, r, h):
        s0, s1 = int(so[r]), int(so[r + 1])
        p = int(rp[r])
        if kind == "drop_prefix" or p < 0:
            return k_suf[s0:s1, h], v_suf[s0:s1, h]
        if kind == "wrong_prefix":
            p = (p + 1) % (len(po) - 1)
        p0, p1 = int(po[p]), int(po[p + 1])
        if kind == "off_by_one":
            p1 = max(p0, p1 - 1)
        hk = (h + 1) % k_suf.shape[1] if kind == "wrong_head" else h
        K = np.concatenate([k_cache[p0:p1, hk], k_suf[s0:s1, hk]])
        V = np.concatenate([v_cache[p0:p1, h], v_suf[s0:s1, h]])
        return K, V
    return f


def _mut_merge(kind):
    def f(parts):
        lses = np.stack([p[1] for p in parts])
        if kind == "merge_plain_sum":
            return sum(p[0] for p in parts), lses.max(axis=0)
        mx = lses.max(axis=0)
        w = np.exp(lses - mx)
        tot = w.sum(axis=0)
        return sum(w[i][:, None] * parts[i][0] for i in range(len(parts))), mx + np.log(tot)   # not normalised
    return f


@pytest.mark.parametrize("target,kind", [
    ("attend", "sign"), ("attend", "scale_inverted"), ("attend", "softmax_axis"),
    ("attend", "k_for_v"), ("attend", "no_normalise"), ("attend", "lse_no_shift"),
    ("request_keys", "drop_prefix"), ("request_keys", "wrong_prefix"),
    ("request_keys", "off_by_one"), ("request_keys", "wrong_head"),
    ("merge_partials", "merge_plain_sum"), ("merge_partials", "merge_unnormalised"),
])
def test_planted_mistake_is_caught(monkeypatch, target, kind):
    assert _pins_pass()
    make = {"attend": _mut_attend, "request_keys": _mut_keys, "merge_partials": _mut_merge}[target]
    monkeypatch.setattr(oa, target, make(kind))
    assert not _pins_pass(), f"planted mistake {target}:{kind} went unnoticed"
