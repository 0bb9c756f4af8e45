"""Plain fp64 definition of bipartite prefix-shared attention (TEST INFRASTRUCTURE ONLY).

Source: "Bat: Efficient Generative Recommender Serving with Bipartite
Attention" (the lead page).  Its section "This paper's idea" says that user
and item tokens are order-agnostic, so either block may be the cached
prefix "without compromising accuracy"; section "Why it works" says the
prefix choice does not change the result; section "Problem" describes the
cached prefix K/V as computed once and reused by every query that shares it.
The page prints no formula, so the oracle takes the plainest reading:

    For request r with cached prefix K/V (Kp, Vp) of Lp rows (Lp = 0 when the
    request has no prefix) and its own suffix (Qs, Ks, Vs) of Ls rows, per head

        O_r = softmax_row( scale * Qs . [Kp ; Ks]^T ) . [Vp ; Vs]

    non-causal (no mask at all), scale = 1/sqrt(d) unless given.  Only the
    suffix rows are produced.

That is exactly the suffix rows of full bidirectional softmax attention over
the request's concatenated tokens, which is why swapping the roles of the two
blocks leaves the result unchanged: softmax attention with no mask is
invariant to the order of its keys.

Readings (the pages are silent on these):
  * scale 1/sqrt(d); heads are plain multi-head (as many K/V heads as Q heads);
  * no causal mask anywhere (order-agnostic tokens);
  * the natural-log LSE of the scaled scores is reported per row;
  * the split form merges per-chunk partials by log-sum-exp (the standard
    identity for softmax over a union of disjoint key sets).

Everything is float64 numpy.  Inputs are whatever values the caller passes
(bf16-rounded values upcast exactly to fp64, or fp32 values).
"""

from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np


def attend(Q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of one head with no mask, fp64.

    Q [n, d], K [m, d], V [m, dv] -> (O [n, dv], lse [n]) where
    O = softmax(scale * Q K^T) V row by row and lse = log sum_j exp(scale * q.k_j).
    With m == 0 the softmax is over an empty set: O = 0 and lse = -inf (the
    identity element of the log-sum-exp merge).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    n, m = Q.shape[0], K.shape[0]
    if m == 0:
        return np.zeros((n, V.shape[1])), np.full(n, -np.inf)
    S = scale * (Q @ K.T)                     # [n, m] scores
    mx = S.max(axis=1, keepdims=True)         # shift for a stable exp (cancels in the ratio)
    E = np.exp(S - mx)
    l = E.sum(axis=1, keepdims=True)
    O = (E @ V) / l
    lse = (mx + np.log(l))[:, 0]
    return O, lse


def request_keys(k_suf, v_suf, k_cache, v_cache, prefix_offsets, suffix_offsets, req_prefix,
                 r: int, h: int) -> Tuple[np.ndarray, np.ndarray]:
    """Keys and values request ``r`` attends over for head ``h``: [cached prefix ; own suffix]."""
    s0, s1 = int(suffix_offsets[r]), int(suffix_offsets[r + 1])
    p = int(req_prefix[r])
    if p >= 0:
        p0, p1 = int(prefix_offsets[p]), int(prefix_offsets[p + 1])
        K = np.concatenate([k_cache[p0:p1, h, :], k_suf[s0:s1, h, :]], axis=0)
        V = np.concatenate([v_cache[p0:p1, h, :], v_suf[s0:s1, h, :]], axis=0)
    else:
        K, V = k_suf[s0:s1, h, :], v_suf[s0:s1, h, :]
    return K, V


def _as64(x):
    if hasattr(x, "detach"):  # a torch tensor; the oracle itself stays numpy
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def bipartite_attention(q, k_suf, v_suf, k_cache, v_cache, prefix_offsets, suffix_offsets,
                        req_prefix, scale: Optional[float] = None,
                        requests: Optional[Iterable[int]] = None):
    """O and LSE for every suffix row of the selected requests.

    q, k_suf, v_suf: [T_suf, H, d]; k_cache, v_cache: [T_cache, H, d];
    prefix_offsets [P+1], suffix_offsets [R+1], req_prefix [R] (-1 = none).
    Returns (out [T_suf, H, d] fp64, lse [H, T_suf] fp64); rows of requests
    that were not selected are NaN.
    """
    q, k_suf, v_suf, k_cache, v_cache = map(_as64, (q, k_suf, v_suf, k_cache, v_cache))
    T, H, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    R = len(req_prefix)
    out = np.full((T, H, v_suf.shape[2]), np.nan)
    lse = np.full((H, T), np.nan)
    for r in (range(R) if requests is None else requests):
        s0, s1 = int(suffix_offsets[r]), int(suffix_offsets[r + 1])
        if s1 == s0:
            continue
        for h in range(H):
            K, V = request_keys(k_suf, v_suf, k_cache, v_cache, prefix_offsets, suffix_offsets,
                                req_prefix, r, h)
            O, L = attend(q[s0:s1, h, :], K, V, scale)
            out[s0:s1, h, :] = O
            lse[h, s0:s1] = L
    return out, lse


def prefix_side_attention(q, k, v, src_offsets, scale: Optional[float] = None,
                          prefixes: Optional[Iterable[int]] = None):
    """The prefix tokens' own outputs (the prefix-side step).

    Lead page, section "Problem": the chosen prefix block's K/V is computed once and cached
    for the requests that reuse it; section "This paper's idea": the tokens of a block are
    order-agnostic.  Within its own block a prefix token therefore attends, with no mask, over
    that block's tokens only, per head:

        O_p = softmax_row( scale * Qp . Kp^T ) . Vp

    q, k, v: [T, H, d]; prefix p owns rows [src_offsets[p], src_offsets[p+1]).
    Returns (out [T, H, d] fp64, lse [H, T] fp64); rows of prefixes not selected are NaN.
    """
    q, k, v = map(_as64, (q, k, v))
    T, H, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    n = len(src_offsets) - 1
    out = np.full((T, H, v.shape[2]), np.nan)
    lse = np.full((H, T), np.nan)
    for p in (range(n) if prefixes is None else prefixes):
        s0, s1 = int(src_offsets[p]), int(src_offsets[p + 1])
        if s1 == s0:
            continue
        for h in range(H):
            O, L = attend(q[s0:s1, h, :], k[s0:s1, h, :], v[s0:s1, h, :], scale)
            out[s0:s1, h, :] = O
            lse[h, s0:s1] = L
    return out, lse


def merge_partials(parts: Sequence[Tuple[np.ndarray, np.ndarray]]) -> Tuple[np.ndarray, np.ndarray]:
    """Log-sum-exp merge of softmax partials over disjoint key sets.

    Each part is (O_i [n, dv], lse_i [n]) with O_i already normalised over its
    own keys.  Then lse = log sum_i exp(lse_i) and O = sum_i exp(lse_i - lse) O_i.
    Parts with lse_i = -inf (no keys) carry zero weight.
    """
    lses = np.stack([p[1] for p in parts], axis=0)          # [k, n]
    mx = lses.max(axis=0)
    safe = np.where(np.isfinite(mx), mx, 0.0)
    w = np.exp(lses - safe)                                   # exp(-inf) = 0
    tot = w.sum(axis=0)
    lse = safe + np.log(tot)
    O = sum(w[i][:, None] * parts[i][0] for i in range(len(parts))) / tot[:, None]
    return O, lse


def chunk_partial(Q, K, V, scale, k0: int, k1: int):
    """Partial (O, lse) of Q over keys [k0, k1) only."""
    return attend(Q, K[k0:k1], V[k0:k1], scale)


def bipartite_attention_split(q, k_suf, v_suf, k_cache, v_cache, prefix_offsets, suffix_offsets,
                              req_prefix, scale: Optional[float] = None, prefix_chunks: int = 1,
                              requests: Optional[Iterable[int]] = None):
    """Split form: the prefix keys cut into ``prefix_chunks`` contiguous chunks, the suffix
    keys as one more part, each part attended separately and the partials merged by
    log-sum-exp.  Must equal :func:`bipartite_attention` (invariant 3)."""
    q, k_suf, v_suf, k_cache, v_cache = map(_as64, (q, k_suf, v_suf, k_cache, v_cache))
    T, H, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.full((T, H, v_suf.shape[2]), np.nan)
    lse = np.full((H, T), np.nan)
    for r in (range(len(req_prefix)) if requests is None else requests):
        s0, s1 = int(suffix_offsets[r]), int(suffix_offsets[r + 1])
        if s1 == s0:
            continue
        p = int(req_prefix[r])
        Lp = 0 if p < 0 else int(prefix_offsets[p + 1] - prefix_offsets[p])
        for h in range(H):
            Qs = q[s0:s1, h, :]
            parts = []
            if p >= 0:
                p0 = int(prefix_offsets[p])
                Kp, Vp = k_cache[p0:p0 + Lp, h, :], v_cache[p0:p0 + Lp, h, :]
                cuts = [(Lp * i) // prefix_chunks for i in range(prefix_chunks + 1)]
                for i in range(prefix_chunks):
                    parts.append(chunk_partial(Qs, Kp, Vp, scale, cuts[i], cuts[i + 1]))
            parts.append(attend(Qs, k_suf[s0:s1, h, :], v_suf[s0:s1, h, :], scale))
            O, L = merge_partials(parts)
            out[s0:s1, h, :] = O
            lse[h, s0:s1] = L
    return out, lse
