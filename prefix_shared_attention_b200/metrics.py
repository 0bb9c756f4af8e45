"""Algorithmic work of one forward launch (for throughput and roofline figures).

FLOPs: Q.K^T and P.V over exactly the keys each suffix row must see, 2 FLOPs per
multiply-add: 4 * Ls * (Lp + Ls) * H * d per request.  The prefix rows' own attention
and the prefix K/V construction are the work the cache avoids and are not counted.

Bytes: Q, K and V of every suffix row read once and O written once, plus the K/V of every
referenced prefix read once: (4 * T_suf + 2 * sum(Lp over referenced prefixes)) * H * d * e.
"""

from __future__ import annotations

import numpy as np


def algorithmic_flops(prefix_len, req_prefix, suffix_len, H: int, d: int) -> float:
    prefix_len = np.asarray(prefix_len, dtype=np.float64)
    req_prefix = np.asarray(req_prefix)
    Ls = np.asarray(suffix_len, dtype=np.float64)
    Lp = np.where(req_prefix >= 0, prefix_len[np.clip(req_prefix, 0, None)] if prefix_len.size else 0.0, 0.0)
    return float(np.sum(4.0 * Ls * (Lp + Ls)) * H * d)


def algorithmic_bytes(prefix_len, req_prefix, suffix_len, H: int, d: int, elt: int) -> float:
    prefix_len = np.asarray(prefix_len, dtype=np.int64)
    req_prefix = np.asarray(req_prefix)
    ref = np.unique(req_prefix[req_prefix >= 0])
    Lp_ref = float(prefix_len[ref].sum()) if ref.size else 0.0
    T_suf = float(np.sum(np.asarray(suffix_len, dtype=np.float64)))
    return (4.0 * T_suf + 2.0 * Lp_ref) * H * d * elt
