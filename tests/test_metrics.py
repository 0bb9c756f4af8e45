"""The algorithmic work figures behind TFLOP/s and the roofline (metrics.py): pinned by brute
force on small tables (every multiply-add and every distinct row read, counted one by one)
and by the closed-form totals of the configs' definitions.  CPU only."""

import numpy as np
import pytest

from prefix_shared_attention_b200.metrics import algorithmic_bytes, algorithmic_flops
from workloads import make_table, random_table


def brute_force(tab, H, d, elt):
    flops = 0
    rows_read = set()
    for r in range(tab.R):
        p = int(tab.req_prefix[r])
        keys = [("cache", i) for i in range(tab.prefix_offsets[p], tab.prefix_offsets[p + 1])] if p >= 0 else []
        keys += [("suffix", i) for i in range(tab.suffix_offsets[r], tab.suffix_offsets[r + 1])]
        for t in range(tab.suffix_offsets[r], tab.suffix_offsets[r + 1]):
            for _ in keys:
                flops += 2 * (2 * d)          # q.k and p*v: d multiply-adds each, 2 FLOPs apiece
            rows_read.add(("q", t))
            rows_read.add(("out", t))
        for kind, i in keys:
            rows_read.add(("k_" + kind, i))
            rows_read.add(("v_" + kind, i))
    return flops * H, len(rows_read) * H * d * elt


@pytest.mark.parametrize("seed", range(5))
def test_brute_force_small_tables(seed):
    tab = random_table(np.random.default_rng(seed), P=3, R=6, max_prefix=40, max_suffix=30)
    H, d = 2, 8
    f, b = brute_force(tab, H, d, 2)
    assert algorithmic_flops(tab.prefix_len, tab.req_prefix, tab.suffix_len, H, d) == f
    assert algorithmic_bytes(tab.prefix_len, tab.req_prefix, tab.suffix_len, H, d, 2) == b


def test_unreferenced_prefix_costs_nothing():
    tab = make_table("tiny")
    f0 = algorithmic_flops(tab.prefix_len, tab.req_prefix, tab.suffix_len, 2, 32)
    b0 = algorithmic_bytes(tab.prefix_len, tab.req_prefix, tab.suffix_len, 2, 32, 4)
    extra = np.concatenate([tab.prefix_len, [1000]])
    assert algorithmic_flops(extra, tab.req_prefix, tab.suffix_len, 2, 32) == f0
    assert algorithmic_bytes(extra, tab.req_prefix, tab.suffix_len, 2, 32, 4) == b0


@pytest.mark.parametrize("name,flops,nbytes", [
    # 512 requests, Ls = 128 over Lp = 256; 64 prefixes of 256; H = 8, d = 64, bf16
    ("user-as-prefix", 512 * 4 * 128 * (256 + 128) * 8 * 64, (4 * 512 * 128 + 2 * 64 * 256) * 8 * 64 * 2),
    # 256 requests, Ls = 256 over Lp = 8192; 16 prefixes of 8192; H = 16, d = 128, bf16
    ("long-user-history", 256 * 4 * 256 * (8192 + 256) * 16 * 128, (4 * 256 * 256 + 2 * 16 * 8192) * 16 * 128 * 2),
    # 8192 requests, Ls = 512 over Lp = 32 (FLOPs do not depend on which items are drawn)
    ("item-as-prefix", 8192 * 4 * 512 * (32 + 512) * 8 * 64, None),
])
def test_config_totals(name, flops, nbytes):
    tab = make_table(name)
    from workloads import CONFIGS
    spec = CONFIGS[name]
    assert algorithmic_flops(tab.prefix_len, tab.req_prefix, tab.suffix_len, spec.H, spec.d) == flops
    if nbytes is not None:
        assert algorithmic_bytes(tab.prefix_len, tab.req_prefix, tab.suffix_len, spec.H, spec.d, 2) == nbytes
