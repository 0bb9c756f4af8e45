"""The pool assembly of the multi-GPU path on one GPU: the row copies that build a rank's local
pool run through the library's K/V pack kernel (bat_copy_rows -> bat_prefix_kv_build) and must
reproduce the prefixes' rows bit for bit, including runs of source-contiguous prefixes, empty
prefixes and ranges out of order.  (The exchange between ranks itself is tested with gloo ranks
on CPU; no run here has more than one GPU.)"""

import numpy as np
import pytest
import torch

from prefix_shared_attention_b200.sharding import bat_copy_rows, exchange_prefixes, hash_owner, local_table, place
from workloads import RequestTable, host_tensors

pytestmark = pytest.mark.gpu


def test_bat_copy_rows_is_exact():
    torch.manual_seed(0)
    src_k = torch.randn(500, 2, 64, device="cuda").bfloat16()
    src_v = torch.randn_like(src_k)
    ranges = [(0, 10, 300), (10, 5, 0), (15, 0, 7), (100, 37, 200), (137, 1, 5), (400, 99, 20)]
    dk = torch.zeros(400, 2, 64, device="cuda", dtype=torch.bfloat16)
    dv = torch.zeros_like(dk)
    bat_copy_rows(src_k, src_v, ranges, dk, dv)
    torch.cuda.synchronize()
    for s0, n, d0 in ranges:
        assert torch.equal(dk[d0:d0 + n], src_k[s0:s0 + n]) and torch.equal(dv[d0:d0 + n], src_v[s0:s0 + n])


def test_single_rank_pool_assembly():
    rng = np.random.default_rng(3)
    tab = RequestTable(rng.integers(1, 300, 9), rng.integers(-1, 9, 30).astype(np.int32), rng.integers(1, 200, 30))
    x = host_tensors(tab, 2, 64, "bf16", 4)
    k, v = x["k_cache"].cuda(), x["v_cache"].cuda()
    pl = place(tab.prefix_len, tab.req_prefix, tab.suffix_len, 1, 2, 64, owner=hash_owner(tab.P, 1))
    assert pl.fetch == [[]]
    kp, vp, nbytes = exchange_prefixes(pl, 0, 1, tab.prefix_len, np.arange(tab.P), k, v, copy_rows=bat_copy_rows)
    torch.cuda.synchronize()
    ltab, pids = local_table(pl, 0, tab)
    po = tab.prefix_offsets
    rows = torch.from_numpy(np.concatenate([np.arange(po[p], po[p + 1]) for p in pids])).cuda()
    assert nbytes == 0 and torch.equal(kp, k[rows]) and torch.equal(vp, v[rows])
    assert ltab.T_cache == kp.shape[0]
