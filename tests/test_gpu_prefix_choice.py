"""The hotness-aware prefix choice run through the forward on the GPU: a synthetic query set
(users with several queries each, items drawn Zipf(1.1)), the cached blocks chosen under a
memory budget, and the resulting batch (some queries reading a cached user, some a cached
item, some a block built for them alone) computed by bat_attention_forward.  Every query's
own rows must match the oracle, and, whichever block was cached, the matching rows of full
bidirectional attention over the query's [user ; item] tokens (Bat lead page, section "This
paper's idea": either block may be the prefix without changing the result)."""

import math

import numpy as np
import pytest
import torch

import oracle
import prefix_shared_attention_b200 as bat
from prefix_shared_attention_b200 import prefix_choice as pc
from workloads import zipf_ranks

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_REL = 2e-2, 5e-3


def blocks(n, lens, H, d, g):
    return [{k: torch.randn(int(L), H, d, generator=g).bfloat16() for k in "qkv"} for L in lens]


@pytest.mark.parametrize("d", [64, 128])
def test_chosen_batch_matches_oracle_and_full_attention(d):
    rng = np.random.default_rng(40 + d)
    H = 2
    n_users, per_user, n_items = 24, 5, 40
    user_len = rng.integers(16, 300, n_users)
    item_len = rng.integers(16, 300, n_items)
    q_user = np.repeat(np.arange(n_users), per_user)
    q_item = rng.permutation(n_items)[zipf_ranks(rng, n_items, 1.1, len(q_user)) - 1]
    budget = 0.5 * 2 * float(user_len.sum()) * H * d * 2
    ch = pc.choose(user_len, item_len, q_user, q_item, budget, H, d)
    kinds = set(ch.prefix_kind.tolist())
    assert pc.ITEM in kinds and pc.USER in kinds, kinds     # both kinds of prefix are exercised
    tab, prefix_src, suffix_src = pc.to_request_table(ch, user_len, item_len, q_user, q_item)

    g = torch.Generator().manual_seed(d)
    U, I = blocks(n_users, user_len, H, d, g), blocks(n_items, item_len, H, d, g)
    blk = lambda kind, idx: U[idx] if kind == pc.USER else I[idx]
    x = {"k_cache": torch.cat([blk(*s)["k"] for s in prefix_src]), "v_cache": torch.cat([blk(*s)["v"] for s in prefix_src]),
         "q": torch.cat([blk(*s)["q"] for s in suffix_src]), "k_suf": torch.cat([blk(*s)["k"] for s in suffix_src]),
         "v_suf": torch.cat([blk(*s)["v"] for s in suffix_src])}
    xd = {k: v.cuda() for k, v in x.items()}
    out = torch.full_like(xd["q"], float("nan"))
    with bat.Plan(tab.req_prefix, tab.suffix_offsets, tab.prefix_offsets, H, d) as plan:
        bat.bat_attention_forward(plan, xd["q"], xd["k_suf"], xd["v_suf"], xd["k_cache"], xd["v_cache"], out=out)
        assert bat.bat_get_device_status() == bat.BAT_OK, bat.last_error()
    o = out.float().cpu().double().numpy()
    ref, _ = oracle.bipartite_attention(x["q"], x["k_suf"], x["v_suf"], x["k_cache"], x["v_cache"],
                                        tab.prefix_offsets, tab.suffix_offsets, tab.req_prefix)
    diff = np.abs(o - ref)
    assert np.isfinite(o).all() and diff.max() <= MAX_ABS and diff.sum() / np.abs(ref).sum() <= MEAN_REL

    # Role-swap check per query: the rows of its own block equal full attention over [user ; item].
    so = tab.suffix_offsets
    for q in range(0, len(q_user), 7):
        u, it = U[int(q_user[q])], I[int(q_item[q])]
        own_user = suffix_src[q][0] == pc.USER
        for h in range(H):
            Q, K, V = (torch.cat([u[k][:, h], it[k][:, h]]).double().numpy() for k in "qkv")
            mono, _ = oracle.attend(Q, K, V, 1 / math.sqrt(d))
            want = mono[:len(u["q"])] if own_user else mono[len(u["q"]):]
            got = o[so[q]:so[q + 1], h]
            err = np.abs(got - want)
            assert err.max() <= MAX_ABS and err.sum() / np.abs(want).sum() <= MEAN_REL, (q, h)
