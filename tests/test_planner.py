"""Host grouping pass (C++, reached through the C ABI with host-only plans; no GPU).

Checked from the work list alone, by reconstruction: every (request, head, suffix row) is
produced exactly once; every query tile sees exactly the keys of [its request's prefix ;
its request's suffix]; items that pair two query tiles read one prefix; split chunks
partition the key stream and their merge jobs cover the split tiles."""

import numpy as np
import pytest

import prefix_shared_attention_b200 as bat
from workloads import RequestTable, make_table, random_table

T = 128


def plan_of(tab: RequestTable, H=2, d=64, **kw):
    return bat.Plan(tab.req_prefix, tab.suffix_offsets, tab.prefix_offsets, H=H, d=d, host_only=True, **kw)


def key_sets_by_tile(items):
    """(head, qX_row0, X-rows) -> list of (prefix range, suffix range) per chunk."""
    out = {}
    for it in items:
        for x in range(int(it["n_q"])):
            q0 = int(it["qA_row0"] if x == 0 else it["qB_row0"])
            rows = int(it["qA_rows"] if x == 0 else it["qB_rows"])
            own_a = it["shared"] or x == 0
            s0 = int(it["sA_row0"] if own_a else it["sB_row0"])
            sl = int(it["sA_len"] if own_a else it["sB_len"])
            key = (int(it["head"]), q0, rows)
            out.setdefault(key, []).append(((int(it["pre_row0"]), int(it["pre_len"])), (s0, sl),
                                            int(it["split_slot"]) + x if it["split_slot"] >= 0 else -1))
    return out


def check_plan(tab: RequestTable, H=2, **kw):
    with plan_of(tab, H=H, **kw) as p:
        items, merges, info = p.items(), p.merges(), p.info()
    so, po = tab.suffix_offsets, tab.prefix_offsets
    row_req = np.repeat(np.arange(tab.R), tab.suffix_len)
    covered = np.zeros((H, tab.T_suf), np.int64)
    tiles = key_sets_by_tile(items)
    merged = {(int(m["head"]), int(m["q_row0"]), int(m["q_rows"])): m for m in merges}
    slots_seen = set()
    for (h, q0, rows), chunks in tiles.items():
        assert 1 <= rows <= T
        r = row_req[q0]
        assert (row_req[q0:q0 + rows] == r).all(), "a query tile straddles requests"
        assert q0 == so[r] + T * ((q0 - so[r]) // T), "query tiles start on 128-row boundaries of the request"
        covered[h, q0:q0 + rows] += 1
        p = tab.req_prefix[r]
        want_pre = set(range(po[p], po[p + 1])) if p >= 0 else set()
        want_suf = set(range(so[r], so[r + 1]))
        got_pre, got_suf = [], []
        for (pr0, pl), (s0, sl), slot in chunks:
            got_pre += list(range(pr0, pr0 + pl))
            got_suf += list(range(s0, s0 + sl))
            if slot >= 0:
                assert slot not in slots_seen
                slots_seen.add(slot)
        assert sorted(got_pre) == sorted(want_pre), "prefix keys of the tile"
        assert sorted(got_suf) == sorted(want_suf), "suffix keys of the tile"
        assert len(got_pre) == len(set(got_pre)) and len(got_suf) == len(set(got_suf)), "chunks overlap"
        if len(chunks) > 1:
            m = merged[(h, q0, rows)]
            assert m["n_chunks"] == len(chunks)
            want_slots = {int(m["slot0"]) + c * int(m["slot_stride"]) for c in range(int(m["n_chunks"]))}
            assert want_slots == {c[2] for c in chunks}
        else:
            assert chunks[0][2] == -1 and (h, q0, rows) not in merged
    assert (covered == 1).all(), "every (head, suffix row) exactly once"
    assert info.n_slots == len(slots_seen)
    # Pairs of query tiles in one item read one prefix (same group).
    for it in items:
        if it["n_q"] == 2:
            ra, rb = row_req[it["qA_row0"]], row_req[it["qB_row0"]]
            assert tab.req_prefix[ra] == tab.req_prefix[rb]
            assert bool(it["shared"]) == (ra == rb)
    return items, merges, info


@pytest.mark.parametrize("name", ["tiny", "user-as-prefix", "item-as-prefix", "long-user-history"])
def test_named_configs(name):
    tab = make_table(name)
    H = 2
    items, _, info = check_plan(tab, H=H)
    if name == "user-as-prefix":
        # 8 one-tile requests per user pair up into 4 items that stream the user's prefix once.
        assert info.n_items == 64 * 4 * H and (items["n_q"] == 2).all() and not items["shared"].any()
    if name == "long-user-history":
        assert (items["shared"] == 1).all() and (items["pre_len"] == 8192).all()


@pytest.mark.parametrize("seed", range(8))
def test_random_ragged_tables(seed):
    rng = np.random.default_rng(seed)
    tab = random_table(rng, P=5, R=23, max_prefix=700, max_suffix=600, min_suffix=0)
    check_plan(tab, H=3)


@pytest.mark.parametrize("chunk", [1, 2, 3])
def test_forced_split(chunk):
    rng = np.random.default_rng(40 + chunk)
    tab = random_table(rng, P=3, R=9, max_prefix=900, max_suffix=500)
    items, merges, info = check_plan(tab, H=2, split_mode=2, split_chunk_tiles=chunk)
    assert info.n_merges > 0 and info.workspace_bytes == info.n_slots * 128 * (64 * 4 + 4)


def test_auto_split_balances_one_long_request():
    # One request with an 8192-token prefix on 148 SMs: the single item would idle 147 SMs.
    tab = RequestTable(np.array([8192]), np.array([0]), np.array([128]))
    items, merges, info = check_plan(tab, H=2)
    assert info.n_items > 2 * 8 and info.n_merges == 2
    tab2 = RequestTable(np.array([8192]), np.array([0]), np.array([128]))
    with plan_of(tab2, H=2, split_mode=1) as p:
        assert p.info().n_merges == 0 and p.info().n_items == 2


def test_edge_tables():
    check_plan(RequestTable(np.zeros(0), np.zeros(0, np.int32), np.zeros(0)), H=1)               # R = 0
    check_plan(RequestTable(np.array([5, 7]), np.array([-1, -1, -1]), np.array([1, 129, 256])))  # no prefix at all
    check_plan(RequestTable(np.array([5, 0, 300]), np.array([2, 1, 2]), np.array([0, 3, 0])))    # empty suffixes, empty prefix
    items, _, info = check_plan(RequestTable(np.array([4, 9]), np.array([0, 0]), np.array([1, 1])), H=1)
    assert info.n_items == 1    # the unreferenced prefix 1 produces nothing


def test_group_items_are_contiguous_and_heaviest_group_first():
    tab = make_table("item-as-prefix")
    with plan_of(tab, H=2) as p:
        items = p.items()
    groups = items["group"]
    seen, last = set(), None
    for g in groups:
        if g != last:
            assert g not in seen, "a group's items are not contiguous"
            seen.add(g)
            last = g
    # The hottest item (most requests) comes first.
    counts = np.bincount(tab.req_prefix, minlength=tab.P)
    assert groups[0] == np.argmax(counts)


def test_prefix_side_plan_is_the_no_cache_plan():
    """bat_plan_create_prefix_side: every prefix becomes a request with no cached prefix whose
    own tokens are the prefix's, so its work list equals bat_plan_create's for that table."""
    lens = [0, 1, 127, 128, 129, 300, 5, 1000]
    tab = RequestTable(np.zeros(0, np.int64), np.full(len(lens), -1), np.array(lens))
    with bat.Plan.prefix_side(tab.suffix_offsets, H=3, d=128, host_only=True) as p:
        items, info = p.items(), p.info()
    with plan_of(tab, H=3, d=128) as q:
        ref = q.items()
    assert info.P == 0 and info.R == len(lens) and info.T_cache == 0 and info.T_suf == sum(lens)
    np.testing.assert_array_equal(items, ref)
    assert (items["pre_len"] == 0).all()
    check_plan(tab, H=3, d=128)


def test_prefix_side_plan_argument_errors():
    with pytest.raises(bat.BatError) as e:
        bat.Plan.prefix_side(np.array([0, 5, 3]), H=2, d=64, host_only=True)   # not monotone
    assert e.value.status == bat.BAT_ERR_INVALID_ARG
    with pytest.raises(bat.BatError) as e:
        bat.Plan.prefix_side(np.array([0, 5]), H=2, d=96, host_only=True)      # unsupported d
    assert e.value.status == bat.BAT_ERR_UNSUPPORTED
    with bat.Plan.prefix_side(np.array([0]), H=2, d=64, host_only=True) as p:  # no prefixes: empty plan
        assert p.info().n_items == 0
