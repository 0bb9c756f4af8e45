"""Deadlock freedom of the attention kernel's mbarrier protocol, on a discrete-event model of
its roles (tests/protocol_model.py): the rings used at d = 128 (a K ring of two and a V ring of
one, one P hand-off per tile) and at d = 64 (one shared ring of ten, P handed off in halves),
plus smaller rings, over work lists from the host grouping pass.  CPU only."""

import numpy as np
import pytest

import prefix_shared_attention_b200 as bat
from protocol_model import simulate
from workloads import RequestTable, make_table, random_table

# (two rings, K stages, V stages, shared-ring stages, P hand-offs per tile)
KERNEL_D128 = (True, 2, 1, 0, 1)
KERNEL_D64 = (False, 0, 0, 10, 2)
SMALLER = [(True, 1, 1, 0, 1), (True, 1, 2, 0, 2), (False, 0, 0, 2, 1), (False, 0, 0, 3, 2)]


def work_items(tab, H=1, **kw):
    with bat.Plan(tab.req_prefix, tab.suffix_offsets, tab.prefix_offsets, H, 128, host_only=True, num_sms=148,
                  **kw) as p:
        return p.items()


def cta_sequences(items, n, seed):
    """Item sequences one CTA may take: list order is handed out by a global counter, so a
    CTA gets an increasing, otherwise arbitrary, subsequence."""
    rng = np.random.default_rng(seed)
    out = [items[: min(len(items), 40)]]
    for _ in range(n):
        k = int(rng.integers(1, min(len(items), 30) + 1))
        idx = np.sort(rng.choice(len(items), size=k, replace=False))
        out.append(items[idx])
    return out


def tables():
    yield "ragged", RequestTable(np.array([300, 77, 0]), np.array([0, 0, 1, -1, 2, 1], np.int32),
                                 np.array([200, 129, 64, 33, 260, 600]))
    for sd in range(6):
        yield f"random{sd}", random_table(np.random.default_rng(sd), P=4, R=9, max_prefix=900, max_suffix=1200,
                                          min_suffix=1)
    yield "user-as-prefix[:64]", make_table("user-as-prefix").compact(np.arange(64))


@pytest.mark.parametrize("cfg", [KERNEL_D128, KERNEL_D64] + SMALLER,
                         ids=["d128-kernel", "d64-kernel", "two-1-1", "two-1-2-halves", "shared-2", "shared-3-halves"])
def test_protocol_has_no_deadlock(cfg):
    for name, tab in tables():
        for split in (0, 2):
            items = work_items(tab, split_mode=split)
            for i, seq in enumerate(cta_sequences(items, 3, seed=len(items) + split)):
                r = simulate(seq, *cfg, seed=1000 * i + split)
                assert r == "ok", f"{name} split={split} sequence {i}: {r}"


def test_model_detects_a_missing_release():
    """The model is not vacuous: a V ring whose slots never free deadlocks once it wraps."""
    import protocol_model as pm

    class NoRelease(pm.Bar):
        def arrive(self, n=1):
            if "v_empty" in self.name:
                return
            super().arrive(n)

    items = work_items(RequestTable(np.array([600]), np.array([0, 0], np.int32), np.array([256, 256])))
    orig = pm.Bar
    pm.Bar = NoRelease
    try:
        r = pm.simulate(items, *KERNEL_D128, seed=3)
    finally:
        pm.Bar = orig
    assert r.startswith("deadlock") and "v_empty" in r


def test_model_needs_the_zeroed_hand_off():
    """The second consumer of a ragged V tile really waits for the first one's zeroing: if the
    zeroing issuer never signals, the model deadlocks on v_zeroed."""
    import protocol_model as pm

    class NoZeroed(pm.Bar):
        def arrive(self, n=1):
            if "v_zeroed" in self.name:
                return
            super().arrive(n)

    # One prefix of 600 keys (last tile holds 88: not a multiple of 16) read by two requests.
    items = work_items(RequestTable(np.array([600]), np.array([0, 0], np.int32), np.array([256, 256])))
    assert any(int(w["n_q"]) == 2 for w in items)
    orig = pm.Bar
    pm.Bar = NoZeroed
    try:
        results = [pm.simulate(items, *cfg, seed=5) for cfg in (KERNEL_D128, KERNEL_D64)]
    finally:
        pm.Bar = orig
    for r in results:
        assert r.startswith("deadlock") and "v_zeroed" in r, r
