"""The GBLA work list (host only): every 128-token tile of every (sequence, head) is in exactly
one chunk, chunks of a pair are consecutive and balanced, empty sequences get none, the
workspace covers the partial states, and bad tables are rejected.  CPU only."""

import numpy as np
import pytest

import prefix_shared_attention_b200 as bat


@pytest.mark.parametrize("lens,H,sms", [([1, 3, 127, 128, 129, 300, 0, 517], 2, 148), ([32768] * 8, 8, 148),
                                        ([700, 1, 256, 383], 3, 4), ([0, 0], 1, 148)])
def test_chunks_cover_every_tile_once(lens, H, sms):
    so = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    with bat.GblaPlan(so, H, host_only=True, num_sms=sms) as p:
        ch = p.chunks()
        ws = p.workspace_bytes
    seen = {}
    for c in ch:
        assert c["n_tiles"] >= 1 and 0 <= c["head"] < H
        i = int(np.searchsorted(so, c["seq_lo"], side="right") - 1)
        while so[i + 1] == so[i]:
            i += 1
        assert c["seq_lo"] == so[i] and c["seq_hi"] == so[i + 1]
        for t in range(c["tile0"], c["tile0"] + c["n_tiles"]):
            key = (i, int(c["head"]), t)
            assert key not in seen, f"tile {key} in two chunks"
            seen[key] = int(c["pair"])
    want = {(i, h, t) for i, L in enumerate(lens) for h in range(H) for t in range((L + 127) // 128)}
    assert set(seen) == want
    # Chunks of one pair are consecutive and differ in size by at most one tile.
    pairs = ch["pair"]
    assert (np.diff(pairs) >= 0).all()
    for pr in np.unique(pairs):
        sizes = ch["n_tiles"][pairs == pr]
        assert sizes.max() - sizes.min() <= 1
    n_pairs = len(np.unique(pairs)) if len(ch) else 0
    assert ws >= len(ch) * (128 * 128 + 128) * 4 + n_pairs * (128 * 128 * 2 + 128 * 4)
    if sum(lens) >= 128 * 2 * sms:
        assert len(ch) >= sms, "too few chunks to fill the GPU"


@pytest.mark.parametrize("kw,code", [(dict(d=64), bat.BAT_ERR_UNSUPPORTED), (dict(H=0), bat.BAT_ERR_INVALID_ARG)])
def test_plan_rejects(kw, code):
    args = dict(H=2, d=128)
    args.update(kw)
    with pytest.raises(bat.BatError) as e:
        bat.GblaPlan(np.array([0, 10]), host_only=True, **args)
    assert e.value.status == code


def test_plan_rejects_non_monotone_offsets():
    with pytest.raises(bat.BatError) as e:
        bat.GblaPlan(np.array([0, 10, 5]), 2, host_only=True)
    assert e.value.status == bat.BAT_ERR_INVALID_ARG and "monotone" in str(e.value)
