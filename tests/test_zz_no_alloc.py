"""bat_attention_forward_noalloc, the forward for callers that cannot allocate device memory
(their memory is owned by another allocator, or cudaMalloc/cudaFree would synchronize a
latency-critical loop).  Its split-path scratch is a fixed array inside the library.

Called through the C ABI and compared with bat_attention_forward (caller-allocated workspace)
on the same plan, twice in a row, since the fixed array keeps the previous call's contents.
This file sorts last so a stop-at-first-failure run has already run every other test; it
also passes on its own in a fresh process."""

import ctypes as C

import numpy as np
import pytest
import torch

import prefix_shared_attention_b200 as bat
from prefix_shared_attention_b200 import _bat
from workloads import RequestTable, host_tensors, random_table

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_REL = 5e-3
SCRATCH_LIMIT = 32 << 20


def _ptr(t):
    return t.data_ptr() if t is not None else None


def _inputs(tab, H, d, dtype, seed):
    x = host_tensors(tab, H, d, dtype, seed)
    return {k: v.cuda() for k, v in x.items()}


def _close(a, b):
    a, b = a.float().cpu().double().numpy(), b.float().cpu().double().numpy()
    assert np.isfinite(a).all()
    diff = np.abs(a - b)
    return float(diff.max()), float(diff.sum() / max(np.abs(b).sum(), 1e-30))


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("fp32", 64)])
def test_noalloc_matches_workspace_entry_point_twice(dtype, d):
    rng = np.random.default_rng(77 + d)
    tab = random_table(rng, P=3, R=6, max_prefix=700, max_suffix=400)
    H = 2
    xd = _inputs(tab, H, d, dtype, 5)
    code = bat.BAT_BF16 if dtype == "bf16" else bat.BAT_FP32
    stream = torch.cuda.current_stream().cuda_stream
    with bat.Plan(tab.req_prefix, tab.suffix_offsets, tab.prefix_offsets, H, d, code, split_mode=2,
                  split_chunk_tiles=1) as plan:
        need = plan.workspace_bytes
        assert 0 < need <= SCRATCH_LIMIT          # the scratch really is used
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        ref = torch.empty_like(xd["q"])
        ref_lse = torch.empty((H, tab.T_suf), device="cuda")
        st = _bat.lib.bat_attention_forward(plan.handle, _ptr(xd["q"]), _ptr(xd["k_suf"]), _ptr(xd["v_suf"]),
                                            _ptr(xd["k_cache"]), _ptr(xd["v_cache"]), 0.0, code, _ptr(ref),
                                            _ptr(ref_lse), _ptr(ws), need, stream)
        assert st == bat.BAT_OK, bat.last_error()
        for call in range(2):
            out = torch.full_like(xd["q"], float("nan"))
            lse = torch.full((H, tab.T_suf), float("nan"), device="cuda")
            st = _bat.lib.bat_attention_forward_noalloc(plan.handle, _ptr(xd["q"]), _ptr(xd["k_suf"]),
                                                        _ptr(xd["v_suf"]), _ptr(xd["k_cache"]), _ptr(xd["v_cache"]),
                                                        0.0, code, _ptr(out), _ptr(lse), stream)
            assert st == bat.BAT_OK, bat.last_error()
            assert bat.bat_get_device_status() == bat.BAT_OK, bat.last_error()
            mx, mr = _close(out, ref)
            assert mx <= MAX_ABS and mr <= MEAN_REL, (call, mx, mr)
            lmx, _ = _close(lse, ref_lse)
            assert lmx <= MAX_ABS, (call, lmx)


def test_noalloc_without_split_scratch():
    tab = RequestTable(np.array([300]), np.array([0, 0, -1], np.int32), np.array([200, 129, 40]))
    xd = _inputs(tab, 2, 128, "bf16", 9)
    with bat.Plan(tab.req_prefix, tab.suffix_offsets, tab.prefix_offsets, 2, 128, split_mode=1) as plan:
        assert plan.workspace_bytes == 0
        ref = bat.bat_attention_forward(plan, xd["q"], xd["k_suf"], xd["v_suf"], xd["k_cache"], xd["v_cache"])
        out = bat.bat_attention_forward_noalloc(plan, xd["q"], xd["k_suf"], xd["v_suf"], xd["k_cache"],
                                                xd["v_cache"], out=torch.empty_like(xd["q"]))
        torch.cuda.synchronize()
        mx, mr = _close(out, ref)
        assert mx <= MAX_ABS and mr <= MEAN_REL


def test_noalloc_rejects_plans_beyond_its_scratch():
    # Eight two-tile requests over an 8192-token prefix, every key tile its own chunk:
    # 8 x 2 heads x 66 chunks x 2 query tiles partial slots of 66 KB each, far above 32 MiB.
    tab = RequestTable(np.array([8192]), np.zeros(8, np.int32), np.full(8, 256))
    xd = _inputs(tab, 2, 128, "bf16", 3)
    with bat.Plan(tab.req_prefix, tab.suffix_offsets, tab.prefix_offsets, 2, 128, split_mode=2,
                  split_chunk_tiles=1) as plan:
        assert plan.workspace_bytes > SCRATCH_LIMIT
        out = torch.empty_like(xd["q"])
        st = _bat.lib.bat_attention_forward_noalloc(plan.handle, _ptr(xd["q"]), _ptr(xd["k_suf"]), _ptr(xd["v_suf"]),
                                                    _ptr(xd["k_cache"]), _ptr(xd["v_cache"]), 0.0, bat.BAT_BF16,
                                                    _ptr(out), None, torch.cuda.current_stream().cuda_stream)
        assert st == bat.BAT_ERR_INVALID_ARG
        msg = bat.last_error()
        assert "split scratch" in msg and str(SCRATCH_LIMIT) in msg and str(plan.workspace_bytes) in msg
    assert bat.bat_get_device_status() == bat.BAT_OK
