"""Per-phase clock breakdown of the attention kernel's warps (a profiling aid).

The library built with ``-DBAT_PHASE`` (``python -m prefix_shared_attention_b200.build
--phase`` writes ``libbat_phase.so``) has every warp of ``bat_attn_tc_kernel`` add up, per
phase of its loop, the SM clocks spent there, and write the totals once when it returns.  This
module loads that library (before the binding is imported), runs one launch of a named
workload three times and prints, per key-tile step of query tile A (one visit of tile A to a
key tile, averaged over the CTAs), the clocks of each phase of the softmax warps and of the
MMA issuer warps, as a Markdown table.

    python -m prefix_shared_attention_b200.build --phase
    python -m prefix_shared_attention_b200.phase_profile item-as-prefix [long-user-history ...]

For ``mixed`` the first of its eight launches is run.
"""

from __future__ import annotations

import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
os.environ["BAT_LIBRARY"] = os.path.join(HERE, "libbat_phase.so")

import ctypes as C  # noqa: E402

import numpy as np  # noqa: E402

WARPS, CODES = 12, 20

# Phase codes of the softmax warps (the clocks since the previous event are added to the code
# of the event that ends them).  With P in two halves (d = 64) "exponentials, first half" also
# covers the first half's P stores and the second half's exponentials, and the P-buffer wait
# counts both halves.
SOFTMAX_PHASES = [
    (15, "next work item (queue wait)"), (16, "item read"), (1, "S wait"), (7, "S: TMEM load"),
    (8, "mask, row max, rescale"), (12, "exponentials, first half"), (11, "P-buffer wait"),
    (2, "P stores, second half, fence"), (5, "to the epilogue"), (13, "epilogue: last PV wait"),
    (14, "epilogue: O out"),
]
ISSUER_PHASES = [
    (6, "to the item's first tile"), (4, "K tile wait"), (7, "Q wait"), (2, "S-free wait + S issue"),
    (3, "V tile wait (+ tail zeroing)"), (1, "P wait + PV issue"),
]


def run(name: str):
    import torch
    from workloads import CONFIGS, device_tensors, make_table, split_launches
    from . import _bat as B
    lib = B.lib
    if not hasattr(lib, "bat_debug_set_phase"):
        raise RuntimeError("libbat_phase.so is not the phase build (python -m prefix_shared_attention_b200.build --phase)")
    lib.bat_debug_set_phase.argtypes = [C.c_void_p]
    lib.bat_debug_set_phase.restype = C.c_int
    spec = CONFIGS[name]
    tab = make_table(name)
    if name == "mixed":
        tab = split_launches(tab, 8)[0]
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    buf = torch.zeros(n_sm * WARPS * CODES, dtype=torch.int32, device="cuda")
    if lib.bat_debug_set_phase(C.c_void_p(buf.data_ptr())) != 0:
        raise RuntimeError("bat_debug_set_phase failed")
    x = device_tensors(tab, spec.H, spec.d, spec.dtype, spec.seed)
    with B.Plan(tab.req_prefix, tab.suffix_offsets, tab.prefix_offsets, spec.H, spec.d, B.BAT_BF16) as plan:
        for _ in range(3):
            B.bat_attention_forward(plan, x["q"], x["k_suf"], x["v_suf"], x["k_cache"], x["v_cache"])
        torch.cuda.synchronize()
        items = plan.items()
        if B.bat_get_device_status() != B.BAT_OK:
            raise RuntimeError(B.last_error())
    lib.bat_debug_set_phase(C.c_void_p(0))
    ph = buf.cpu().numpy().view(np.uint32).reshape(n_sm, WARPS, CODES).astype(np.float64)
    tiles = lambda a: -(-a.astype(np.int64) // 128)
    steps = float((tiles(items["pre_len"]) + tiles(items["sA_len"])).sum()) / n_sm
    return spec, len(items), steps, ph


def report(name: str) -> str:
    spec, n_items, steps, ph = run(name)
    soft = ph[:, 0:8, :].mean(axis=(0, 1)) / steps
    iss = ph[:, 9:11, :].mean(axis=(0, 1)) / steps
    out = [f"### {name} (H={spec.H}, d={spec.d}): {n_items} work items, {steps:.1f} key-tile steps of "
           f"query tile A per CTA", "",
           "| softmax warps: phase | clk / step | share |", "|---|---|---|"]
    tot = soft.sum()
    out += [f"| {nm} | {soft[k]:.0f} | {100 * soft[k] / tot:.1f} % |" for k, nm in SOFTMAX_PHASES]
    out += [f"| **total** | **{tot:.0f}** | |", "", "| MMA issuer warps: phase | clk / step |", "|---|---|"]
    out += [f"| {nm} | {iss[k]:.0f} |" for k, nm in ISSUER_PHASES]
    out += [f"| **total** | **{iss.sum():.0f}** |", ""]
    return "\n".join(out)


def main(argv=None):
    names = (argv if argv is not None else sys.argv[1:]) or ["item-as-prefix"]
    for n in names:
        print(report(n), flush=True)


if __name__ == "__main__":
    main()
