"""The debug build, libbat_debug.so (-DBAT_DEBUG): the same kernels, with every tensor-map
coordinate and store index checked against the tensors' bounds before use.  A failed check
is recorded in the device status word (bat_get_device_status -> BAT_ERR_DEVICE_CHECK) and the
access is skipped or clamped into the tensor; nothing traps.  With a memory checker closed on
the GPU pool, this build and the guard rows of the parity tests stand in for it.

The small parity cases run in a subprocess that selects the debug library through
BAT_LIBRARY: every run must report BAT_OK (no check failed) and meet the parity bar.  The
negative control makes the checks treat the tensors as one row shorter than they are (the
accesses themselves stay inside the real tensors) and expects the failure to be reported.
"""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SMALL_CASES = ("tiny_config or bf16_ragged or fp32_ragged or forced_split or edge_lengths or short_key_tiles "
               "or explicit_scale or rescale_path or role_swap or nan_neighbour or prefix_side")


def debug_env(**extra):
    from prefix_shared_attention_b200 import build
    lib = build.build(debug=True)
    env = dict(os.environ, BAT_LIBRARY=lib)
    env.update(extra)
    return env


def run_py(code, env):
    return subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=600)


def test_debug_library_is_the_checked_build():
    p = run_py("import prefix_shared_attention_b200 as b; print(b.LIB_PATH, b.bat_debug_checks())", debug_env())
    assert p.returncode == 0, p.stderr[-2000:]
    path, flag = p.stdout.split()
    assert path.endswith("libbat_debug.so") and flag == "True"


def test_small_parity_cases_pass_every_device_check():
    p = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_gpu_parity.py"), "-q", "-x",
                        "-m", "gpu", "-k", SMALL_CASES, "-p", "no:cacheprovider"],
                       cwd=ROOT, env=debug_env(), capture_output=True, text=True, timeout=1800)
    assert p.returncode == 0, p.stdout[-4000:] + p.stderr[-2000:]
    assert " passed" in p.stdout and " failed" not in p.stdout


NEGATIVE = r"""
import numpy as np, torch
import prefix_shared_attention_b200 as bat
from workloads import RequestTable, host_tensors
assert bat.bat_debug_checks()
tab = RequestTable(np.array([300, 77]), np.array([0, 0, 1, -1], np.int32), np.array([200, 129, 64, 33]))
for dt, d in (("bf16", 128), ("bf16", 64), ("fp32", 64)):
    x = {k: v.cuda() for k, v in host_tensors(tab, 2, d, dt, 5).items()}
    code = bat.BAT_BF16 if dt == "bf16" else bat.BAT_FP32
    with bat.Plan(tab.req_prefix, tab.suffix_offsets, tab.prefix_offsets, 2, d, code) as plan:
        out = torch.zeros_like(x["q"])
        bat.bat_attention_forward(plan, x["q"], x["k_suf"], x["v_suf"], x["k_cache"], x["v_cache"], out=out)
        st = bat.bat_get_device_status()
        msg = bat.last_error()   # read before the plan's release clears this thread's message
    print(dt, d, st, msg)
    assert st == bat.BAT_ERR_DEVICE_CHECK, (dt, d, st)
    assert "bounds check failed" in msg
    assert bat.bat_get_device_status() == bat.BAT_OK   # reported once, then cleared
print("negative control ok")
"""


def test_checks_fire_when_the_bounds_are_shrunk():
    p = run_py(NEGATIVE, debug_env(BAT_DEBUG_SHRINK_BOUNDS="1"))
    assert p.returncode == 0, p.stdout[-3000:] + p.stderr[-2000:]
    assert "negative control ok" in p.stdout
