"""The C ABI: the library loads without a GPU, exports every function include/bat.h declares,
and rejects bad arguments with error codes (no compute calls are made here)."""

import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

import prefix_shared_attention_b200 as bat
from prefix_shared_attention_b200 import _bat

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bat.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bat_[a-z_]+)\s*\(", text)))


def test_header_declarations_are_all_exported():
    names = declared_functions()
    assert "bat_attention_forward" in names and "bat_prefix_kv_build" in names
    out = subprocess.run(["nm", "-D", "--defined-only", bat.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r" T (bat_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    # The binding wraps exactly the declared functions.
    assert sorted(_bat.exported_symbols()) == names


def test_version_and_last_error():
    assert bat.bat_version() >> 16 == 1
    assert isinstance(bat.last_error(), str)


def _tables():
    return np.array([0, -1, 0], np.int32), np.array([0, 5, 9, 200], np.int64), np.array([0, 17], np.int64)


def test_host_only_plan_builds_without_gpu():
    rp, so, po = _tables()
    with bat.Plan(rp, so, po, H=4, d=128, host_only=True, num_sms=148) as p:
        info = p.info()
        assert info.on_device == 0 and info.R == 3 and info.P == 1 and info.T_suf == 200 and info.T_cache == 17
        assert info.n_items > 0


@pytest.mark.parametrize("kw,code", [
    (dict(H=0, d=64), bat.BAT_ERR_INVALID_ARG),
    (dict(H=2, d=32), bat.BAT_ERR_UNSUPPORTED),          # bf16 needs d in {64, 128}
    (dict(H=2, d=96, dtype=bat.BAT_FP32), bat.BAT_ERR_UNSUPPORTED),
    (dict(H=2, d=64, split_mode=7), bat.BAT_ERR_INVALID_ARG),
])
def test_plan_argument_errors(kw, code):
    rp, so, po = _tables()
    with pytest.raises(bat.BatError) as e:
        bat.Plan(rp, so, po, host_only=True, **kw)
    assert e.value.status == code


@pytest.mark.parametrize("mutate,needle", [
    (lambda rp, so, po: (rp, np.array([0, 5, 4, 200]), po), "monotone"),
    (lambda rp, so, po: (np.array([0, 2, 0], np.int32), so, po), "out of range"),
    (lambda rp, so, po: (np.array([0, -2, 0], np.int32), so, po), "out of range"),
    (lambda rp, so, po: (rp, so, np.array([0, -3])), "monotone"),
    (lambda rp, so, po: (rp, np.array([-1, 5, 9, 200]), po), "negative"),
    (lambda rp, so, po: (rp, np.array([0, 5, 9, 2**31]), po), "int32"),
])
def test_plan_rejects_bad_tables(mutate, needle):
    rp, so, po = mutate(*_tables())
    with pytest.raises(bat.BatError) as e:
        bat.Plan(rp, so, po, H=2, d=64, host_only=True)
    assert e.value.status == bat.BAT_ERR_INVALID_ARG
    assert needle in str(e.value)


def test_forward_rejects_host_only_plan_and_null_plan():
    rp, so, po = _tables()
    with bat.Plan(rp, so, po, H=2, d=64, host_only=True) as p:
        st = _bat.lib.bat_attention_forward(p.handle, 16, 16, 16, 16, 16, 0.0, bat.BAT_BF16, 16, None, None, 0, None)
        assert st == bat.BAT_ERR_INVALID_ARG and "host-only" in bat.last_error()
    st = _bat.lib.bat_attention_forward(None, 16, 16, 16, 16, 16, 0.0, 0, 16, None, None, 0, None)
    assert st == bat.BAT_ERR_INVALID_ARG


def test_prefix_kv_build_argument_errors():
    src = np.array([0, 4, 3], np.int64)
    dst = np.array([0, 4], np.int64)
    p = lambda a: a.ctypes.data_as(C.c_void_p)
    st = _bat.lib.bat_prefix_kv_build(16, 16, p(src), 2, p(dst), 2, 64, bat.BAT_BF16, 16, 16, None)
    assert st == bat.BAT_ERR_INVALID_ARG and "monotone" in bat.last_error()
    src = np.array([0, 4], np.int64)
    st = _bat.lib.bat_prefix_kv_build(17, 16, p(src), 1, p(dst), 2, 64, bat.BAT_BF16, 16, 16, None)
    assert st == bat.BAT_ERR_INVALID_ARG and "aligned" in bat.last_error()
    st = _bat.lib.bat_prefix_kv_build(None, 16, p(src), 1, p(dst), 2, 64, bat.BAT_BF16, 16, 16, None)
    assert st == bat.BAT_ERR_INVALID_ARG
    # Nothing to copy is a valid no-op.
    assert _bat.lib.bat_prefix_kv_build(None, None, p(np.array([3, 3], np.int64)), 1, p(dst), 2, 64, 0, None, None,
                                        None) == bat.BAT_OK


def test_wait_timeout_setter():
    bat.bat_set_wait_timeout_ns(5)
    bat.bat_set_wait_timeout_ns(0)   # back to the default


def test_product_path_does_not_import_the_oracle():
    import sys
    pkg_dir = os.path.dirname(bat.__file__)
    for root, _, files in os.walk(pkg_dir):
        for f in files:
            if f.endswith((".py", ".cu", ".cpp", ".h")):
                text = open(os.path.join(root, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f


def test_plain_c_consumer(tmp_path):
    """The ABI from plain C: tests/c_consumer/plan_consumer.c, compiled with gcc against
    include/bat.h and linked to libbat.so, builds host-only plans and checks error codes."""
    import shutil
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc is not installed")
    lib_dir = os.path.dirname(bat.LIB_PATH)
    exe = str(tmp_path / "plan_consumer")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_consumer", "plan_consumer.c"), "-L", lib_dir, "-lbat",
                    f"-Wl,-rpath,{lib_dir}", "-o", exe], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c consumer: ok" in r.stdout
