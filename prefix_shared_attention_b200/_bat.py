"""ctypes binding of libbat.so: argument marshalling only.

Every entry point of ``include/bat.h`` is exposed under the same name.  The helpers below
turn numpy tables and torch device tensors into the pointers and sizes the C ABI takes;
no step of the attention is computed here.  Importing this module fails loudly when the
library has not been built: there is no fallback implementation.
"""

from __future__ import annotations

import ctypes as C
import os
from typing import Optional

import numpy as np

# The library this process uses: the in-tree libbat.so, or the file BAT_LIBRARY names (the
# debug build, libbat_debug.so, whose kernels check their bounds).
LIB_PATH = os.environ.get("BAT_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbat.so")

(BAT_OK, BAT_ERR_INVALID_ARG, BAT_ERR_UNSUPPORTED, BAT_ERR_CUDA, BAT_ERR_TIMEOUT, BAT_ERR_OOM,
 BAT_ERR_DEVICE_CHECK) = range(7)
STATUS_NAMES = {0: "BAT_OK", 1: "BAT_ERR_INVALID_ARG", 2: "BAT_ERR_UNSUPPORTED", 3: "BAT_ERR_CUDA",
                4: "BAT_ERR_TIMEOUT", 5: "BAT_ERR_OOM", 6: "BAT_ERR_DEVICE_CHECK"}
BAT_BF16, BAT_FP32 = 0, 1


class BatError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class PlanOptions(C.Structure):
    _fields_ = [("split_mode", C.c_int32), ("split_chunk_tiles", C.c_int32), ("num_sms", C.c_int32),
                ("host_only", C.c_int32), ("reserved", C.c_int32 * 4)]


class PlanInfo(C.Structure):
    _fields_ = [("n_items", C.c_int64), ("n_merges", C.c_int64), ("n_slots", C.c_int64),
                ("workspace_bytes", C.c_int64), ("total_cost", C.c_int64), ("T_suf", C.c_int64),
                ("T_cache", C.c_int64), ("R", C.c_int32), ("P", C.c_int32), ("H", C.c_int32),
                ("d", C.c_int32), ("dtype", C.c_int32), ("on_device", C.c_int32)]


# Layout of one work item / merge job record (see the library's internal header).
WORK_ITEM_DTYPE = np.dtype([(n, np.int32) for n in (
    "head", "n_q", "shared", "split_slot", "pre_row0", "pre_len",
    "qA_row0", "qA_rows", "sA_row0", "sA_len", "qB_row0", "qB_rows", "sB_row0", "sB_len",
    "cost", "group")])
MERGE_JOB_DTYPE = np.dtype([(n, np.int32) for n in (
    "q_row0", "q_rows", "head", "slot0", "n_chunks", "slot_stride", "pad0", "pad1")])

_vp, _i32, _i64, _f32, _sz, _u64 = C.c_void_p, C.c_int32, C.c_int64, C.c_float, C.c_size_t, C.c_uint64
_SIGNATURES = {
    "bat_prefix_kv_build": (_i32, [_vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _vp, _vp, _vp]),
    "bat_plan_create": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, C.POINTER(PlanOptions), _vp,
                               C.POINTER(_vp)]),
    "bat_plan_create_prefix_side": (_i32, [_vp, _i32, _i32, _i32, _i32, C.POINTER(PlanOptions), _vp, C.POINTER(_vp)]),
    "bat_plan_destroy": (_i32, [_vp]),
    "bat_plan_info": (_i32, [_vp, C.POINTER(PlanInfo)]),
    "bat_workspace_bytes": (_sz, [_vp]),
    "bat_plan_items": (_i32, [_vp, _vp, _sz]),
    "bat_plan_merges": (_i32, [_vp, _vp, _sz]),
    "bat_attention_forward": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _f32, _i32, _vp, _vp, _vp, _sz, _vp]),
    "bat_attention_forward_noalloc": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _f32, _i32, _vp, _vp, _vp]),
    "bat_get_device_status": (_i32, [_vp]),
    "bat_set_wait_timeout_ns": (_i32, [_u64]),
    "bat_last_error": (C.c_char_p, []),
    "bat_version": (_i32, []),
    "bat_debug_checks": (_i32, []),
    "bat_gbla_plan_create": (_i32, [_vp, _i32, _i32, _i32, _i32, _i32, _vp, C.POINTER(_vp)]),
    "bat_gbla_plan_destroy": (_i32, [_vp]),
    "bat_gbla_workspace_bytes": (_sz, [_vp]),
    "bat_gbla_plan_chunks": (_i32, [_vp, _vp, _sz, C.POINTER(_i64)]),
    "bat_gbla_forward": (_i32, [_vp] + [_vp] * 10 + [_vp, _sz, _vp]),
}


def _load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m prefix_shared_attention_b200.build`"
                          " (there is no fallback implementation)")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def exported_symbols():
    return sorted(_SIGNATURES)


def last_error() -> str:
    return lib.bat_last_error().decode()


def check(status: int) -> None:
    if status != BAT_OK:
        raise BatError(status, last_error())


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p) if a.size else None


def dtype_code(torch_dtype) -> int:
    import torch
    if torch_dtype == torch.bfloat16:
        return BAT_BF16
    if torch_dtype == torch.float32:
        return BAT_FP32
    raise BatError(BAT_ERR_UNSUPPORTED, f"dtype {torch_dtype} (bf16 or fp32 only)")


class Plan:
    """Owns a ``bat_plan``: the work list of one batch (host grouping pass)."""

    def __init__(self, req_prefix, suffix_offsets, prefix_offsets, H: int, d: int, dtype: int = BAT_BF16,
                 split_mode: int = 0, split_chunk_tiles: int = 0, num_sms: int = 0, host_only: bool = False,
                 stream=None):
        self._rp = np.ascontiguousarray(req_prefix, dtype=np.int32)
        self._so = np.ascontiguousarray(suffix_offsets, dtype=np.int64)
        self._po = np.ascontiguousarray(prefix_offsets, dtype=np.int64)
        R = int(self._rp.shape[0])
        P = int(self._po.shape[0]) - 1 if self._po.size else 0
        if self._so.shape[0] != R + 1:
            raise BatError(BAT_ERR_INVALID_ARG, f"suffix_offsets has {self._so.shape[0]} entries, need R+1={R + 1}")
        opts = PlanOptions(split_mode, split_chunk_tiles, num_sms, 1 if host_only else 0)
        h = C.c_void_p()
        st = None if host_only else _stream_handle(stream)
        check(lib.bat_plan_create(_ptr(self._rp), _ptr(self._so), _ptr(self._po) if P >= 0 and self._po.size else None,
                                  R, max(P, 0), H, d, dtype, C.byref(opts), st, C.byref(h)))
        self.handle = h
        self.H, self.d, self.dtype = H, d, dtype

    @classmethod
    def prefix_side(cls, src_offsets, H: int, d: int, dtype: int = BAT_BF16, split_mode: int = 0,
                    split_chunk_tiles: int = 0, num_sms: int = 0, host_only: bool = False, stream=None) -> "Plan":
        """Plan of the prefix-side step: prefix i's tokens (rows ``src_offsets[i] ..
        src_offsets[i+1]`` of the q/k/v given to the forward as q, k_suf, v_suf) attend over
        that prefix's tokens only (no cached prefix)."""
        self = cls.__new__(cls)
        so = np.ascontiguousarray(src_offsets, dtype=np.int64)
        n = int(so.shape[0]) - 1
        if n < 0:
            raise BatError(BAT_ERR_INVALID_ARG, "src_offsets needs at least one entry")
        self._rp = np.full(n, -1, dtype=np.int32)
        self._so = so
        self._po = np.zeros(1, dtype=np.int64)
        opts = PlanOptions(split_mode, split_chunk_tiles, num_sms, 1 if host_only else 0)
        h = C.c_void_p()
        st = None if host_only else _stream_handle(stream)
        check(lib.bat_plan_create_prefix_side(_ptr(so), n, H, d, dtype, C.byref(opts), st, C.byref(h)))
        self.handle = h
        self.H, self.d, self.dtype = H, d, dtype
        return self

    def info(self) -> PlanInfo:
        i = PlanInfo()
        check(lib.bat_plan_info(self.handle, C.byref(i)))
        return i

    @property
    def workspace_bytes(self) -> int:
        return int(lib.bat_workspace_bytes(self.handle))

    def items(self) -> np.ndarray:
        n = self.info().n_items
        out = np.zeros(n, dtype=WORK_ITEM_DTYPE)
        check(lib.bat_plan_items(self.handle, _ptr(out), out.nbytes))
        return out

    def merges(self) -> np.ndarray:
        n = self.info().n_merges
        out = np.zeros(n, dtype=MERGE_JOB_DTYPE)
        check(lib.bat_plan_merges(self.handle, _ptr(out), out.nbytes))
        return out

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            check(lib.bat_plan_destroy(self.handle))
        self.handle = C.c_void_p()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


GBLA_CHUNK_DTYPE = np.dtype([(n, np.int32) for n in ("pair", "head", "seq_lo", "seq_hi", "tile0", "n_tiles",
                                                      "pad0", "pad1")])


class GblaPlan:
    """Owns a ``bat_gbla_plan``: the chunk list of one batch of sequences for the GBLA layer."""

    def __init__(self, seq_offsets, H: int, d: int = 128, num_sms: int = 0, host_only: bool = False, stream=None):
        self._so = np.ascontiguousarray(seq_offsets, dtype=np.int64)
        n = int(self._so.shape[0]) - 1
        if n < 0:
            raise BatError(BAT_ERR_INVALID_ARG, "seq_offsets needs at least one entry")
        h = C.c_void_p()
        st = None if host_only else _stream_handle(stream)
        check(lib.bat_gbla_plan_create(_ptr(self._so), n, H, d, num_sms, 1 if host_only else 0, st, C.byref(h)))
        self.handle = h
        self.H, self.d = H, d

    @property
    def workspace_bytes(self) -> int:
        return int(lib.bat_gbla_workspace_bytes(self.handle))

    def chunks(self) -> np.ndarray:
        n = C.c_int64()
        check(lib.bat_gbla_plan_chunks(self.handle, None, 0, C.byref(n)))
        out = np.zeros(n.value, dtype=GBLA_CHUNK_DTYPE)
        check(lib.bat_gbla_plan_chunks(self.handle, _ptr(out), out.nbytes, C.byref(n)))
        return out

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            check(lib.bat_gbla_plan_destroy(self.handle))
        self.handle = C.c_void_p()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def bat_gbla_forward(plan: GblaPlan, q, k, v, a, z, conv_q, conv_k, conv_v, norm_weight, y=None, workspace=None,
                     stream=None):
    """GBLA layer on torch device tensors (q, k, v, z bf16 [T, H, 128]; a bf16 [T, H]; conv_* fp32
    [H, 4, 128]; norm_weight fp32 [H, 128]); allocates ``y`` and the workspace when not given.
    Returns ``y``."""
    import torch
    if y is None:
        y = torch.empty_like(q)
    need = plan.workspace_bytes
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    ptrs = [t.data_ptr() for t in (q, k, v, a, z, conv_q, conv_k, conv_v, norm_weight, y)]
    check(lib.bat_gbla_forward(plan.handle, *ptrs, workspace.data_ptr(), int(workspace.numel()),
                               _stream_handle(stream)))
    return y


def bat_prefix_kv_build(k_src, v_src, src_offsets, dst_offsets, k_cache, v_cache, stream=None) -> None:
    """Pack prefixes' K/V rows into the cache pool (torch device tensors [T, H, d])."""
    so = np.ascontiguousarray(src_offsets, dtype=np.int64)
    do = np.ascontiguousarray(dst_offsets, dtype=np.int64)
    n = int(so.shape[0]) - 1
    H, d = int(k_src.shape[1]), int(k_src.shape[2])
    check(lib.bat_prefix_kv_build(k_src.data_ptr(), v_src.data_ptr(), _ptr(so), n, _ptr(do), H, d,
                                  dtype_code(k_src.dtype), k_cache.data_ptr(), v_cache.data_ptr(),
                                  _stream_handle(stream)))


def prefix_build(q_src, k_src, v_src, src_offsets, dst_offsets, k_cache, v_cache, out=None, lse=None,
                 scale: float = 0.0, stream=None):
    """Prefix-side step for newly cached prefixes: pack their K/V into the pool
    (bat_prefix_kv_build) and compute the prefix tokens' own outputs (a prefix-side plan and
    bat_attention_forward).  Tensors are torch device tensors [T, H, d]; returns ``out``
    (rows of q_src)."""
    bat_prefix_kv_build(k_src, v_src, src_offsets, dst_offsets, k_cache, v_cache, stream=stream)
    H, d = int(q_src.shape[1]), int(q_src.shape[2])
    with Plan.prefix_side(src_offsets, H, d, dtype_code(q_src.dtype), stream=stream) as plan:
        out = bat_attention_forward(plan, q_src, k_src, v_src, out=out, lse=lse, scale=scale, stream=stream)
    return out


def bat_attention_forward(plan: Plan, q, k_suf, v_suf, k_cache=None, v_cache=None, out=None, lse=None,
                          scale: float = 0.0, workspace=None, stream=None):
    """Run the forward on torch device tensors; allocates ``out`` (and the workspace) when
    not given.  Returns ``out``."""
    import torch
    if out is None:
        out = torch.empty_like(q)
    need = plan.workspace_bytes
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ptr = lambda t: t.data_ptr() if t is not None else None
    check(lib.bat_attention_forward(plan.handle, ptr(q), ptr(k_suf), ptr(v_suf), ptr(k_cache), ptr(v_cache),
                                    float(scale), dtype_code(q.dtype), ptr(out), ptr(lse), ptr(workspace),
                                    int(workspace.numel()) if workspace is not None else 0,
                                    _stream_handle(stream)))
    return out


def bat_attention_forward_noalloc(plan: Plan, q, k_suf, v_suf, k_cache=None, v_cache=None, out=None, lse=None,
                                  scale: float = 0.0, stream=None):
    """The forward without a workspace argument: split scratch comes from a fixed array inside
    the library (for callers that cannot allocate device memory).  ``out`` must be given by
    callers that cannot allocate; when omitted it is allocated here for convenience."""
    import torch
    if out is None:
        out = torch.empty_like(q)
    ptr = lambda t: t.data_ptr() if t is not None else None
    check(lib.bat_attention_forward_noalloc(plan.handle, ptr(q), ptr(k_suf), ptr(v_suf), ptr(k_cache), ptr(v_cache),
                                            float(scale), dtype_code(q.dtype), ptr(out), ptr(lse),
                                            _stream_handle(stream)))
    return out


def bat_get_device_status(stream=None) -> int:
    """Synchronises the stream; returns the status code (BAT_OK or BAT_ERR_TIMEOUT, ...)."""
    return int(lib.bat_get_device_status(_stream_handle(stream)))


def bat_set_wait_timeout_ns(ns: int) -> None:
    check(lib.bat_set_wait_timeout_ns(int(ns)))


def bat_version() -> int:
    return int(lib.bat_version())


def bat_debug_checks() -> bool:
    return bool(lib.bat_debug_checks())
