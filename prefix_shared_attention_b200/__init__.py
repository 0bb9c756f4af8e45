"""Bipartite prefix-shared attention on B200 (sm_100a).

Python surface of ``libbat.so`` (C ABI in ``include/bat.h``).  The library computes, for
every request, non-causal softmax attention of its suffix tokens over [its cached prefix
K/V ; its own suffix K/V] (Bat: Efficient Generative Recommender Serving with Bipartite
Attention, sections "This paper's idea" and "Why it works").  PyTorch only provides device
memory and streams.

The library is loaded on first use of a name that needs it (``Plan``,
``bat_attention_forward``, ...), not at import: the host-side modules (``metrics``,
``sharding``, ``prefix_choice``) run without it.  Using a library name when ``libbat.so``
is missing raises ImportError; there is no fallback implementation.
"""

from .metrics import algorithmic_bytes, algorithmic_flops  # noqa: F401

_BINDING_NAMES = (
    "BAT_BF16", "BAT_FP32", "BAT_OK", "BAT_ERR_CUDA", "BAT_ERR_INVALID_ARG", "BAT_ERR_OOM", "BAT_ERR_TIMEOUT",
    "BAT_ERR_UNSUPPORTED", "LIB_PATH", "MERGE_JOB_DTYPE", "WORK_ITEM_DTYPE", "BatError", "Plan",
    "bat_attention_forward", "bat_attention_forward_noalloc", "bat_get_device_status", "bat_prefix_kv_build",
    "bat_set_wait_timeout_ns", "bat_version", "bat_debug_checks", "BAT_ERR_DEVICE_CHECK", "exported_symbols", "last_error", "prefix_build",
    "GblaPlan", "GBLA_CHUNK_DTYPE", "bat_gbla_forward",
)

__all__ = list(_BINDING_NAMES) + ["algorithmic_bytes", "algorithmic_flops"]


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import _bat   # loads libbat.so (raises ImportError when it is missing)
        return getattr(_bat, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")


def __dir__():
    return sorted(set(globals()) | set(_BINDING_NAMES))
