"""Bipartite prefix-shared attention on B200 (sm_100a).

Python surface of ``libbat.so`` (C ABI in ``include/bat.h``).  The library computes, for
every request, non-causal softmax attention of its suffix tokens over [its cached prefix
K/V ; its own suffix K/V] (Bat: Efficient Generative Recommender Serving with Bipartite
Attention, sections "This paper's idea" and "Why it works").  PyTorch only provides device
memory and streams.
"""

from ._bat import (  # noqa: F401
    BAT_BF16,
    BAT_FP32,
    BAT_OK,
    BAT_ERR_CUDA,
    BAT_ERR_INVALID_ARG,
    BAT_ERR_OOM,
    BAT_ERR_TIMEOUT,
    BAT_ERR_UNSUPPORTED,
    LIB_PATH,
    MERGE_JOB_DTYPE,
    WORK_ITEM_DTYPE,
    BatError,
    Plan,
    bat_attention_forward,
    bat_attention_forward_noalloc,
    bat_get_device_status,
    bat_prefix_kv_build,
    bat_set_wait_timeout_ns,
    bat_version,
    exported_symbols,
    last_error,
    prefix_build,
)
from .metrics import algorithmic_bytes, algorithmic_flops  # noqa: F401
