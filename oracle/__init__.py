"""fp64 CPU oracle for bipartite prefix-shared attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and its ``--impl reference`` arm) may
import, call or execute anything in this package.  The CUDA library and its
Python binding never import it, and the oracle imports nothing from them: the
two share no code.  Inputs for both come from the separate ``workloads``
generator module.

What it computes is the plain definition of each operation, written out with
no blocking, fusion or reordering beyond what the definition states; see
``oracle.attention`` (bipartite prefix-shared attention) and ``oracle.gbla``
(gated bidirectional linear attention) for the definitions and the readings
they rest on.

Parity status: every function here is pinned, by ``tests/test_oracle.py``
(brute force, closed forms, the four invariants, a library routine) and by
``tests/test_gbla_oracle.py`` (element-by-element loops, the linear-time form,
closed forms, invariants, planted mistakes); none is "parity unpinned".
"""

from .attention import (  # noqa: F401
    attend,
    request_keys,
    bipartite_attention,
    bipartite_attention_split,
    merge_partials,
    chunk_partial,
    prefix_side_attention,
)
from . import gbla  # noqa: F401
