"""fp64 CPU oracle for exact attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never does.
Every function is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle.py``, ``tests/test_oracle_sparse.py`` and
``tests/test_oracle_varlen.py``; no function here is "parity unpinned".
"""
from .attention import (  # noqa: F401
    BLOCK,
    attention_backward_varlen,
    attention_forward_varlen,
    attention_backward,
    attention_backward_dq_rows,
    attention_backward_kv_rows,
    attention_forward,
    attention_forward_rows,
    kv_head,
    scores,
)
