"""Plain fp64 CPU oracle for the Matryoshka suite junction and multi-exit head loss.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import or call anything in this package.
The library path never routes through it and shares no code with it: the
oracle restates the definitions in numpy fp64 (one library matmul per logit
block, no fusion, no chunked online statistics), while the CUDA kernels are
written independently.

Every function is pinned by the ``-m "not gpu"`` tests in ``tests/`` against
closed forms, invariants, brute-force enumeration and finite differences.
Parity is pinned for every function here; nothing in this package is
"parity unpinned".
"""
from .junction import junction_fwd, junction_bwd, JUNCTION_EPS
from . import junction as junction_variants
from .loss import (exit_agreement, logsumexp_rows, multiexit_loss, multiexit_loss_vocab_rows,
                   softmax_rows)

__all__ = ["junction_fwd", "junction_bwd", "JUNCTION_EPS", "multiexit_loss", "multiexit_loss_vocab_rows",
           "softmax_rows", "logsumexp_rows", "exit_agreement"]
