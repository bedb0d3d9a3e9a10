"""Matryoshka LM-suite junction and multi-exit LM-head loss on B200 (sm_100a).

The compute lives in the CUDA library ``libmls.so`` (C ABI in include/mls.h);
this package is a thin binding.  Importing the package does not load the
library; the first call does, and fails loudly if it is not built.
"""
from .api import (exit_agreement, junction_bwd, junction_bwd_multi, junction_bwd_multi_workspace,  # noqa: F401
                  junction_bwd_workspace, junction_fwd, junction_fwd_multi,
                  multiexit_loss_bwd, multiexit_loss_bwd_plan,
                  multiexit_loss_fwd, multiexit_loss_workspace, new_status, status_read)
