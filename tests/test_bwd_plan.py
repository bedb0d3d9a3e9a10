"""Host-side plan of the chunked loss backward (mls_multiexit_loss_bwd_plan).

The backward pass forms the dense logit gradient G' one block of tokens x one
chunk of the vocabulary at a time, in a workspace that does not grow with
T x V.  These checks need no GPU: the plan and the workspace sizes are host
arithmetic in the library.
"""
import pytest
import torch

from lm_head_loss_junction_b200 import _lib, multiexit_loss_bwd_plan, multiexit_loss_workspace
from lm_head_loss_junction_b200 import workloads as wl

BUDGET = 3 << 29          # the 1.5 GiB budget of the workspace query
BF16 = torch.bfloat16


def _plan(cfg, ws):
    return multiexit_loss_bwd_plan(cfg.T, cfg.D, cfg.V, BF16, ws)


@pytest.mark.parametrize("name", ["proxy2", "main3", "main3_aligned", "suite4"])
def test_default_workspace_is_bounded_and_fits_its_plan(name):
    cfg = wl.CONFIGS[name]
    _, bwd = multiexit_loss_workspace(cfg.T, cfg.D, cfg.V, BF16)
    assert bwd <= BUDGET
    Tb, Vc, mn = _plan(cfg, bwd)
    assert 0 < Tb <= cfg.T and 0 < Vc <= cfg.V and mn <= bwd
    # the G' piece alone fits in the workspace
    assert cfg.M * Tb * Vc * 2 <= bwd
    # blocks are whole 128-token tiles, chunks whole 256-column tiles (but for the last ones)
    assert Tb == cfg.T or Tb % 128 == 0
    assert Vc == cfg.V or Vc % 256 == 0


def test_default_workspace_does_not_grow_with_tokens():
    base = wl.CONFIGS["main3"]
    for T in (8192, 32768, 131072, 1 << 20):
        _, bwd = multiexit_loss_workspace(T, base.D, base.V, BF16)
        assert bwd <= BUDGET, (T, bwd)
        Tb, Vc, _ = multiexit_loss_bwd_plan(T, base.D, base.V, BF16, bwd)
        assert 0 < Tb <= T and 0 < Vc <= base.V


def test_main_suite_plan():
    cfg = wl.CONFIGS["main3"]
    _, bwd = multiexit_loss_workspace(cfg.T, cfg.D, cfg.V, BF16)
    # the 8192 tokens in one block (no read-modify-write of dW), the vocabulary in three chunks
    Tb, Vc, _ = _plan(cfg, bwd)
    assert (Tb, Vc) == (8192, 16384)
    # a workspace with room for the whole problem: one piece
    assert _plan(cfg, 4 << 30)[:2] == (cfg.T, cfg.V)
    big = wl.CONFIGS["main3_aligned"]
    _, bwd = multiexit_loss_workspace(big.T, big.D, big.V, BF16)
    Tb, Vc, _ = _plan(big, bwd)
    assert Tb < big.T and Vc < big.V


def test_plan_limits_and_monotonicity():
    cfg = wl.small_variant(wl.CONFIGS["main3"], batch=1, seq=300, V=1024)
    whole = cfg.M * cfg.T * cfg.V * 2
    Tb, Vc, mn = _plan(cfg, whole + (64 << 20))
    assert (Tb, Vc) == (cfg.T, cfg.V)                        # room for everything: one piece
    Tb, Vc, _ = _plan(cfg, mn)                               # the minimum: one token tile per block
    assert Tb == 128 and Vc in (256, cfg.V)
    assert _plan(cfg, mn - 1)[:2] == (0, 0)
    big = wl.CONFIGS["main3"]
    _, _, mn_big = _plan(big, 0)
    assert _plan(big, mn_big)[:2] == (128, 256)               # wide heads: one tile of columns per chunk
    pieces = []
    for ws in sorted((mn, mn * 2, mn * 4, mn + whole // 2, mn + whole, mn + whole * 4, whole + (64 << 20))):
        Tb, Vc, _ = _plan(cfg, ws)
        pieces.append(-(-cfg.T // Tb) * -(-cfg.V // Vc))
    assert all(a >= b for a, b in zip(pieces, pieces[1:])), pieces


def test_fp32_path_has_no_split():
    cfg = wl.CONFIGS["tiny3"]
    _, bwd = multiexit_loss_workspace(cfg.T, cfg.D, cfg.V, torch.float32)
    Tb, Vc, mn = multiexit_loss_bwd_plan(cfg.T, cfg.D, cfg.V, torch.float32, 0)
    assert (Tb, Vc, mn) == (cfg.T, cfg.V, bwd)


def test_backward_rejects_workspace_below_minimum():
    cfg = wl.small_variant(wl.CONFIGS["main3"], batch=1, seq=300, V=1024)
    _, _, mn = _plan(cfg, 0)
    fake = 0x10000
    lib = _lib.lib()
    args = (cfg.M, cfg.T, cfg.V, _lib.i64_array(cfg.D), fake, _lib.ptr_array([fake] * cfg.M),
            _lib.ptr_array([fake] * cfg.M), 0.3, _lib.MLS_BF16, fake, 1.0, _lib.ptr_array([fake] * cfg.M),
            _lib.ptr_array([fake] * cfg.M), 0, fake)
    assert lib.mls_multiexit_loss_bwd(*args, mn - 1, None, None) == 3      # MLS_ERR_WORKSPACE
