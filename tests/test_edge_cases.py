"""Edge shapes through the C ABI: one token, a vocabulary of one half tile,
exits narrower than one N tile (single-CTA GEMM path), four exits with a
ragged vocabulary tile, the smallest junction, and fp32 shapes the tensor-core
path does not take."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from lm_head_loss_junction_b200 import (exit_agreement, junction_bwd, junction_fwd, multiexit_loss_bwd,
                                        multiexit_loss_fwd)
from lm_head_loss_junction_b200 import workloads as wl
from tests.helpers import assert_grad_close, assert_loss_close, assert_stats_close, f64

pytestmark = pytest.mark.gpu


def _run_and_check(cfg, alpha=0.3):
    d = wl.make_inputs(cfg, with_tables=False)
    y = torch.from_numpy(d.y).cuda()
    h = [t.cuda() for t in d.o]
    W = [t.cuda() for t in d.W]
    losses, stats = multiexit_loss_fwd(y, h, W, alpha)
    dh, dW = multiexit_loss_bwd(y, h, W, stats, alpha)
    r = oracle.multiexit_loss(d.y, d.o, d.W, alpha_d=alpha)
    M = cfg.M
    assert_loss_close(losses, np.concatenate([r["ce_lm"], r["ce_kd"], [r["loss"]]]))
    assert_stats_close(f64(stats)[:M], r["lse"], "lse")
    for m in range(M):
        assert_grad_close(dh[m], r["dh"][m], f"dh[{m}]")
        assert_grad_close(dW[m], r["dW"][m], f"dW[{m}]")
    return d, h, W, stats


def _cfg(D, V, T, dtype="bf16", **kw):
    return dataclasses.replace(wl.CONFIGS["main3"], name="edge", D=tuple(D), V=V, batch=1, seq=T, dtype=dtype, **kw)


def test_single_token_and_half_vocab_tile():
    _run_and_check(_cfg((1024, 2304, 4352), V=128, T=1))


def test_widths_narrower_than_one_n_tile():
    _run_and_check(_cfg((64, 128), V=256, T=130))


def test_four_exits_ragged_vocab_tile_and_agreement():
    d, h, W, stats = _run_and_check(_cfg((64, 128, 192, 256), V=384, T=3))
    metrics, rows, top1 = exit_agreement(h, W, stats, per_token=True, want_top1=True)
    r = oracle.exit_agreement(d.o, d.W)
    assert_stats_close(f64(rows)[:3], r["beta"], "beta")


def test_fp32_any_vocabulary_and_width():
    _run_and_check(_cfg((3, 5, 9), V=100, T=17, dtype="f32"))


def test_smallest_junction():
    x = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = torch.randn(1, 8, device="cuda").to(torch.bfloat16)
    E = torch.randn(1, 8, device="cuda").to(torch.bfloat16) * 0.02
    y = junction_fwd(x, o, E)
    ye, _ = oracle.junction_fwd(x.cpu().numpy(), o.cpu(), E.cpu())
    assert torch.equal(y[:, 8:].cpu(), E.cpu())
    np.testing.assert_allclose(f64(y[:, :8]), ye[:, :8], rtol=2 ** -8 + 1e-5)
    dy = torch.randn(1, 16, device="cuda").to(torch.bfloat16)
    dE = torch.zeros(1, 8, dtype=torch.float32, device="cuda")
    do, de, dE = junction_bwd(x, o, E, dy, dE=dE)
    do_e, de_e, dE_e = oracle.junction_bwd(x.cpu().numpy(), o.cpu(), E.cpu(), dy.cpu())
    assert_grad_close(do, do_e, "do")
    assert_grad_close(dE, dE_e, "dE")
