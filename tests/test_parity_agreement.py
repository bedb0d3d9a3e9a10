"""GPU inter-exit agreement (acceptance beta, KL(p_M || q_m), top-1 agreement)
against the fp64 oracle, through the C ABI.

The argmax is decided in fp32 on the GPU and fp64 in the oracle; where the
oracle's two largest logits are closer than the fp32 error of a logit, either
index is a valid answer, so those tokens are checked for validity instead of
identity, and the agreement mean may differ by their share.
"""
import numpy as np
import pytest
import torch

import oracle
from lm_head_loss_junction_b200 import exit_agreement, multiexit_loss_fwd
from lm_head_loss_junction_b200 import workloads as wl
from tests.helpers import assert_stats_close, f64

pytestmark = pytest.mark.gpu


def _logits(d, rows):
    return [f64(d.o[m][torch.from_numpy(rows)]) @ f64(d.W[m]).T for m in range(d.cfg.M)]


def _check(d, rows=None):
    cfg = d.cfg
    M = cfg.M
    y = torch.from_numpy(d.y).cuda()
    h = [t.cuda() for t in d.o]
    W = [t.cuda() for t in d.W]
    _, stats = multiexit_loss_fwd(y, h, W, cfg.alpha_d)
    metrics, per_tok, top1 = exit_agreement(h, W, stats, per_token=True, want_top1=True)
    pt = f64(per_tok)
    # the reported means are the token means of the per-token rows
    np.testing.assert_allclose(f64(metrics), pt.mean(axis=1), rtol=2e-6, atol=1e-7)
    sel = np.arange(cfg.T) if rows is None else rows
    r = oracle.exit_agreement(d.o, d.W, rows=sel)
    S = M - 1
    assert_stats_close(pt[:S, sel], r["beta"], "beta")
    assert_stats_close(pt[S:2 * S, sel], r["kl"], "KL")
    # top-1: identical where the decision is clear, a near-maximum otherwise
    logits = _logits(d, sel)
    got = top1.cpu().numpy()[:, sel]
    ties = np.zeros(len(sel), dtype=bool)
    for m in range(M):
        l = logits[m]
        srt = np.sort(l, axis=1)
        tol = 1e-3 + 1e-4 * np.abs(srt[:, -1])
        near = (srt[:, -1] - srt[:, -2]) <= tol
        ties |= near
        clear = ~near
        assert np.array_equal(got[m][clear], r["top1"][m][clear]), f"exit {m}: top-1 differs on a clear maximum"
        chosen = l[np.arange(len(sel)), got[m]]
        assert np.all(srt[:, -1] - chosen <= tol), f"exit {m}: top-1 is not a maximum"
    for s in range(S):
        agree_gpu = pt[2 * S + s, sel]
        assert np.all(agree_gpu[~ties] == r["agree"][s][~ties])
    if rows is None:
        np.testing.assert_allclose(f64(metrics)[:S], r["beta_mean"], rtol=2e-3)
        np.testing.assert_allclose(f64(metrics)[S:2 * S], r["kl_mean"], rtol=2e-3, atol=2e-3 * np.max(r["kl_mean"]))
        assert np.all(np.abs(f64(metrics)[2 * S:] - r["agree_mean"]) <= ties.mean() + 1e-6)


def test_agreement_tiny_fp32():
    _check(wl.make_inputs(wl.CONFIGS["tiny3"], with_tables=False))


@pytest.mark.parametrize("name,small", [("main3", dict(batch=1, seq=300, V=1024)),
                                        ("suite4", dict(batch=1, seq=200, V=640)),
                                        ("main3_aligned", dict(batch=1, seq=256, V=768))])
def test_agreement_bf16_small(name, small):
    _check(wl.make_inputs(wl.small_variant(wl.CONFIGS[name], **small), with_tables=False))


# Vocabulary sizes whose split counts give the agreement merge's thread rows
# (16 per 32-token block, four splits loaded per batch) a full batch and a
# partial one (V = 10240: 80 splits, 5 per row) or exact batches (V = 24576:
# 192 splits, 12 per row).
@pytest.mark.parametrize("V", [10240, 24576])
def test_agreement_merge_split_batches(V):
    _check(wl.make_inputs(wl.small_variant(wl.CONFIGS["main3"], batch=1, seq=130, V=V), with_tables=False))


@pytest.mark.parametrize("name", ["main3", "main3_aligned"])
def test_agreement_full_size_sampled(name):
    d = wl.make_inputs(wl.CONFIGS[name], with_tables=False)
    rows = np.sort(np.random.default_rng(9).choice(d.cfg.T, size=64, replace=False))
    _check(d, rows)
