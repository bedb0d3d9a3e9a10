"""GPU multi-exit loss (forward and backward) against the fp64 oracle.

Small cases compare every output element; they span several 128x128 tiles
with ragged token tails.  All calls go through the C ABI (libmls).
"""
import numpy as np
import pytest
import torch

import oracle
from lm_head_loss_junction_b200 import (multiexit_loss_bwd, multiexit_loss_bwd_plan, multiexit_loss_fwd, new_status,
                                        status_read)
from lm_head_loss_junction_b200 import workloads as wl
from tests.helpers import acceptance_tie_mass, assert_grad_close, assert_loss_close, assert_stats_close, f64

pytestmark = pytest.mark.gpu


def _gpu_inputs(d):
    y = torch.from_numpy(d.y).cuda()
    h = [t.cuda() for t in d.o]
    W = [t.cuda() for t in d.W]
    return y, h, W


def _oracle(d, alpha, grad_scale=1.0, rows=None, need_grad=True, exit_weights=None, distill="ce",
            teacher_grad=False):
    return oracle.multiexit_loss(d.y, d.o, d.W, alpha_d=alpha, grad_scale=grad_scale, rows=rows,
                                 need_grad=need_grad, exit_weights=exit_weights, distill=distill,
                                 teacher_grad=teacher_grad)


def _losses_expected(r, M):
    return np.concatenate([r["ce_lm"], r["ce_kd"], [r["loss"]]])


def _check_all(d, alpha, grad_scale=1.0, exit_weights=None, distill="ce", teacher_grad=False, bwd_ws_bytes=None):
    """Every output against the oracle.  bwd_ws_bytes: the backward call's workspace
    size (None: the size the workspace query returns), which sets how the call
    splits its work into token blocks and vocabulary chunks."""
    cfg = d.cfg
    M = cfg.M
    y, h, W = _gpu_inputs(d)
    st = new_status()
    losses, stats = multiexit_loss_fwd(y, h, W, alpha, status=st, exit_weights=exit_weights, distill=distill,
                                       teacher_grad=teacher_grad)
    ws = None if bwd_ws_bytes is None else torch.empty(bwd_ws_bytes, dtype=torch.uint8, device="cuda")
    dh, dW = multiexit_loss_bwd(y, h, W, stats, alpha, grad_scale, status=st, exit_weights=exit_weights,
                                distill=distill, teacher_grad=teacher_grad, workspace=ws)
    assert status_read(st) == (0, 0)
    r = _oracle(d, alpha, grad_scale, exit_weights=exit_weights, distill=distill, teacher_grad=teacher_grad)
    assert_loss_close(losses, _losses_expected(r, M), "losses")
    s = f64(stats)
    assert_stats_close(s[:M], r["lse"], "lse")
    assert_stats_close(s[M:2 * M], r["tgt"], "target logits")
    if M > 1:
        slack = acceptance_tie_mass(d.y, d.o, d.W) if distill == "accept" else None
        assert_stats_close(s[2 * M:3 * M - 1],
                           {"ce": r["S"], "reverse_kl": r["R"], "js": r["J"], "accept": r["A"]}[distill],
                           "distillation statistic", slack=slack)
        if distill in ("js", "accept") and teacher_grad:
            assert_stats_close(s[3 * M - 1:], {"js": r["Jp"], "accept": r["B"]}[distill],
                               "teacher-side distillation statistic", slack=slack)
    for m in range(M):
        assert_grad_close(dh[m], r["dh"][m], f"dh[{m}]")
        assert_grad_close(dW[m], r["dW"][m], f"dW[{m}]")


def test_tiny_fp32_suite_full():
    d = wl.make_inputs(wl.CONFIGS["tiny3"])
    _check_all(d, 0.3)


SMALL_BF16 = [
    ("main3", dict(batch=1, seq=300, V=1024)),
    ("proxy2", dict(batch=2, seq=97, V=2048)),
    ("suite4", dict(batch=1, seq=200, V=512)),
    ("main3_aligned", dict(batch=1, seq=256, V=640)),
]


@pytest.mark.parametrize("name,small", SMALL_BF16)
def test_bf16_tensor_core_path_small(name, small):
    cfg = wl.small_variant(wl.CONFIGS[name], **small)
    d = wl.make_inputs(cfg, with_tables=False)
    _check_all(d, cfg.alpha_d, grad_scale=1.0)


# Vocabulary sizes whose split counts leave the loss merge's thread rows (32
# per 32-token block, four splits loaded per batch) partial batches:
# V = 10240 is 80 splits (3 per row, one row of 2, the last five rows empty),
# V = 24576 is 192 splits (6 per row: a full batch and a partial one).
@pytest.mark.parametrize("V", [10240, 24576])
def test_forward_merge_split_batches(V):
    cfg = wl.small_variant(wl.CONFIGS["main3"], batch=1, seq=130, V=V)
    d = wl.make_inputs(cfg, with_tables=False)
    y, h, W = _gpu_inputs(d)
    st = new_status()
    losses, stats = multiexit_loss_fwd(y, h, W, cfg.alpha_d, status=st)
    assert status_read(st) == (0, 0)
    r = _oracle(d, cfg.alpha_d, need_grad=False)
    M = cfg.M
    assert_loss_close(losses, _losses_expected(r, M), "losses")
    s = f64(stats)
    assert_stats_close(s[:M], r["lse"], "lse")
    assert_stats_close(s[M:2 * M], r["tgt"], "target logits")
    assert_stats_close(s[2 * M:3 * M - 1], r["S"], "distillation statistic")


def _pieces(cfg, ws_bytes):
    Tb, Vc, _ = multiexit_loss_bwd_plan(cfg.T, cfg.D, cfg.V, torch.bfloat16, ws_bytes)
    return Tb, Vc, -(-cfg.T // Tb), -(-cfg.V // Vc)


# Small workspaces force the backward pass into many token blocks and
# vocabulary chunks: ragged last blocks (T not a multiple of 128), a half-tile
# last chunk (V = 640), first / middle / last chunks of the dh partial sums and
# the dW additions of later blocks.
CHUNKED = [
    ("main3", dict(batch=1, seq=300, V=1024)),
    ("proxy2", dict(batch=2, seq=97, V=2048)),
    ("suite4", dict(batch=1, seq=200, V=512)),
    ("main3_aligned", dict(batch=1, seq=256, V=640)),
]


@pytest.mark.parametrize("name,small", CHUNKED)
def test_chunked_backward_smallest_workspace(name, small):
    cfg = wl.small_variant(wl.CONFIGS[name], **small)
    d = wl.make_inputs(cfg, with_tables=False)
    _, _, mn = multiexit_loss_bwd_plan(cfg.T, cfg.D, cfg.V, torch.bfloat16, 0)
    Tb, Vc, nT, nV = _pieces(cfg, mn)
    assert Tb == 128 and nT > 1
    _check_all(d, cfg.alpha_d, grad_scale=1.0, bwd_ws_bytes=mn)
    # a middle size: fewer, larger pieces, same results within the tolerance
    mid = mn
    while _pieces(cfg, mid)[2:] == (nT, nV):
        mid = mid * 5 // 4
    _check_all(d, cfg.alpha_d, grad_scale=1.0, bwd_ws_bytes=mid)


@pytest.mark.parametrize("distill,teacher_grad", [("ce", True), ("reverse_kl", False), ("js", True),
                                                  ("accept", False)])
def test_chunked_backward_options(distill, teacher_grad):
    cfg = wl.small_variant(wl.CONFIGS["main3"], batch=1, seq=300, V=1024)
    d = wl.make_inputs(cfg, with_tables=False)
    _, _, mn = multiexit_loss_bwd_plan(cfg.T, cfg.D, cfg.V, torch.bfloat16, 0)
    assert _pieces(cfg, mn)[3] > 2
    _check_all(d, 0.6, 2.0, exit_weights=[1.5, 0.7, 0.8], distill=distill, teacher_grad=teacher_grad,
               bwd_ws_bytes=mn)


def test_chunked_backward_accumulate_and_determinism():
    cfg = wl.small_variant(wl.CONFIGS["suite4"], batch=1, seq=200, V=512)
    d = wl.make_inputs(cfg, with_tables=False)
    y, h, W = _gpu_inputs(d)
    _, _, mn = multiexit_loss_bwd_plan(cfg.T, cfg.D, cfg.V, torch.bfloat16, 0)
    ws = torch.empty(mn, dtype=torch.uint8, device="cuda")
    _, stats = multiexit_loss_fwd(y, h, W, 0.3)
    r = oracle.multiexit_loss(d.y, d.o, d.W, alpha_d=0.3)
    base = [torch.randn(w.shape, dtype=torch.float32, device="cuda") for w in W]
    dW = [b.clone() for b in base]
    dh1, _ = multiexit_loss_bwd(y, h, W, stats, 0.3, dW=dW, accumulate_dW=True, workspace=ws)
    for m in range(cfg.M):
        assert_grad_close(dW[m] - base[m], r["dW"][m], f"accumulated dW[{m}]")
    g1 = multiexit_loss_bwd(y, h, W, stats, 0.3, workspace=ws)
    g2 = multiexit_loss_bwd(y, h, W, stats, 0.3, workspace=ws)
    for a, b in zip(g1[0] + g1[1], g2[0] + g2[1]):
        assert torch.equal(a, b)
    for a, b in zip(dh1, g1[0]):
        assert torch.equal(a, b)


def test_alpha_and_grad_scale_are_runtime_arguments():
    cfg = wl.small_variant(wl.CONFIGS["proxy2"], batch=1, seq=130, V=256)
    d = wl.make_inputs(cfg, with_tables=False)
    for alpha, gs in ((0.0, 1.0), (0.7, 3.5)):
        _check_all(d, alpha, gs)


@pytest.mark.parametrize("name,small", [("tiny3", None), ("main3", dict(batch=1, seq=200, V=512))])
def test_exit_weights(name, small):
    cfg = wl.CONFIGS[name] if small is None else wl.small_variant(wl.CONFIGS[name], **small)
    d = wl.make_inputs(cfg, with_tables=False)
    _check_all(d, 0.3, 1.0, exit_weights=[0.5, 2.0, 1.25])


@pytest.mark.parametrize("name,small", [("tiny3", None), ("main3", dict(batch=1, seq=200, V=512)),
                                        ("suite4", dict(batch=1, seq=130, V=384)),
                                        ("main3_aligned", dict(batch=1, seq=256, V=768))])
@pytest.mark.parametrize("distill", ["reverse_kl", "js", "accept"])
def test_alternative_distillation(name, small, distill):
    cfg = wl.CONFIGS[name] if small is None else wl.small_variant(wl.CONFIGS[name], **small)
    d = wl.make_inputs(cfg, with_tables=False)
    _check_all(d, 0.3, 1.0, distill=distill)
    _check_all(d, 0.6, 2.0, exit_weights=[1.5, 0.5] + [1.0] * (cfg.M - 2), distill=distill)


@pytest.mark.parametrize("name,small", [("tiny3", None), ("main3", dict(batch=1, seq=200, V=512)),
                                        ("suite4", dict(batch=1, seq=130, V=384)),
                                        ("main3_aligned", dict(batch=1, seq=256, V=768)),
                                        ("proxy2", dict(batch=1, seq=160, V=512))])
@pytest.mark.parametrize("distill", ["ce", "reverse_kl", "js", "accept"])
def test_teacher_gradient(name, small, distill):
    cfg = wl.CONFIGS[name] if small is None else wl.small_variant(wl.CONFIGS[name], **small)
    d = wl.make_inputs(cfg, with_tables=False)
    _check_all(d, 0.3, 1.0, distill=distill, teacher_grad=True)
    _check_all(d, 0.6, 2.0, exit_weights=[1.5] + [0.7] * (cfg.M - 2) + [0.8], distill=distill,
               teacher_grad=True)


def test_single_exit_and_accumulate():
    cfg = wl.small_variant(wl.CONFIGS["main3"], batch=1, seq=130, V=256)
    d = wl.make_inputs(cfg, with_tables=False)
    y, h, W = _gpu_inputs(d)
    losses, stats = multiexit_loss_fwd(y, h[:1], W[:1], 0.3)
    r = oracle.multiexit_loss(d.y, d.o[:1], d.W[:1], alpha_d=0.3)
    assert_loss_close(losses, [r["ce_lm"][0], r["loss"]])
    base = [torch.randn(w.shape, dtype=torch.float32, device="cuda") for w in W[:1]]
    dW = [b.clone() for b in base]
    multiexit_loss_bwd(y, h[:1], W[:1], stats, 0.3, dW=dW, accumulate_dW=True)
    assert_grad_close(dW[0] - base[0], r["dW"][0], "accumulated dW")


def test_bad_targets_are_flagged():
    cfg = wl.small_variant(wl.CONFIGS["proxy2"], batch=1, seq=128, V=256)
    d = wl.make_inputs(cfg, with_tables=False)
    y, h, W = _gpu_inputs(d)
    y = y.clone()
    y[3] = -5
    y[77] = cfg.V + 1
    st = new_status()
    losses, stats = multiexit_loss_fwd(y, h, W, 0.3, status=st)
    code, word = status_read(st)
    assert code == 5 and word & 1
    assert torch.isfinite(losses).all()
    dh, dW = multiexit_loss_bwd(y, h, W, stats, 0.3, status=st)
    assert status_read(st)[0] == 5
    for m in range(cfg.M):
        assert torch.all(dh[m][3] == 0) and torch.all(dh[m][77] == 0)
        assert torch.isfinite(dW[m]).all()


def test_repeated_calls_are_deterministic():
    cfg = wl.small_variant(wl.CONFIGS["main3"], batch=1, seq=257, V=512)
    d = wl.make_inputs(cfg, with_tables=False)
    y, h, W = _gpu_inputs(d)
    l1, s1 = multiexit_loss_fwd(y, h, W, 0.3)
    l2, s2 = multiexit_loss_fwd(y, h, W, 0.3)
    assert torch.equal(l1, l2) and torch.equal(s1, s2)
    g1 = multiexit_loss_bwd(y, h, W, s1, 0.3)
    g2 = multiexit_loss_bwd(y, h, W, s1, 0.3)
    for a, b in zip(g1[0] + g1[1], g2[0] + g2[1]):
        assert torch.equal(a, b)


FULL = ["proxy2", "main3", "main3_aligned", "suite4"]


def _oracle_vocab_rows_by_slices(d, alpha, vrows, n_slices):
    """oracle.multiexit_loss_vocab_rows over all tokens, evaluated on token
    slices and summed (every term is a sum over tokens: with grad_scale =
    |slice|/T each slice's gradient rows carry the full 1/T, and its means are
    rescaled by |slice|/T).  Only bounds the memory of one call."""
    T = d.cfg.T
    M = d.cfg.M
    bounds = np.linspace(0, T, n_slices + 1).astype(int)
    ce_lm = np.zeros(M)
    ce_kd = np.zeros(max(M - 1, 0))
    rows = None
    for a, b in zip(bounds[:-1], bounds[1:]):
        r = oracle.multiexit_loss_vocab_rows(d.y[a:b], [h[a:b] for h in d.o], d.W, alpha_d=alpha,
                                             grad_scale=(b - a) / T, vrows=vrows)
        ce_lm += r["ce_lm"] * (b - a) / T
        ce_kd += r["ce_kd"] * (b - a) / T
        rows = r["dW_rows"] if rows is None else [x + y for x, y in zip(rows, r["dW_rows"])]
    loss = float(np.sum((1.0 - alpha) * ce_lm[:M - 1]) + np.sum(alpha * ce_kd) + ce_lm[M - 1])
    return {"ce_lm": ce_lm, "ce_kd": ce_kd, "loss": loss, "dW_rows": rows}


@pytest.mark.slow
@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(name):
    """Full-size workloads in the benchmark's launch configuration (the backward
    call with the workspace the query returns, so split into token blocks and
    vocabulary chunks as the benchmark runs it).

    Sampled tokens: the per-token statistics and dh rows against the oracle.
    The losses and sampled vocabulary rows of dW (random ids and target ids)
    against the oracle over all tokens, which takes the full fp64 forward
    (about 2.5e13 flop for the T = 32768 workloads).  At any size: the reported
    losses equal the token means of the reported statistics, and the columns of
    every dW sum to zero up to rounding.
    """
    cfg = wl.CONFIGS[name]
    d = wl.make_inputs(cfg, with_tables=False)
    y, h, W = _gpu_inputs(d)
    M = cfg.M
    st = new_status()
    losses, stats = multiexit_loss_fwd(y, h, W, cfg.alpha_d, status=st)
    dh, dW = multiexit_loss_bwd(y, h, W, stats, cfg.alpha_d, 1.0, status=st)
    assert status_read(st) == (0, 0)
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(cfg.T, size=64, replace=False))
    r = oracle.multiexit_loss(d.y, d.o, d.W, alpha_d=cfg.alpha_d, rows=rows)
    s = f64(stats)
    assert_stats_close(s[:M, rows], r["lse"], "lse")
    assert_stats_close(s[M:2 * M, rows], r["tgt"], "target logits")
    assert_stats_close(s[2 * M:, rows], r["S"], "teacher-weighted logits")
    for m in range(M):
        assert_grad_close(dh[m][torch.from_numpy(rows).cuda()], r["dh"][m], f"dh[{m}] rows")
    # losses are the token means of the statistics
    L = f64(losses)
    ce_lm = (s[:M] - s[M:2 * M]).mean(axis=1)
    ce_kd = (s[:M - 1] - s[2 * M:]).mean(axis=1)
    assert_loss_close(L[:M], ce_lm, "CE_LM vs stats")
    assert_loss_close(L[M:2 * M - 1], ce_kd, "CE_KD vs stats")
    tot = np.sum((1 - cfg.alpha_d) * ce_lm[:M - 1]) + np.sum(cfg.alpha_d * ce_kd) + ce_lm[M - 1]
    assert_loss_close(L[-1:], [tot], "L vs stats")
    # sum over the vocabulary of every dW column vanishes (softmax rows sum to one)
    dW_host = [t.cpu() for t in dW]
    for m in range(M):
        col = dW_host[m].double().sum(dim=0)
        scale = dW_host[m].double().abs().sum(dim=0)
        assert float((col.abs() / scale.clamp_min(1e-30)).max()) < 2e-3, f"dW[{m}] column sums"
    # losses and >= 48 vocabulary rows of dW (random ids, and the targets of the
    # first tokens) against the oracle over every token
    vrows = np.unique(np.concatenate([rng.choice(cfg.V, size=48, replace=False), d.y[:16]]))
    rv = _oracle_vocab_rows_by_slices(d, cfg.alpha_d, vrows, max(1, cfg.T // 4096))
    assert_loss_close(losses, np.concatenate([rv["ce_lm"], rv["ce_kd"], [rv["loss"]]]), "losses")
    for m in range(M):
        assert_grad_close(dW_host[m][torch.from_numpy(vrows)], rv["dW_rows"][m], f"dW[{m}] rows")
