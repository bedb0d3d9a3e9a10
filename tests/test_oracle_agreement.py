"""Pins for the inter-exit agreement oracle (acceptance, KL, top-1 agreement)."""
import math

import numpy as np

from oracle import exit_agreement, multiexit_loss


def _sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def _rand(M=3, T=7, D=(3, 4, 6), V=13, seed=0):
    rng = np.random.default_rng(seed)
    h = [rng.normal(0, 2.0, size=(T, d)) for d in D[:M]]
    W = [rng.normal(0, 1.0 / math.sqrt(d), size=(V, d)) for d in D[:M]]
    return h, W


def test_two_class_closed_form():
    # p = (s(a), 1 - s(a)), q = (s(b), 1 - s(b)): beta = 1 - |s(a) - s(b)|,
    # KL(p || q) = s(a) log(s(a)/s(b)) + s(-a) log(s(-a)/s(-b)); argmax decided by sign
    a, b = 1.3, -0.4
    h = [np.array([[b]]), np.array([[a]])]
    W = [np.array([[1.0], [0.0]]), np.array([[1.0], [0.0]])]
    r = exit_agreement(h, W)
    pa, pb = _sig(a), _sig(b)
    np.testing.assert_allclose(r["beta"][0, 0], 1.0 - abs(pa - pb), rtol=1e-14)
    kl = pa * math.log(pa / pb) + (1 - pa) * math.log((1 - pa) / (1 - pb))
    np.testing.assert_allclose(r["kl"][0, 0], kl, rtol=1e-13)
    assert r["top1"][0, 0] == 1 and r["top1"][1, 0] == 0 and r["agree"][0, 0] == 0.0


def test_identical_exits_agree_completely():
    h, W = _rand(M=2, D=(5, 5), seed=1)
    h[0], W[0] = h[1].copy(), W[1].copy()
    r = exit_agreement(h, W)
    np.testing.assert_allclose(r["beta"], 1.0, rtol=1e-13)
    np.testing.assert_allclose(r["kl"], 0.0, atol=1e-13)
    assert np.all(r["agree"] == 1.0)


def test_acceptance_is_one_minus_total_variation_and_kl_nonnegative():
    h, W = _rand(seed=2)
    r = exit_agreement(h, W)
    logits = [hm @ w.T for hm, w in zip(h, W)]
    P = [np.exp(l - l.max(1, keepdims=True)) for l in logits]
    P = [p / p.sum(1, keepdims=True) for p in P]
    for m in range(2):
        tv = 0.5 * np.abs(P[m] - P[2]).sum(1)
        np.testing.assert_allclose(r["beta"][m], 1.0 - tv, rtol=1e-12)
        assert np.all(r["kl"][m] >= -1e-14)


def test_kl_is_distillation_cross_entropy_minus_teacher_entropy():
    # CE_KD,m = H(p_M) + KL(p_M || q_m) token by token
    h, W = _rand(seed=3)
    y = np.zeros(7, dtype=np.int64)
    r = exit_agreement(h, W)
    lo = multiexit_loss(y, h, W, need_grad=False)
    lM = h[2] @ W[2].T
    p = np.exp(lM - lo["lse"][2][:, None])
    H = -(p * np.log(p)).sum(1)
    for m in range(2):
        ce = lo["lse"][m] - lo["S"][m]
        np.testing.assert_allclose(ce, H + r["kl"][m], rtol=1e-12)


def test_top1_brute_force_and_means():
    h, W = _rand(M=3, T=9, V=16, seed=4)
    r = exit_agreement(h, W)
    for m in range(3):
        for t in range(9):
            l = [float(np.dot(h[m][t], W[m][v])) for v in range(16)]
            best = 0
            for v in range(1, 16):
                if l[v] > l[best]:
                    best = v
            assert r["top1"][m, t] == best
    for m in range(2):
        np.testing.assert_allclose(r["agree_mean"][m], np.mean(r["top1"][m] == r["top1"][2]), rtol=0)
        np.testing.assert_allclose(r["beta_mean"][m], np.mean(r["beta"][m]), rtol=1e-15)
    rows = np.array([4, 0, 8])
    rs = exit_agreement(h, W, rows=rows)
    np.testing.assert_allclose(rs["kl"], r["kl"][:, rows], rtol=1e-14)
