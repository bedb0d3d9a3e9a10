"""Pins for the multi-exit loss oracle.

Closed forms, special cases, brute-force enumeration on V <= 16 and finite
differences, chosen so a dropped term, a swapped mixing weight, a wrong sign or
a transposed operand in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import multiexit_loss, multiexit_loss_vocab_rows, softmax_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")


def _rand_suite(M=3, T=6, D=(3, 5, 8), V=11, seed=0, scale=1.0):
    rng = np.random.default_rng(seed)
    y = rng.integers(0, V, size=T)
    h = [rng.normal(0, 2.0, size=(T, d)) for d in D[:M]]
    W = [scale * rng.normal(0, 1.0 / math.sqrt(d), size=(V, d)) for d in D[:M]]
    return y, h, W


def _softplus(z):
    return math.log1p(math.exp(z))


def _sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def test_two_class_closed_form_with_page_mix():
    # V=2, one token, target 0; teacher logits (a, 0), student logits (b, 0).
    # With the pages' mix (0.7 next-token + 0.3 cross-entropy to the largest exit):
    #   CE_LM = softplus(-logit gap), CE_KD = -(s(a) log s(b) + s(-a) log s(-b)).
    fig = json.load(open(GOLDEN))
    alpha = fig["alpha_d"]["value"]
    assert (fig["mix_weights"]["lm"], fig["mix_weights"]["kd"]) == (0.7, 0.3)
    a, b = 2.0, -1.0
    y = np.array([0])
    h = [np.array([[b]]), np.array([[a]])]
    W = [np.array([[1.0], [0.0]]), np.array([[1.0], [0.0]])]
    r = multiexit_loss(y, h, W, alpha_d=alpha)
    ce_lm1, ce_lm2 = _softplus(-b), _softplus(-a)
    ce_kd1 = -(_sig(a) * math.log(_sig(b)) + _sig(-a) * math.log(_sig(-b)))
    L = 0.7 * ce_lm1 + 0.3 * ce_kd1 + ce_lm2
    np.testing.assert_allclose(r["ce_lm"], [ce_lm1, ce_lm2], rtol=1e-14)
    np.testing.assert_allclose(r["ce_kd"], [ce_kd1], rtol=1e-14)
    np.testing.assert_allclose(r["loss"], L, rtol=1e-14)
    # dL/dh_1 = d/db: s(b) - 0.7 - 0.3 s(a); teacher is stop-gradient:
    # dL/dh_2 = d/da of CE_LM,2 only: s(a) - 1
    np.testing.assert_allclose(r["dh"][0][0, 0], _sig(b) - 0.7 - 0.3 * _sig(a), rtol=1e-13)
    np.testing.assert_allclose(r["dh"][1][0, 0], _sig(a) - 1.0, rtol=1e-13)
    # dW^1 rows: row 0 gets (q0 - 0.7 - 0.3 p0) * h, row 1 gets (q1 - 0.3 p1) * h
    np.testing.assert_allclose(r["dW"][0][:, 0],
                               [(_sig(b) - 0.7 - 0.3 * _sig(a)) * b,
                                (_sig(-b) - 0.3 * _sig(-a)) * b], rtol=1e-13)


def test_zero_heads_closed_form():
    # W = 0 -> every softmax is uniform: lse = log V, CE_LM = CE_KD = log V,
    # L = M log V; dh = 0; dW^m[v] = c_m/T sum_t (1/V - [y_t = v]) h_t with
    # c_m = 1 - alpha_d for students and 1 for the teacher.
    M, T, V, D = 3, 7, 13, (2, 3, 4)
    rng = np.random.default_rng(1)
    y = rng.integers(0, V, size=T)
    h = [rng.normal(size=(T, d)) for d in D]
    W = [np.zeros((V, d)) for d in D]
    alpha = 0.3
    r = multiexit_loss(y, h, W, alpha_d=alpha, grad_scale=1.0)
    logV = math.log(V)
    np.testing.assert_allclose(r["lse"], logV, rtol=1e-14)
    np.testing.assert_allclose(r["ce_lm"], logV, rtol=1e-14)
    np.testing.assert_allclose(r["ce_kd"], logV, rtol=1e-14)
    np.testing.assert_allclose(r["loss"], M * logV, rtol=1e-14)
    for m in range(M):
        assert np.all(r["dh"][m] == 0.0)
        c = (1 - alpha) if m < M - 1 else 1.0
        exp = np.zeros((V, D[m]))
        for t in range(T):
            for v in range(V):
                exp[v] += c / T * ((1.0 / V) - (1.0 if y[t] == v else 0.0)) * h[m][t]
        np.testing.assert_allclose(r["dW"][m], exp, rtol=1e-12, atol=1e-15)


def test_alpha_zero_is_plain_cross_entropy_textbook():
    # alpha_d = 0: L = sum_m CE_LM,m, with CE written as log(sum exp) - l_y
    # without any max shift (V <= 16 keeps exp in range).
    y, h, W = _rand_suite(M=3, T=5, D=(2, 3, 4), V=9, seed=2)
    r = multiexit_loss(y, h, W, alpha_d=0.0, need_grad=False)
    tot = 0.0
    for m in range(3):
        s = 0.0
        for t in range(5):
            l = [sum(h[m][t, k] * W[m][v, k] for k in range(h[m].shape[1])) for v in range(9)]
            s += math.log(sum(math.exp(z) for z in l)) - l[y[t]]
        tot += s / 5
    np.testing.assert_allclose(r["loss"], tot, rtol=1e-13)


def test_student_equal_to_teacher_gives_teacher_entropy():
    y, h, W = _rand_suite(M=2, T=8, D=(6, 6), V=15, seed=3)
    h[0], W[0] = h[1].copy(), W[1].copy()
    r = multiexit_loss(y, h, W, alpha_d=0.3)
    H = 0.0
    for t in range(8):
        l = [float(np.dot(h[1][t], W[1][v])) for v in range(15)]
        z = sum(math.exp(v) for v in l)
        p = [math.exp(v) / z for v in l]
        H += -sum(pi * math.log(pi) for pi in p)
    np.testing.assert_allclose(r["ce_kd"][0], H / 8, rtol=1e-13)
    # KD part of the student gradient vanishes: G_student = (1 - alpha) G_teacher
    np.testing.assert_allclose(r["dh"][0], 0.7 * r["dh"][1], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(r["dW"][0], 0.7 * r["dW"][1], rtol=1e-12, atol=1e-15)


def test_probabilities_sum_to_one():
    rng = np.random.default_rng(4)
    l = rng.normal(0, 30, size=(20, 50))
    p = softmax_rows(l)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(p >= 0)


def test_brute_force_enumeration_small_vocab():
    # V <= 16, T <= 8, D <= 8: every quantity by explicit loops over v.
    M, T, D, V, alpha = 3, 6, (2, 5, 8), 16, 0.3
    y, h, W = _rand_suite(M=M, T=T, D=D, V=V, seed=5)
    r = multiexit_loss(y, h, W, alpha_d=alpha)
    ce_lm = [0.0] * M
    ce_kd = [0.0] * (M - 1)
    for t in range(T):
        logits = [[sum(h[m][t, k] * W[m][v, k] for k in range(D[m])) for v in range(V)]
                  for m in range(M)]
        Z = [sum(math.exp(l) for l in logits[m]) for m in range(M)]
        lse = [math.log(z) for z in Z]
        pM = [math.exp(l) / Z[M - 1] for l in logits[M - 1]]
        for m in range(M):
            np.testing.assert_allclose(r["lse"][m, t], lse[m], rtol=1e-13)
            np.testing.assert_allclose(r["tgt"][m, t], logits[m][y[t]], rtol=1e-13)
            ce_lm[m] += lse[m] - logits[m][y[t]]
        for m in range(M - 1):
            Sm = sum(pM[v] * logits[m][v] for v in range(V))
            np.testing.assert_allclose(r["S"][m, t], Sm, rtol=1e-12, atol=1e-14)
            ce_kd[m] += -sum(pM[v] * (logits[m][v] - lse[m]) for v in range(V))
    ce_lm = [c / T for c in ce_lm]
    ce_kd = [c / T for c in ce_kd]
    np.testing.assert_allclose(r["ce_lm"], ce_lm, rtol=1e-13)
    np.testing.assert_allclose(r["ce_kd"], ce_kd, rtol=1e-13)
    L = sum((1 - alpha) * ce_lm[m] + alpha * ce_kd[m] for m in range(M - 1)) + ce_lm[M - 1]
    np.testing.assert_allclose(r["loss"], L, rtol=1e-13)


def _teacher_fixed_loss(y, h, W, alpha, hM_fixed, WM_fixed, m_var):
    """Loss with the teacher's softmax held at the given (fixed) parameters.

    The teacher is stop-gradient, so finite differences of the student terms
    must hold the teacher's distribution fixed while the student moves.
    """
    M = len(h)
    r_t = multiexit_loss(y, h[:M - 1] + [hM_fixed], W[:M - 1] + [WM_fixed], alpha_d=alpha,
                         need_grad=False)
    return r_t["loss"]


def test_gradients_match_finite_differences():
    M, T, D, V, alpha, gs = 3, 4, (2, 3, 5), 7, 0.3, 1.7
    y, h, W = _rand_suite(M=M, T=T, D=D, V=V, seed=6)
    r = multiexit_loss(y, h, W, alpha_d=alpha, grad_scale=gs)
    eps = 1e-6
    # students: the teacher enters L through CE_LM,M (independent of students)
    # and through p_M inside CE_KD (held fixed because it is stop-gradient;
    # moving a student parameter does not change it anyway).
    for m in range(M - 1):
        for arr, grad in ((h, r["dh"][m]), (W, r["dW"][m])):
            num = np.zeros_like(arr[m])
            for idx in np.ndindex(arr[m].shape):
                base = arr[m][idx]
                arr[m][idx] = base + eps
                lp = multiexit_loss(y, h, W, alpha_d=alpha, need_grad=False)["loss"]
                arr[m][idx] = base - eps
                lm = multiexit_loss(y, h, W, alpha_d=alpha, need_grad=False)["loss"]
                arr[m][idx] = base
                num[idx] = gs * (lp - lm) / (2 * eps)
            np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-9)
    # teacher: stop-gradient means only CE_LM,M depends on it -> a 1-exit loss
    m = M - 1
    for which in ("h", "W"):
        arr = h if which == "h" else W
        grad = r["dh"][m] if which == "h" else r["dW"][m]
        num = np.zeros_like(arr[m])
        for idx in np.ndindex(arr[m].shape):
            base = arr[m][idx]
            arr[m][idx] = base + eps
            lp = multiexit_loss(y, [h[m]], [W[m]], need_grad=False)["loss"]
            arr[m][idx] = base - eps
            lm = multiexit_loss(y, [h[m]], [W[m]], need_grad=False)["loss"]
            arr[m][idx] = base
            num[idx] = gs * (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-9)


def test_head_gradient_columns_sum_to_zero():
    # sum_v G[t, v] = 0 for every token, hence sum_v dW^m[v, :] = 0.
    y, h, W = _rand_suite(M=3, T=9, D=(4, 6, 8), V=21, seed=7)
    r = multiexit_loss(y, h, W, alpha_d=0.3)
    for m in range(3):
        np.testing.assert_allclose(r["dW"][m].sum(axis=0), 0.0, atol=1e-14)


def test_token_blocking_and_row_selection_do_not_change_results():
    y, h, W = _rand_suite(M=3, T=23, D=(4, 6, 8), V=19, seed=8)
    a = multiexit_loss(y, h, W, token_block=1)
    b = multiexit_loss(y, h, W, token_block=256)
    np.testing.assert_allclose(a["loss"], b["loss"], rtol=1e-13)
    for m in range(3):
        np.testing.assert_allclose(a["dW"][m], b["dW"][m], rtol=1e-12, atol=1e-15)
    rows = np.array([3, 0, 22, 7])
    c = multiexit_loss(y, h, W, rows=rows)
    for m in range(3):
        np.testing.assert_allclose(c["dh"][m], b["dh"][m][rows], rtol=1e-13)
        np.testing.assert_allclose(c["lse"][m], b["lse"][m][rows], rtol=1e-13)


def test_single_exit_has_no_distillation():
    y, h, W = _rand_suite(M=1, T=5, D=(4,), V=10, seed=9)
    r = multiexit_loss(y, h, W, alpha_d=0.3)
    assert r["ce_kd"].shape == (0,)
    np.testing.assert_allclose(r["loss"], r["ce_lm"][0], rtol=1e-15)


def test_vocab_row_restriction_matches_full_gradient():
    # the restricted form must agree with the full definition on every requested row
    y, h, W = _rand_suite(M=3, T=37, D=(4, 6, 8), V=29, seed=10)
    full = multiexit_loss(y, h, W, alpha_d=0.3, grad_scale=2.0, token_block=5)
    rows = np.array([0, 28, 3, int(y[0]), 17])
    r = multiexit_loss_vocab_rows(y, h, W, alpha_d=0.3, grad_scale=2.0, vrows=rows, token_block=8)
    np.testing.assert_allclose(r["loss"], full["loss"], rtol=1e-13)
    np.testing.assert_allclose(r["ce_kd"], full["ce_kd"], rtol=1e-13)
    for m in range(3):
        np.testing.assert_allclose(r["dW_rows"][m], full["dW"][m][rows], rtol=1e-12, atol=1e-15)


def test_exit_weights_are_linear_in_each_exit():
    # L(lambda) = sum_m lambda_m L_m and each gradient scales with its own lambda
    y, h, W = _rand_suite(M=3, T=6, D=(3, 5, 8), V=11, seed=21)
    lam = np.array([0.5, 2.0, 1.25])
    base = multiexit_loss(y, h, W, alpha_d=0.3)
    r = multiexit_loss(y, h, W, alpha_d=0.3, exit_weights=lam)
    Lm = [0.7 * base["ce_lm"][0] + 0.3 * base["ce_kd"][0], 0.7 * base["ce_lm"][1] + 0.3 * base["ce_kd"][1],
          base["ce_lm"][2]]
    np.testing.assert_allclose(r["loss"], float(np.dot(lam, Lm)), rtol=1e-14)
    for m in range(3):
        np.testing.assert_allclose(r["dh"][m], lam[m] * base["dh"][m], rtol=1e-13, atol=1e-16)
        np.testing.assert_allclose(r["dW"][m], lam[m] * base["dW"][m], rtol=1e-13, atol=1e-16)
    ones = multiexit_loss(y, h, W, alpha_d=0.3, exit_weights=[1.0, 1.0, 1.0])
    np.testing.assert_allclose(ones["loss"], base["loss"], rtol=1e-15)


def test_exit_weights_finite_differences():
    M, T, D, V, alpha = 2, 3, (2, 4), 5, 0.3
    y, h, W = _rand_suite(M=M, T=T, D=D, V=V, seed=22)
    lam = [1.7, 0.4]
    r = multiexit_loss(y, h, W, alpha_d=alpha, exit_weights=lam)
    eps = 1e-6
    # student: its whole loss term moves; teacher held fixed inside CE_KD (stop-gradient)
    num = np.zeros_like(h[0])
    for idx in np.ndindex(h[0].shape):
        b = h[0][idx]
        h[0][idx] = b + eps
        lp = multiexit_loss(y, h, W, alpha_d=alpha, need_grad=False, exit_weights=lam)["loss"]
        h[0][idx] = b - eps
        lm = multiexit_loss(y, h, W, alpha_d=alpha, need_grad=False, exit_weights=lam)["loss"]
        h[0][idx] = b
        num[idx] = (lp - lm) / (2 * eps)
    np.testing.assert_allclose(r["dh"][0], num, rtol=1e-6, atol=1e-9)


# ------------------------------------------------------------------ reverse KL distillation
def test_reverse_kl_two_class_closed_form():
    # student (b, 0), teacher (a, 0): KL(q || p) = s(b) log(s(b)/s(a)) + s(-b) log(s(-b)/s(-a))
    a, b = 2.0, -1.0
    y = np.array([0])
    h = [np.array([[b]]), np.array([[a]])]
    W = [np.array([[1.0], [0.0]]), np.array([[1.0], [0.0]])]
    r = multiexit_loss(y, h, W, alpha_d=0.3, distill="reverse_kl")
    rkl = _sig(b) * math.log(_sig(b) / _sig(a)) + _sig(-b) * math.log(_sig(-b) / _sig(-a))
    np.testing.assert_allclose(r["ce_kd"][0], rkl, rtol=1e-13)
    np.testing.assert_allclose(r["loss"], 0.7 * _softplus(-b) + 0.3 * rkl + _softplus(-a), rtol=1e-13)


def test_reverse_kl_vanishes_for_identical_exits_and_is_nonnegative():
    y, h, W = _rand_suite(M=2, T=6, D=(5, 5), V=12, seed=31)
    h[0], W[0] = h[1].copy(), W[1].copy()
    r = multiexit_loss(y, h, W, alpha_d=0.3, distill="reverse_kl")
    np.testing.assert_allclose(r["ce_kd"], 0.0, atol=1e-13)
    y, h, W = _rand_suite(M=3, T=6, seed=32)
    r = multiexit_loss(y, h, W, alpha_d=0.3, distill="reverse_kl")
    assert np.all(r["ce_kd"] >= 0)
    # per token KL(q||p) = R - lse_m + lse_M
    base = multiexit_loss(y, h, W, alpha_d=0.3)
    for m in range(2):
        kl_t = r["R"][m] - r["lse"][m] + r["lse"][2]
        np.testing.assert_allclose(kl_t.mean(), r["ce_kd"][m], rtol=1e-12)
    np.testing.assert_allclose(r["ce_lm"], base["ce_lm"], rtol=1e-15)


def test_reverse_kl_gradients_match_finite_differences():
    M, T, D, V, alpha = 2, 3, (3, 4), 6, 0.4
    y, h, W = _rand_suite(M=M, T=T, D=D, V=V, seed=33)
    r = multiexit_loss(y, h, W, alpha_d=alpha, grad_scale=1.3, distill="reverse_kl")
    eps = 1e-6
    for arr, grad in ((h, r["dh"][0]), (W, r["dW"][0])):
        num = np.zeros_like(arr[0])
        for idx in np.ndindex(arr[0].shape):
            b = arr[0][idx]
            arr[0][idx] = b + eps
            lp = multiexit_loss(y, h, W, alpha_d=alpha, need_grad=False, distill="reverse_kl")["loss"]
            arr[0][idx] = b - eps
            lm = multiexit_loss(y, h, W, alpha_d=alpha, need_grad=False, distill="reverse_kl")["loss"]
            arr[0][idx] = b
            num[idx] = 1.3 * (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-9)
    # alpha_d = 0 gives the same gradients as the cross-entropy form
    a = multiexit_loss(y, h, W, alpha_d=0.0, distill="reverse_kl")
    c = multiexit_loss(y, h, W, alpha_d=0.0)
    np.testing.assert_allclose(a["dh"][0], c["dh"][0], rtol=1e-13, atol=1e-16)


# ------------------------------------------------------------------ Jensen-Shannon distillation
def test_js_matches_scipy_distance_by_enumeration():
    # scipy's jensenshannon returns the square root of the divergence (natural log by default)
    from scipy.spatial.distance import jensenshannon
    y, h, W = _rand_suite(M=3, T=5, D=(3, 5, 8), V=9, seed=41, scale=3.0)
    r = multiexit_loss(y, h, W, alpha_d=0.3, distill="js")
    pM = softmax_rows(h[2] @ W[2].T)
    for m in range(2):
        q = softmax_rows(h[m] @ W[m].T)
        js = np.array([jensenshannon(q[t], pM[t]) ** 2 for t in range(5)])
        np.testing.assert_allclose(r["ce_kd"][m], js.mean(), rtol=1e-10)
        # J = KL(q || mixture) / 2, written out per token and per vocabulary entry
        mix = 0.5 * (q + pM)
        kq = np.array([sum(q[t, v] * math.log(q[t, v] / mix[t, v]) for v in range(9)) for t in range(5)])
        np.testing.assert_allclose(r["J"][m], 0.5 * kq, rtol=1e-12)
        kp = np.array([sum(pM[t, v] * math.log(pM[t, v] / mix[t, v]) for v in range(9)) for t in range(5)])
        np.testing.assert_allclose(r["Jp"][m], 0.5 * kp, rtol=1e-12)
        np.testing.assert_allclose(np.mean(r["J"][m] + r["Jp"][m]), r["ce_kd"][m], rtol=1e-12)
    assert np.all(r["ce_kd"] >= 0) and np.all(r["ce_kd"] <= math.log(2.0))


def test_js_is_symmetric_in_student_and_teacher():
    y, h, W = _rand_suite(M=2, T=7, D=(6, 6), V=13, seed=42)
    a = multiexit_loss(y, h, W, alpha_d=0.3, distill="js")
    b = multiexit_loss(y, h[::-1], W[::-1], alpha_d=0.3, distill="js")
    np.testing.assert_allclose(a["ce_kd"], b["ce_kd"], rtol=1e-13)
    assert abs(a["J"][0].mean() - b["J"][0].mean()) > 1e-6    # each half is one-sided


def test_js_limits():
    # identical exits: zero divergence and no distillation gradient
    y, h, W = _rand_suite(M=2, T=6, D=(5, 5), V=12, seed=43)
    h[0], W[0] = h[1].copy(), W[1].copy()
    r = multiexit_loss(y, h, W, alpha_d=0.3, distill="js")
    np.testing.assert_allclose(r["ce_kd"], 0.0, atol=1e-14)
    c = multiexit_loss(y, h, W, alpha_d=0.0, distill="js")
    np.testing.assert_allclose(r["dh"][0], 0.7 * c["dh"][0], rtol=1e-12, atol=1e-15)
    # disjoint peaks: the divergence tends to log 2
    y = np.array([0])
    h = [np.array([[60.0]]), np.array([[60.0]])]
    W = [np.array([[1.0], [0.0]]), np.array([[0.0], [1.0]])]
    r = multiexit_loss(y, h, W, alpha_d=0.3, distill="js")
    np.testing.assert_allclose(r["ce_kd"][0], math.log(2.0), rtol=1e-12)


def test_js_two_class_closed_form():
    # student (b, 0), teacher (a, 0); mixture probabilities m1 = (s(a) + s(b)) / 2
    a, b = 1.5, -0.5
    y = np.array([1])
    h = [np.array([[b]]), np.array([[a]])]
    W = [np.array([[1.0], [0.0]]), np.array([[1.0], [0.0]])]
    r = multiexit_loss(y, h, W, alpha_d=0.3, distill="js")
    qa, qb = _sig(a), _sig(b)
    m1, m0 = 0.5 * (qa + qb), 0.5 * (2.0 - qa - qb)
    js = 0.5 * (qb * math.log(qb / m1) + (1 - qb) * math.log((1 - qb) / m0)
                + qa * math.log(qa / m1) + (1 - qa) * math.log((1 - qa) / m0))
    np.testing.assert_allclose(r["ce_kd"][0], js, rtol=1e-13)
    np.testing.assert_allclose(r["loss"], 0.7 * _softplus(b) + 0.3 * js + _softplus(a), rtol=1e-13)


def test_js_gradients_match_finite_differences():
    M, T, D, V, alpha = 3, 3, (3, 4, 5), 7, 0.45
    y, h, W = _rand_suite(M=M, T=T, D=D, V=V, seed=44, scale=2.0)
    lam = [1.4, 0.6, 0.9]
    r = multiexit_loss(y, h, W, alpha_d=alpha, grad_scale=0.8, distill="js", exit_weights=lam)
    eps = 1e-6
    for s in range(2):
        for arr, grad in ((h, r["dh"][s]), (W, r["dW"][s])):
            num = np.zeros_like(arr[s])
            for idx in np.ndindex(arr[s].shape):
                b = arr[s][idx]
                arr[s][idx] = b + eps
                lp = multiexit_loss(y, h, W, alpha_d=alpha, need_grad=False, distill="js", exit_weights=lam)["loss"]
                arr[s][idx] = b - eps
                lm = multiexit_loss(y, h, W, alpha_d=alpha, need_grad=False, distill="js", exit_weights=lam)["loss"]
                arr[s][idx] = b
                num[idx] = 0.8 * (lp - lm) / (2 * eps)
            np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-9)
    # the teacher is stop-gradient: its gradient is the plain cross-entropy one
    c = multiexit_loss(y, h, W, alpha_d=alpha, grad_scale=0.8, exit_weights=lam)
    np.testing.assert_allclose(r["dh"][2], c["dh"][2], rtol=1e-14, atol=1e-16)


# ------------------------------------------------------------------ teacher gradient (no stop-gradient)
@pytest.mark.parametrize("distill", ["ce", "reverse_kl", "js", "accept"])
def test_teacher_gradient_matches_finite_differences_of_the_whole_loss(distill):
    # Without the stop-gradient every parameter's gradient, the largest exit's
    # included, is the plain derivative of the total loss.
    M, T, D, V, alpha = 3, 3, (3, 4, 5), 7, 0.35
    y, h, W = _rand_suite(M=M, T=T, D=D, V=V, seed=51, scale=2.0)
    lam = [1.2, 0.7, 0.9]
    kw = dict(alpha_d=alpha, distill=distill, exit_weights=lam)
    r = multiexit_loss(y, h, W, grad_scale=1.1, teacher_grad=True, **kw)
    eps = 1e-6
    for m in range(M):
        for arr, grad in ((h, r["dh"][m]), (W, r["dW"][m])):
            num = np.zeros_like(arr[m])
            for idx in np.ndindex(arr[m].shape):
                b = arr[m][idx]
                arr[m][idx] = b + eps
                lp = multiexit_loss(y, h, W, need_grad=False, **kw)["loss"]
                arr[m][idx] = b - eps
                lm = multiexit_loss(y, h, W, need_grad=False, **kw)["loss"]
                arr[m][idx] = b
                num[idx] = 1.1 * (lp - lm) / (2 * eps)
            # central differences at eps = 1e-6 on a loss of order 10 carry about
            # 1e-16 * 10 / 1e-6 ~ 1e-9 of rounding error
            np.testing.assert_allclose(grad, num, rtol=1e-6, atol=5e-9)
    # the students' gradients do not depend on the option
    s = multiexit_loss(y, h, W, grad_scale=1.1, **kw)
    for m in range(M - 1):
        np.testing.assert_allclose(r["dh"][m], s["dh"][m], rtol=1e-14, atol=1e-16)
    # and at alpha_d = 0 the teacher's does not either
    a = multiexit_loss(y, h, W, alpha_d=0.0, distill=distill, exit_weights=lam, teacher_grad=True)
    b = multiexit_loss(y, h, W, alpha_d=0.0, distill=distill, exit_weights=lam)
    np.testing.assert_allclose(a["dh"][M - 1], b["dh"][M - 1], rtol=1e-14, atol=1e-16)


def test_teacher_gradient_of_identical_exits_ce():
    # Student equal to the teacher, cross-entropy form: KD = H(p), whose
    # derivative in l is -p (log p + H); the extra teacher term must equal it.
    y, h, W = _rand_suite(M=2, T=5, D=(6, 6), V=10, seed=52)
    h[0], W[0] = h[1].copy(), W[1].copy()
    a = multiexit_loss(y, h, W, alpha_d=0.4, teacher_grad=True)
    b = multiexit_loss(y, h, W, alpha_d=0.4)
    p = softmax_rows(h[1] @ W[1].T)
    H = -np.sum(p * np.log(p), axis=1)
    extra = 0.4 / 5 * (-p * (np.log(p) + H[:, None]))
    np.testing.assert_allclose(a["dh"][1] - b["dh"][1], extra @ W[1], rtol=1e-10, atol=1e-15)


# ------------------------------------------------------------------ acceptance loss
def test_acceptance_is_total_variation_written_out():
    # 1 - sum min(q, p) = (1/2) sum |q - p| (total variation), token by token
    y, h, W = _rand_suite(M=3, T=6, D=(3, 5, 8), V=11, seed=61, scale=2.5)
    r = multiexit_loss(y, h, W, alpha_d=0.3, distill="accept")
    pM = softmax_rows(h[2] @ W[2].T)
    for m in range(2):
        q = softmax_rows(h[m] @ W[m].T)
        tv = np.array([0.5 * sum(abs(q[t, v] - pM[t, v]) for v in range(11)) for t in range(6)])
        np.testing.assert_allclose(r["ce_kd"][m], tv.mean(), rtol=1e-12)
        # A = sum over q < p of q, B = sum over q >= p of p, beta = A + B
        a = np.array([sum(q[t, v] for v in range(11) if q[t, v] < pM[t, v]) for t in range(6)])
        np.testing.assert_allclose(r["A"][m], a, rtol=1e-12)
        np.testing.assert_allclose(1.0 - (r["A"][m] + r["B"][m]), tv, rtol=1e-10, atol=1e-15)


def test_acceptance_two_class_closed_form_and_limits():
    # student (b, 0), teacher (a, 0): beta = 1 - |s(a) - s(b)|
    a, b = 1.2, -0.7
    y = np.array([0])
    h = [np.array([[b]]), np.array([[a]])]
    W = [np.array([[1.0], [0.0]]), np.array([[1.0], [0.0]])]
    r = multiexit_loss(y, h, W, alpha_d=0.3, distill="accept")
    kd = abs(_sig(a) - _sig(b))
    np.testing.assert_allclose(r["ce_kd"][0], kd, rtol=1e-13)
    np.testing.assert_allclose(r["loss"], 0.7 * _softplus(-b) + 0.3 * kd + _softplus(-a), rtol=1e-13)
    # identical exits: beta = 1, no distillation gradient
    y, h, W = _rand_suite(M=2, T=5, D=(4, 4), V=9, seed=62)
    h[0], W[0] = h[1].copy(), W[1].copy()
    r = multiexit_loss(y, h, W, alpha_d=0.4, distill="accept")
    c = multiexit_loss(y, h, W, alpha_d=0.0, distill="accept")
    np.testing.assert_allclose(r["ce_kd"], 0.0, atol=1e-14)
    np.testing.assert_allclose(r["dh"][0], 0.6 * c["dh"][0], rtol=1e-12, atol=1e-15)


def test_acceptance_gradients_match_finite_differences():
    M, T, D, V, alpha = 3, 3, (3, 4, 5), 7, 0.45
    y, h, W = _rand_suite(M=M, T=T, D=D, V=V, seed=63, scale=2.0)
    lam = [1.3, 0.6, 0.9]
    kw = dict(alpha_d=alpha, distill="accept", exit_weights=lam)
    r = multiexit_loss(y, h, W, grad_scale=0.9, **kw)
    eps = 1e-6
    for s in range(2):
        for arr, grad in ((h, r["dh"][s]), (W, r["dW"][s])):
            num = np.zeros_like(arr[s])
            for idx in np.ndindex(arr[s].shape):
                b = arr[s][idx]
                arr[s][idx] = b + eps
                lp = multiexit_loss(y, h, W, need_grad=False, **kw)["loss"]
                arr[s][idx] = b - eps
                lm = multiexit_loss(y, h, W, need_grad=False, **kw)["loss"]
                arr[s][idx] = b
                num[idx] = 0.9 * (lp - lm) / (2 * eps)
            np.testing.assert_allclose(grad, num, rtol=1e-6, atol=5e-9)
