"""Pins for the junction oracle against what the pages and the mathematics fix.

The junction rescales the block output to the norm of the fresh embedding and
concatenates the embedding after it, with no parameters ("Visualizing the
core idea of Matryoshka LM Suites", bottom panel: the junction; "Matryoshka
Language Model Suites", agihunt.info summary, junction paragraph).
"""
import numpy as np
import pytest

from oracle import junction_bwd, junction_fwd

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _case(T=17, D=12, dl=7, V=9, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.integers(0, V, size=T)
    o = rng.normal(0, 4.0, size=(T, D))
    E = rng.normal(0, 0.02, size=(V, dl))
    return x, o, E


def test_rescaled_part_has_embedding_norm():
    x, o, E = _case()
    y, s = junction_fwd(x, o, E)
    D = o.shape[1]
    n_scaled = np.linalg.norm(y[:, :D], axis=1)
    n_e = np.linalg.norm(E[x], axis=1)
    np.testing.assert_allclose(n_scaled, n_e, rtol=1e-12)


def test_rescaled_part_keeps_direction():
    x, o, E = _case(seed=1)
    y, _ = junction_fwd(x, o, E)
    D = o.shape[1]
    cos = np.sum(y[:, :D] * o, axis=1) / (np.linalg.norm(y[:, :D], axis=1) * np.linalg.norm(o, axis=1))
    np.testing.assert_allclose(cos, 1.0, rtol=0, atol=1e-12)


def test_embedding_fills_extra_channels_exactly():
    x, o, E = _case(seed=2)
    y, _ = junction_fwd(x, o, E)
    D = o.shape[1]
    assert y.shape == (x.shape[0], D + E.shape[1])
    assert np.array_equal(y[:, D:], E[x])


def test_no_parameters_and_scale_invariance():
    # The junction has no weight argument, and the output depends on o only
    # through its direction: y(c o) = y(o) for any c > 0.
    import inspect
    assert set(inspect.signature(junction_fwd).parameters) <= {"x", "o", "E", "variant"}
    x, o, E = _case(seed=3)
    y1, _ = junction_fwd(x, o, E)
    y2, _ = junction_fwd(x, 37.5 * o, E)
    np.testing.assert_allclose(y1, y2, rtol=1e-13, atol=0)


def test_scale_value_by_hand():
    # one token, o = (3, 4) (norm 5), e = (0.6, 0.8, 0) (norm 1) -> s = 1/5
    x = np.array([1])
    o = np.array([[3.0, 4.0]])
    E = np.array([[9.0, 9.0, 9.0], [0.6, 0.8, 0.0]])
    y, s = junction_fwd(x, o, E)
    np.testing.assert_allclose(s, [0.2], rtol=1e-15)
    np.testing.assert_allclose(y, [[0.6, 0.8, 0.6, 0.8, 0.0]], rtol=1e-15)


def test_degenerate_rows():
    x = np.array([0, 1])
    o = np.array([[0.0, 0.0], [1.0, -2.0]])
    E = np.array([[0.3, 0.4], [0.0, 0.0]])
    y, s = junction_fwd(x, o, E)
    assert np.all(y[0, :2] == 0.0)          # zero block output stays zero
    assert s[1] == 0.0 and np.all(y[1, :2] == 0.0)  # zero embedding -> scale 0
    dy = np.array([[1.0, 2.0, 3.0, 4.0], [0.5, -0.5, 0.25, 0.125]])
    do, de, dE = junction_bwd(x, o, E, dy)
    # zero embedding: de = g_e, do = 0
    np.testing.assert_array_equal(de[1], dy[1, 2:])
    np.testing.assert_array_equal(do[1], [0.0, 0.0])
    # zero block output: u = 0 so de = g_e and do = s g_o
    np.testing.assert_array_equal(de[0], dy[0, 2:])
    np.testing.assert_allclose(do[0], s[0] * dy[0, :2])


def _loss(x, o, E, R):
    y, _ = junction_fwd(x, o, E)
    return float(np.sum(y * R))


def test_backward_matches_finite_differences():
    x, o, E = _case(T=5, D=6, dl=4, V=3, seed=4)
    rng = np.random.default_rng(44)
    R = rng.normal(size=(5, 10))           # L = <y, R>  ->  dy = R
    do, de, dE = junction_bwd(x, o, E, R)
    h = 1e-6
    num_do = np.zeros_like(o)
    for i in range(o.shape[0]):
        for j in range(o.shape[1]):
            op = o.copy(); op[i, j] += h
            om = o.copy(); om[i, j] -= h
            num_do[i, j] = (_loss(x, op, E, R) - _loss(x, om, E, R)) / (2 * h)
    np.testing.assert_allclose(do, num_do, rtol=1e-6, atol=1e-9)
    num_dE = np.zeros_like(E)
    for i in range(E.shape[0]):
        for j in range(E.shape[1]):
            Ep = E.copy(); Ep[i, j] += h
            Em = E.copy(); Em[i, j] -= h
            num_dE[i, j] = (_loss(x, o, Ep, R) - _loss(x, o, Em, R)) / (2 * h)
    np.testing.assert_allclose(dE, num_dE, rtol=1e-6, atol=1e-9)


def test_backward_orthogonal_to_output():
    # Scale invariance in o implies o . do = 0 for every token.
    x, o, E = _case(T=33, D=16, dl=8, V=5, seed=5)
    dy = np.random.default_rng(55).normal(size=(33, 24))
    do, _, _ = junction_bwd(x, o, E, dy)
    dots = np.sum(o * do, axis=1) / (np.linalg.norm(o, axis=1) * np.linalg.norm(do, axis=1))
    np.testing.assert_allclose(dots, 0.0, atol=1e-12)


def test_table_gradient_is_one_hot_product():
    # dE = onehot(x)^T de, built here with a dense indicator matrix.
    x, o, E = _case(T=40, D=8, dl=6, V=7, seed=6)
    dy = np.random.default_rng(66).normal(size=(40, 14))
    _, de, dE = junction_bwd(x, o, E, dy)
    P = np.zeros((40, 7))
    P[np.arange(40), x] = 1.0
    np.testing.assert_allclose(dE, P.T @ de, rtol=1e-13, atol=1e-15)
    # tokens that never occur get exactly zero
    unused = np.setdiff1d(np.arange(7), x)
    assert np.all(dE[unused] == 0.0)


# ------------------------------------------------------------------ variants
from oracle import junction_variants as jv  # noqa: E402


def _fd_check(x, o, E, R, variant, wrt_o=True):
    do, de, dE = junction_bwd(x, o, E, R, variant=variant)
    h = 1e-6

    def L(oo, EE):
        y, _ = junction_fwd(x, oo, EE, variant=variant)
        return float(np.sum(y * R))
    num_dE = np.zeros_like(E)
    for idx in np.ndindex(E.shape):
        Ep = E.copy(); Ep[idx] += h
        Em = E.copy(); Em[idx] -= h
        num_dE[idx] = (L(o, Ep) - L(o, Em)) / (2 * h)
    np.testing.assert_allclose(dE, num_dE, rtol=1e-6, atol=1e-9)
    if wrt_o:
        num_do = np.zeros_like(o)
        for idx in np.ndindex(o.shape):
            op = o.copy(); op[idx] += h
            om = o.copy(); om[idx] -= h
            num_do[idx] = (L(op, E) - L(om, E)) / (2 * h)
        np.testing.assert_allclose(do, num_do, rtol=1e-6, atol=1e-9)
    return do, de, dE


def test_variant_no_rescale_is_plain_concatenation():
    x, o, E = _case(T=6, D=5, dl=3, V=4, seed=11)
    y, s = junction_fwd(x, o, E, variant=jv.NO_RESCALE)
    assert np.array_equal(y, np.concatenate([o, E[x]], axis=1)) and np.all(s == 1.0)
    R = np.random.default_rng(1).normal(size=(6, 8))
    do, de, _ = _fd_check(x, o, E, R, jv.NO_RESCALE)
    np.testing.assert_array_equal(do, R[:, :5])
    np.testing.assert_array_equal(de, R[:, 5:])


def test_variant_zero_fill_keeps_the_rescale():
    x, o, E = _case(T=6, D=5, dl=3, V=4, seed=12)
    y, s = junction_fwd(x, o, E, variant=jv.ZERO_FILL)
    assert np.all(y[:, 5:] == 0.0)
    np.testing.assert_allclose(np.linalg.norm(y[:, :5], axis=1), np.linalg.norm(E[x], axis=1), rtol=1e-12)
    R = np.random.default_rng(2).normal(size=(6, 8))
    _fd_check(x, o, E, R, jv.ZERO_FILL)


def test_variant_zero_fill_without_rescale():
    x, o, E = _case(T=4, D=3, dl=2, V=3, seed=13)
    y, _ = junction_fwd(x, o, E, variant=jv.NO_RESCALE | jv.ZERO_FILL)
    assert np.array_equal(y, np.concatenate([o, np.zeros((4, 2))], axis=1))
    do, de, dE = junction_bwd(x, o, E, np.ones((4, 5)), variant=jv.NO_RESCALE | jv.ZERO_FILL)
    assert np.all(do == 1.0) and np.all(de == 0.0) and np.all(dE == 0.0)


def test_variant_stop_gradient():
    x, o, E = _case(T=6, D=5, dl=3, V=4, seed=14)
    y0, _ = junction_fwd(x, o, E)
    y1, _ = junction_fwd(x, o, E, variant=jv.STOP_GRAD)
    assert np.array_equal(y0, y1)                      # forward unchanged
    R = np.random.default_rng(3).normal(size=(6, 8))
    do, de, dE = _fd_check(x, o, E, R, jv.STOP_GRAD, wrt_o=False)   # embedding gradient = true derivative
    assert np.all(do == 0.0)                           # nothing flows back into the block output
    _, de0, _ = junction_bwd(x, o, E, R)
    np.testing.assert_array_equal(de, de0)
