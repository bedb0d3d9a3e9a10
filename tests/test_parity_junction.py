"""GPU junction (forward, backward, table scatter) against the fp64 oracle.

All calls go through the C ABI (libmls) via the package binding.
"""
import numpy as np
import pytest
import torch

import oracle
from lm_head_loss_junction_b200 import junction_bwd, junction_fwd, new_status, status_read
from lm_head_loss_junction_b200 import workloads as wl
from tests.helpers import assert_grad_close, f64, unit_roundoff

pytestmark = pytest.mark.gpu


def _junction_case(cfg, j):
    """Inputs of junction j -> j+1 of a workload, on the GPU."""
    d = wl.make_inputs(cfg, with_heads=False)
    x = torch.from_numpy(d.x).cuda()
    o = d.o[j].cuda()
    E = d.E[j + 1].cuda()
    dy = wl.make_grad(cfg, j).cuda()
    return d, x, o, E, dy


def _check_fwd(x, o, E, y, s):
    y_exp, s_exp = oracle.junction_fwd(x.cpu().numpy(), o.cpu(), E.cpu())
    D = o.shape[1]
    # the embedding part is a bit-exact copy of the gathered table rows
    assert torch.equal(y[:, D:].cpu(), E.cpu()[x.cpu().long()])
    np.testing.assert_allclose(f64(s), s_exp, rtol=2e-6)
    u = unit_roundoff(o.dtype)
    got = f64(y[:, :D])
    exp = y_exp[:, :D]
    bound = u * np.abs(exp) * (1 + 1e-5) + 4e-6 * np.abs(exp) + 1e-30
    bad = np.abs(got - exp) > bound
    assert not bad.any(), f"{int(bad.sum())} scaled elements off; worst {np.max(np.abs(got - exp) - bound):.3e}"
    # invariant: the scaled part has the embedding's norm
    n_scaled = np.linalg.norm(got, axis=1)
    n_e = np.linalg.norm(f64(E)[x.cpu().numpy()], axis=1)
    np.testing.assert_allclose(n_scaled, n_e, rtol=4 * u + 1e-5)


SMALL = [
    ("tiny3", 0, None),
    ("tiny3", 1, None),
    ("main3", 0, dict(batch=1, seq=300, V=512)),
    ("main3", 1, dict(batch=1, seq=300, V=512)),
    ("proxy2", 0, dict(batch=2, seq=97, V=256)),
    ("suite4", 0, dict(batch=1, seq=129, V=300)),
    ("suite4", 2, dict(batch=1, seq=129, V=300)),
]


def _cfg(name, small):
    cfg = wl.CONFIGS[name]
    return cfg if small is None else wl.small_variant(cfg, **small)


@pytest.mark.parametrize("name,j,small", SMALL)
def test_junction_fwd_matches_oracle(name, j, small):
    cfg = _cfg(name, small)
    _, x, o, E, _ = _junction_case(cfg, j)
    s = torch.empty(x.shape[0], dtype=torch.float32, device="cuda")
    st = new_status()
    y = junction_fwd(x, o, E, scale_out=s, status=st)
    assert status_read(st) == (0, 0)
    _check_fwd(x, o, E, y, s)


@pytest.mark.parametrize("name,j,small", SMALL)
def test_junction_bwd_matches_oracle(name, j, small):
    cfg = _cfg(name, small)
    _, x, o, E, dy = _junction_case(cfg, j)
    dE = torch.full(E.shape, 7.0, dtype=torch.float32, device="cuda")   # overwritten
    do, de, dE = junction_bwd(x, o, E, dy, dE=dE)
    do_e, de_e, dE_e = oracle.junction_bwd(x.cpu().numpy(), o.cpu(), E.cpu(), dy.cpu())
    assert_grad_close(do, do_e, "do")
    assert_grad_close(de, de_e, "de")
    assert_grad_close(dE, dE_e, "dE")
    # o . do = 0 for every token (scale invariance), up to rounding
    dots = np.sum(f64(o) * do_e, axis=1)
    assert np.max(np.abs(dots)) < 1e-9 * np.max(np.abs(f64(o))) * np.max(np.abs(do_e)) * o.shape[1]


def test_table_gradient_accumulates_and_is_deterministic():
    cfg = wl.small_variant(wl.CONFIGS["main3"], batch=2, seq=700, V=64)   # many repeats per id
    _, x, o, E, dy = _junction_case(cfg, 0)
    base = torch.randn(E.shape, dtype=torch.float32, device="cuda")
    dE1 = base.clone()
    junction_bwd(x, o, E, dy, want_de_rows=False, dE=dE1, accumulate_dE=True)
    dE2 = base.clone()
    junction_bwd(x, o, E, dy, want_de_rows=False, dE=dE2, accumulate_dE=True)
    assert torch.equal(dE1, dE2), "table scatter must be deterministic"
    _, _, dE_e = oracle.junction_bwd(x.cpu().numpy(), o.cpu(), E.cpu(), dy.cpu())
    assert_grad_close(dE1 - base, dE_e, "dE accumulated")


def test_bad_ids_are_flagged_and_zeroed():
    cfg = wl.small_variant(wl.CONFIGS["proxy2"], batch=1, seq=64, V=128)
    _, x, o, E, dy = _junction_case(cfg, 0)
    x = x.clone()
    x[5] = -1
    x[9] = cfg.V
    st = new_status()
    y = junction_fwd(x, o, E, status=st)
    code, word = status_read(st)
    assert word & 1 and code == 5
    assert torch.all(y[5] == 0) and torch.all(y[9] == 0)
    good = torch.ones(x.shape[0], dtype=torch.bool)
    good[[5, 9]] = False
    xe = x.cpu().numpy().copy()
    xe[~good.numpy()] = 0
    y_exp, _ = oracle.junction_fwd(xe, o.cpu(), E.cpu())
    D = o.shape[1]
    assert torch.equal(y[good.cuda(), D:].cpu(), torch.from_numpy(y_exp[good.numpy(), D:]).to(o.dtype))
    dE = torch.zeros(E.shape, dtype=torch.float32, device="cuda")
    do, de, dE = junction_bwd(x, o, E, dy, dE=dE, status=st)
    code, word = status_read(st)
    assert code == 5
    assert torch.all(do[5] == 0) and torch.all(de[9] == 0)


@pytest.mark.parametrize("name", ["main3", "suite4", "proxy2", "main3_aligned"])
def test_junction_full_size_sampled(name):
    """Full-size junctions in the benchmark's launch configuration, checked on
    sampled tokens against the oracle and on the bit-exact copy everywhere."""
    cfg = wl.CONFIGS[name]
    d = wl.make_inputs(cfg, with_heads=False)
    x = torch.from_numpy(d.x).cuda()
    rng = np.random.default_rng(123)
    rows = np.sort(rng.choice(cfg.T, size=256, replace=False))
    for j in range(cfg.M - 1):
        o = d.o[j].cuda()
        E = d.E[j + 1].cuda()
        s = torch.empty(cfg.T, dtype=torch.float32, device="cuda")
        y = junction_fwd(x, o, E, scale_out=s)
        D = o.shape[1]
        assert torch.equal(y[:, D:], E[x.long()])
        sel = torch.from_numpy(rows).cuda()
        _check_fwd(x[sel], o[sel], E, y[sel], s[sel])
        dy = wl.make_grad(cfg, j).cuda()
        do, de, _ = junction_bwd(x, o, E, dy)
        do_e, de_e, _ = oracle.junction_bwd(d.x[rows], d.o[j][rows], d.E[j + 1], dy.cpu()[rows])
        assert_grad_close(do[sel], do_e, "do")
        assert_grad_close(de[sel], de_e, "de")


VARIANTS = [1, 2, 4, 3, 5, 6, 7]   # no rescale, zero fill, stop-gradient and their combinations


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("name,j,small", [("main3", 1, dict(batch=1, seq=300, V=512)),    # long rows
                                          ("main3", 0, dict(batch=1, seq=300, V=512)),    # prefetching forward
                                          ("proxy2", 0, dict(batch=1, seq=300, V=256)),   # prefetching both ways
                                          ("tiny3", 0, None)])
def test_junction_variants_match_oracle(variant, name, j, small):
    cfg = _cfg(name, small)
    _, x, o, E, dy = _junction_case(cfg, j)
    s = torch.empty(x.shape[0], dtype=torch.float32, device="cuda")
    y = junction_fwd(x, o, E, scale_out=s, variant=variant)
    y_e, s_e = oracle.junction_fwd(x.cpu().numpy(), o.cpu(), E.cpu(), variant=variant)
    D = o.shape[1]
    # the filled channels are an exact copy (or exact zeros)
    assert torch.equal(y[:, D:].cpu(), torch.from_numpy(y_e[:, D:]).to(o.dtype))
    np.testing.assert_allclose(f64(s), s_e, rtol=2e-6)
    u = unit_roundoff(o.dtype)
    got, exp = f64(y[:, :D]), y_e[:, :D]
    assert np.all(np.abs(got - exp) <= u * np.abs(exp) * (1 + 1e-5) + 4e-6 * np.abs(exp) + 1e-30)
    dE = torch.zeros(E.shape, dtype=torch.float32, device="cuda")
    do, de, dE = junction_bwd(x, o, E, dy, dE=dE, variant=variant)
    do_e, de_e, dE_e = oracle.junction_bwd(x.cpu().numpy(), o.cpu(), E.cpu(), dy.cpu(), variant=variant)
    if variant & 4:
        assert torch.all(do == 0)
    else:
        assert_grad_close(do, do_e, "do")
    if (variant & 3) == 3:
        assert torch.all(de == 0) and torch.all(dE == 0)
    else:
        assert_grad_close(de, de_e, "de")
        assert_grad_close(dE, dE_e, "dE")
