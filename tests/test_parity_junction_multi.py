"""Every junction of a suite in one call (mls_junction_fwd_multi / _bwd_multi).

The multi calls run the same per-token arithmetic as the single calls (one
launch whose blocks are split among the junctions; one id grouping shared by
all table gradients), so their results must equal J single calls bit for bit;
the single calls are checked against the fp64 oracle in
test_parity_junction.py, and the multi results are checked against it here
too.  All calls go through the C ABI.
"""
import numpy as np
import pytest
import torch

import oracle
from lm_head_loss_junction_b200 import (junction_bwd, junction_bwd_multi, junction_fwd, junction_fwd_multi,
                                        new_status, status_read)
from lm_head_loss_junction_b200 import workloads as wl
from tests.helpers import assert_grad_close

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny3", None),                                   # fp32: one launch per junction
    ("proxy2", dict(batch=2, seq=97, V=256)),          # one junction, prefetching body
    ("main3", dict(batch=1, seq=300, V=512)),          # prefetching + whole-row bodies
    ("suite4", dict(batch=1, seq=129, V=300)),         # three junctions
    ("main3", None),                                   # full size, Zipf ids
]


def _inputs(name, small):
    cfg = wl.CONFIGS[name] if small is None else wl.small_variant(wl.CONFIGS[name], **small)
    d = wl.make_inputs(cfg, with_heads=False)
    x = torch.from_numpy(d.x).cuda()
    J = cfg.M - 1
    o = [d.o[j].cuda() for j in range(J)]
    E = [d.E[j + 1].cuda() for j in range(J)]
    dy = [wl.make_grad(cfg, j).cuda() for j in range(J)]
    return cfg, d, x, o, E, dy


@pytest.mark.parametrize("name,small", CASES)
def test_fwd_multi_equals_single_calls(name, small):
    cfg, d, x, o, E, _ = _inputs(name, small)
    J = len(o)
    st = new_status()
    s_multi = [torch.full((cfg.T,), -1.0, device="cuda") for _ in range(J)]
    y_multi = junction_fwd_multi(x, o, E, scale_out=s_multi, status=st)
    for j in range(J):
        s1 = torch.empty(cfg.T, device="cuda")
        y1 = junction_fwd(x, o[j], E[j], scale_out=s1, status=st)
        assert torch.equal(y_multi[j], y1), f"junction {j}: y"
        assert torch.equal(s_multi[j], s1), f"junction {j}: scale"
    assert status_read(st) == (0, 0)
    if small is not None:
        for j in range(J):
            y_exp, _ = oracle.junction_fwd(d.x, d.o[j], d.E[j + 1])
            np.testing.assert_allclose(y_multi[j].double().cpu().numpy(), y_exp, rtol=2 ** -7, atol=1e-30)


@pytest.mark.parametrize("name,small", CASES)
@pytest.mark.parametrize("accumulate", [False, True])
def test_bwd_multi_equals_single_calls(name, small, accumulate):
    cfg, d, x, o, E, dy = _inputs(name, small)
    J = len(o)
    st = new_status()
    base = [torch.randn(e.shape, dtype=torch.float32, device="cuda") for e in E]
    dE_multi = [b.clone() for b in base]
    # the last junction's de rows are not asked for
    de_out = [torch.empty((cfg.T, e.shape[1]), dtype=e.dtype, device="cuda") for e in E[:-1]] + [None]
    do_m, de_m, _ = junction_bwd_multi(x, o, E, dy, de_out=de_out, dE=dE_multi, accumulate_dE=accumulate, status=st)
    for j in range(J):
        dE1 = base[j].clone()
        do1, de1, _ = junction_bwd(x, o[j], E[j], dy[j], dE=dE1, accumulate_dE=accumulate, status=st)
        assert torch.equal(do_m[j], do1), f"junction {j}: do"
        if de_m[j] is not None:
            assert torch.equal(de_m[j], de1), f"junction {j}: de"
        assert torch.equal(dE_multi[j], dE1), f"junction {j}: dE"
    assert status_read(st) == (0, 0)
    if small is not None:
        for j in range(J):
            do_e, _, dE_e = oracle.junction_bwd(d.x, d.o[j], d.E[j + 1], dy[j].cpu())
            assert_grad_close(do_m[j], do_e, f"do[{j}]")
            exp = dE_e + (base[j].double().cpu().numpy() if accumulate else 0.0)
            assert_grad_close(dE_multi[j], exp, f"dE[{j}]")


def test_bwd_multi_without_tables_needs_no_workspace():
    cfg, d, x, o, E, dy = _inputs("main3", dict(batch=1, seq=200, V=256))
    do_m, de_m, dE_m = junction_bwd_multi(x, o, E, dy)
    assert all(t is None for t in dE_m)
    for j in range(len(o)):
        do1, _, _ = junction_bwd(x, o[j], E[j], dy[j])
        assert torch.equal(do_m[j], do1)


def test_multi_bad_ids_are_flagged():
    cfg, d, x, o, E, dy = _inputs("suite4", dict(batch=1, seq=129, V=300))
    x = x.clone()
    x[5] = -1
    x[100] = cfg.V
    st = new_status()
    y = junction_fwd_multi(x, o, E, status=st)
    code, word = status_read(st)
    assert code == 5 and word & 1
    for j in range(len(o)):
        assert torch.all(y[j][5] == 0) and torch.all(y[j][100] == 0)
    dE = [torch.zeros(e.shape, dtype=torch.float32, device="cuda") for e in E]
    junction_bwd_multi(x, o, E, dy, dE=dE, status=st)
    assert status_read(st)[0] == 5
    for t in dE:
        assert torch.isfinite(t).all()
