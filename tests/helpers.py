"""Comparison helpers and tolerances for the GPU-vs-oracle parity tests.

Tolerances (fixed by the method's problem statement for this path):
  * gather/copy/index results: bit-exact;
  * losses and per-token loss statistics: 2e-3 relative;
  * gradients: 1e-2 relative, per tensor in Frobenius norm, and per element as
    |g - g*| <= 1e-2 |g*| + 1e-2 rms(g*) (elementwise relative error alone is
    ill-posed near zero, hence the rms term);
  * the rescaled junction output, a stored activation, is the exact value
    rounded once to the storage dtype: |y - y*| <= u |y*| (1 + 1e-5) + tiny,
    u = 2^-8 for bf16 (unit roundoff of an 8-bit significand), 2^-23 for f32,
    plus the fp32 error of the scale (a few ulp).
"""
import json
import os

import numpy as np
import torch

LOSS_RTOL = 2e-3
GRAD_RTOL = 1e-2


def f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def unit_roundoff(dtype) -> float:
    return 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -23


def _log_grad_error(name, got, exp, rtol, rms, scale, nrm, err):
    """With MLS_GRAD_ERR_LOG set, appends one JSON line per compared tensor: the
    worst element's error as a fraction of the per-element bound (tensor-rms
    term, the one asserted) and of a looser bound with the rms of the
    element's row in place of the tensor's (recorded for comparison only),
    and the Frobenius error as a fraction of its bound; a value above 1
    fails that bound."""
    path = os.environ.get("MLS_GRAD_ERR_LOG")
    if not path or not exp.size:
        return
    d = np.abs(got - exp)
    rec = {
        "test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], "tensor": name,
        "shape": list(exp.shape), "rms": float(rms),
        "worst_abs": float(d.max()),
        "worst_frac_tensor_bound": float(np.max(d / (rtol * np.abs(exp) + rtol * rms + 1e-300))),
        "worst_frac_row_bound": float(np.max(d / (rtol * np.abs(exp) + rtol * scale + 1e-300))),
        "n_outside_tensor_bound": int(np.sum(d > rtol * np.abs(exp) + rtol * rms)),
        "frobenius_frac": float(err / (rtol * nrm + 1e-300)),
    }
    with open(path, "a") as f:
        f.write(json.dumps(rec) + "\n")


def assert_grad_close(got, exp, name="grad", rtol=GRAD_RTOL):
    got = f64(got)
    exp = f64(exp)
    assert got.shape == exp.shape, (name, got.shape, exp.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    nrm = np.linalg.norm(exp)
    err = np.linalg.norm(got - exp)
    rms = np.sqrt(np.mean(exp * exp)) if exp.size else 0.0
    scale = rms
    row_scale = rms
    if exp.ndim == 2 and exp.size:
        row_scale = np.maximum(np.sqrt(np.mean(exp * exp, axis=1, keepdims=True)), rms)
    _log_grad_error(name, got, exp, rtol, rms, row_scale, nrm, err)
    assert err <= rtol * nrm + 1e-30, f"{name}: Frobenius rel err {err / max(nrm, 1e-300):.3e} > {rtol}"
    bad = np.abs(got - exp) > rtol * np.abs(exp) + rtol * scale
    assert not bad.any(), (f"{name}: {int(bad.sum())} elements outside tolerance; worst "
                           f"{np.max(np.abs(got - exp)):.3e} (rms {rms:.3e})")


def assert_loss_close(got, exp, name="loss", rtol=LOSS_RTOL):
    got = f64(got)
    exp = f64(exp)
    assert got.shape == exp.shape, (name, got.shape, exp.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    rel = np.abs(got - exp) / np.maximum(np.abs(exp), 1e-30)
    assert np.all(rel <= rtol), f"{name}: max rel err {rel.max():.3e} > {rtol}"


def assert_stats_close(got, exp, name="stats", rtol=LOSS_RTOL, slack=None):
    """Per-token statistics (lse, target logit, teacher-weighted mean).

    Individual target logits and S values can sit near zero, so the bound is
    relative to the row's typical magnitude: |g - e| <= rtol (|e| + rms(row)).
    slack (same shape, optional) widens the bound element by element: the
    acceptance statistic sums q over the elements with q < p, a decision the
    GPU takes in fp32 and the oracle in fp64, so near-ties may fall on either
    side (see acceptance_tie_mass).
    """
    got = f64(got)
    exp = f64(exp)
    assert got.shape == exp.shape, (name, got.shape, exp.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    rms = np.sqrt(np.mean(exp * exp, axis=-1, keepdims=True))
    bound = rtol * (np.abs(exp) + rms)
    if slack is not None:
        bound = bound + slack
    bad = np.abs(got - exp) > bound
    assert not bad.any(), f"{name}: {int(bad.sum())} outside; worst {np.max(np.abs(got - exp)):.3e}"


def acceptance_tie_mass(y, h, W, eps=5e-4):
    """Per smaller exit and token, the probability mass whose side of the
    acceptance decision [q < p] rounding can flip: the sum of max(q_v, p_v)
    over the columns where |log q_v - log p_v| <= eps (q of the exit, p of the
    largest exit, fp64 from the same inputs).  An fp32 decision (logits from
    fp32 accumulation, errors around 1e-5 of their magnitude) agrees with the
    exact one outside that band.  Returns [M-1, T]."""
    M = len(h)
    hs = [f64(t) for t in h]
    Ws = [f64(t) for t in W]
    out = np.zeros((M - 1, hs[0].shape[0]))
    lM = hs[M - 1] @ Ws[M - 1].T
    lp = lM - (lM.max(1, keepdims=True) + np.log(np.exp(lM - lM.max(1, keepdims=True)).sum(1, keepdims=True)))
    for m in range(M - 1):
        lm = hs[m] @ Ws[m].T
        lq = lm - (lm.max(1, keepdims=True) + np.log(np.exp(lm - lm.max(1, keepdims=True)).sum(1, keepdims=True)))
        near = np.abs(lq - lp) <= eps
        out[m] = np.sum(np.where(near, np.exp(np.maximum(lq, lp)), 0.0), axis=1)
    return out
