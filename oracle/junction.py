"""Oracle for the parameter-free junction between block m and block m+1.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Definition followed.  "Visualizing the core idea of Matryoshka LM Suites"
(How to read it, bottom panel: the junction) and "Matryoshka Language Model
Suites" (agihunt.info summary, junction paragraph): the output of block m is
rescaled to the L2 norm of the next block's fresh residual embedding of the
same token, then concatenated with that embedding along channels; the
embedding fills the D_{m+1} - D_m extra channels and nothing is learned.
"Editing the methods of sub-models are made of blocks" (Modeling paragraph,
after version): the residual table e_{m+1} has width D_{m+1} - D_m and is
applied to the original token ids x.

Readings where the pages are silent (each is listed in the design notes):
  * the norm is per token, over channels;
  * the rescaled block output comes first and the embedding second;
  * s = ||e|| / max(||o||, 1e-12); in the backward pass e_hat := 0 when ||e|| = 0.

Variants (bit flags, combinable), after the pages' two negative controls of
the junction ("Visualizing Core ideas", bullet (c): dropping the rescaling,
and filling the new channels with zeros instead of the fresh embedding) and
the stop-gradient follow-up ("Is nesting the cheapest way to build a model
suite?", section 5 (B): each block learns only from its own exit):
  * NO_RESCALE: s := 1, so y = [o ; e];
  * ZERO_FILL: the new channels are zeros, y = [s o ; 0]; the rescale still
    uses the fresh embedding's norm (only the fill changes);
  * STOP_GRAD: the forward pass is unchanged; no gradient flows back into the
    block output (do = 0); the embedding keeps its gradient.

The backward pass is derived by hand from the forward definition (the pages
give no gradient): with u = o/||o||, e_hat = e/||e||, s = ||e||/||o|| and the
incoming gradient split as dy = [g_o ; g_e],
    do = s * (g_o - u (u . g_o))
    de = g_e + (u . g_o) e_hat
and the table gradient dE[v] is the sum of de over tokens with x_t = v, taken
in ascending t.
"""
from __future__ import annotations

import numpy as np

JUNCTION_EPS = 1e-12
STANDARD = 0
NO_RESCALE = 1
ZERO_FILL = 2
STOP_GRAD = 4


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        import torch
        return a.detach().to(torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


def junction_fwd(x, o, E, variant=STANDARD):
    """y_t = [ s_t * o_t ; E[x_t] ],  s_t = ||E[x_t]||_2 / max(||o_t||_2, eps).

    x: int [T]; o: [T, D]; E: [V, delta].  Returns (y [T, D+delta] fp64, s [T] fp64).
    """
    x = np.asarray(x, dtype=np.int64)
    o = _f64(o)
    e = _f64(E)[x]
    n_o = np.sqrt(np.sum(o * o, axis=1))
    n_e = np.sqrt(np.sum(e * e, axis=1))
    s = n_e / np.maximum(n_o, JUNCTION_EPS)
    if variant & NO_RESCALE:
        s = np.ones_like(s)
    fill = np.zeros_like(e) if variant & ZERO_FILL else e
    y = np.concatenate([s[:, None] * o, fill], axis=1)
    return y, s


def junction_bwd(x, o, E, dy, V=None, variant=STANDARD):
    """Gradients of the junction.  Returns (do [T,D], de [T,delta], dE [V,delta]), fp64."""
    x = np.asarray(x, dtype=np.int64)
    o = _f64(o)
    Ef = _f64(E)
    e = Ef[x]
    dy = _f64(dy)
    D = o.shape[1]
    g_o, g_e = dy[:, :D], dy[:, D:]
    n_o = np.sqrt(np.sum(o * o, axis=1))
    n_e = np.sqrt(np.sum(e * e, axis=1))
    n_o_c = np.maximum(n_o, JUNCTION_EPS)
    s = n_e / n_o_c
    u = o / n_o_c[:, None]
    e_hat = np.where(n_e[:, None] > 0, e / np.where(n_e > 0, n_e, 1.0)[:, None], 0.0)
    ug = np.sum(u * g_o, axis=1)
    if variant & NO_RESCALE:
        do = g_o.copy()                       # y = [o ; .]: identity on the block output
        de_s = np.zeros_like(e)               # s no longer depends on e
    else:
        do = s[:, None] * (g_o - u * ug[:, None])
        de_s = ug[:, None] * e_hat
    de = de_s if variant & ZERO_FILL else g_e + de_s
    if variant & STOP_GRAD:
        do = np.zeros_like(do)
    Vn = Ef.shape[0] if V is None else V
    dE = np.zeros((Vn, e.shape[1]), dtype=np.float64)
    for t in range(x.shape[0]):          # ascending t, one row at a time
        dE[x[t]] += de[t]
    return do, de, dE
