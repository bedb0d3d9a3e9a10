"""Oracle for the multi-exit LM-head loss with online distillation.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Definition followed.
  * Logits per exit: l_m = W^m h_m with W^m in R^{V x D_m} ("Editing the methods
    of sub-models are made of blocks", Modeling paragraph: every sub-model ends
    in its own LM head; h_m is the block-m output o_m).
  * Next-token cross-entropy at every exit (same paragraph).
  * Distillation: the largest exit's softmax is the teacher and every smaller
    exit gets a token-level cross-entropy against it, mixed with its own LM loss
    with weight alpha_d ("Matryoshka Language Model Suites", agihunt.info
    summary, distillation paragraph); the mix is (1 - alpha_d) next-token loss
    + alpha_d cross-entropy to the largest exit ("Is nesting the cheapest way to
    build a model suite?", section 4: 0.7 and 0.3 at alpha_d = 0.3); the
    distillation term exists only for the smaller exits ("Visualizing Core
    ideas", bullet (b)).
  * Per-exit losses are summed with equal weight ("Matryoshka Language Model
    Suites", limitations paragraph).

Readings where the pages are silent: the teacher is stop-gradient; the
distillation temperature is 1; every term is a mean over the T tokens;
``grad_scale`` multiplies dL (so a caller can fold in a global token count).

    CE_LM,m = mean_t ( lse(l_{m,t}) - l_{m,t,y_t} )
    CE_KD,m = mean_t ( - sum_v p_{M,t,v} log q_{m,t,v} ),  m < M
    L = sum_{m<M} [ (1 - alpha_d) CE_LM,m + alpha_d CE_KD,m ] + CE_LM,M

Backward (derived by hand; the pages give no gradient), with q_m = softmax(l_m):
    G_m = grad_scale/T * (q_m - (1 - alpha_d) onehot(y) - alpha_d p_M),  m < M
    G_M = grad_scale/T * (q_M - onehot(y))
    dh_m = G_m W^m,     dW^m = G_m^T h_m

Tokens are independent, so the token loop below processes a block of rows at
a time only to bound memory; each block is the plain definition.
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        import torch
        return a.detach().to(torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


def logsumexp_rows(l: np.ndarray) -> np.ndarray:
    """log sum_v exp(l[t, v]) per row, with the row max factored out."""
    mx = np.max(l, axis=1)
    return mx + np.log(np.sum(np.exp(l - mx[:, None]), axis=1))


def softmax_rows(l: np.ndarray) -> np.ndarray:
    return np.exp(l - logsumexp_rows(l)[:, None])


def multiexit_loss(y, h, W, alpha_d=0.3, grad_scale=1.0, need_grad=True,
                   rows=None, token_block=256, exit_weights=None, distill="ce", teacher_grad=False):
    """Multi-exit loss, per-token statistics and (optionally) gradients, fp64.

    y: int [T] targets; h: list of M arrays [T, D_m]; W: list of M arrays [V, D_m].
    rows: optional int array of token indices; when given, only those tokens are
    evaluated (their per-token statistics and dh rows; the means and dW are then
    over the selected tokens, normalised by the full T).
    exit_weights: optional per-exit weights lambda_m (default 1 each: "summed
    with equal weight"; "Matryoshka Language Model Suites", limitations
    paragraph, notes that reweighting the exits closes much of the gap):
    L = sum_{m<M} lambda_m [(1 - alpha_d) CE_LM,m + alpha_d CE_KD,m] + lambda_M CE_LM,M,
    and each exit's gradient is scaled by its lambda_m.
    distill: "ce" (the pages' token-level cross-entropy to the largest exit) or
    "reverse_kl", the alternative distillation term the follow-ups propose to
    swap in ("Is nesting the cheapest way to build a model suite?", section 4):
    KD_m = mean_t KL(q_m || p_M) = mean_t sum_v q_m,v (log q_m,v - log p_M,v).
    Its student gradient (teacher still stop-gradient) is
    G_m = lambda_m grad_scale/T ((1 - alpha_d)(q_m - onehot) + alpha_d q_m (log q_m - log p_M - KL_t)),
    and the per-token statistic returned in "R" is sum_v q_m,v (l_m,v - l_M,v).
    distill="js" takes the Jensen-Shannon divergence, the other alternative the
    same section names:  with the mixture mu = (q_m + p_M) / 2,
    KD_m = mean_t [ KL(q_m || mu) + KL(p_M || mu) ] / 2   (natural log, <= log 2).
    Since d JS / d q_v = log(q_v / mu_v) / 2 (the other terms cancel), the
    student gradient through the softmax is
    G_m = lambda_m grad_scale/T ((1 - alpha_d)(q_m - onehot) + alpha_d q_m (g - K_t)),
    g_v = log(q_v / mu_v) / 2,  K_t = sum_v q_v g_v = KL(q_m || mu) / 2,
    and K_t is returned per token in "J" (KL(p_M || mu)/2 in "Jp").
    distill="accept" takes the acceptance loss the same section lists: train
    the draft for the probability that its sampled token is accepted,
    beta = sum_v min(q_v, p_v), i.e. KD_m = mean_t (1 - beta_t), the total
    variation distance.  Its student (sub)gradient, with the indicator of
    q_v < p_v taken strictly, is
    G_m = lambda_m grad_scale/T ((1 - alpha_d)(q_m - onehot) + alpha_d q_m (A_t - [q < p])),
    A_t = sum_{v: q_v < p_v} q_v, returned per token in "A" (and
    B_t = beta_t - A_t = sum_{v: q_v >= p_v} p_v in "B").
    teacher_grad: the largest exit also receives the gradient of every
    distillation term (no stop-gradient; the pages leave this open).  With
    T_m = d KD_m / d l_M, the teacher's logit gradient gains
    lambda_m alpha_d T_m per smaller exit m, where
      cross-entropy:  T_m = -p_M (l_m - S_m)           (S_m = sum_v p_M l_m)
      reverse KL:     T_m = p_M - q_m
      Jensen-Shannon: T_m = p_M (log(p_M / mu) / 2 - KL(p_M || mu) / 2)
      acceptance:     T_m = p_M (B_t - [q_m >= p_M]).

    Returns a dict with
      ce_lm [M], ce_kd [M-1], loss (scalar)         -- means over the tokens
      lse [M, T'], tgt [M, T'], S [M-1, T']          -- per-token statistics,
          S_m,t = sum_v p_{M,t,v} l_{m,t,v}  (R and J as above, for every distill)
      dh (list of [T', D_m]) and dW (list of [V, D_m]) when need_grad.
    """
    y = np.asarray(y, dtype=np.int64)
    M = len(h)
    T = y.shape[0]
    idx = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    Tn = idx.shape[0]
    Ws = [_f64(w) for w in W]
    V = Ws[0].shape[0]
    if distill not in ("ce", "reverse_kl", "js", "accept"):
        raise ValueError(distill)
    out = {
        "lse": np.zeros((M, Tn)), "tgt": np.zeros((M, Tn)), "S": np.zeros((max(M - 1, 0), Tn)),
        "R": np.zeros((max(M - 1, 0), Tn)), "J": np.zeros((max(M - 1, 0), Tn)),
        "Jp": np.zeros((max(M - 1, 0), Tn)), "A": np.zeros((max(M - 1, 0), Tn)),
        "B": np.zeros((max(M - 1, 0), Tn)),
        "ce_lm_sum": np.zeros(M), "ce_kd_sum": np.zeros(max(M - 1, 0)),
    }
    if need_grad:
        out["dh"] = [np.zeros((Tn, w.shape[1])) for w in Ws]
        out["dW"] = [np.zeros_like(w) for w in Ws]
    lam = np.ones(M) if exit_weights is None else np.asarray(exit_weights, dtype=np.float64)
    g = grad_scale / T
    for b0 in range(0, Tn, token_block):
        sel = idx[b0:b0 + token_block]
        n = sel.shape[0]
        yb = y[sel]
        hb = [_f64(hm[sel]) for hm in h]
        logits = [hb[m] @ Ws[m].T for m in range(M)]           # [n, V] each
        lse = [logsumexp_rows(l) for l in logits]
        logq = [logits[m] - lse[m][:, None] for m in range(M)]
        pM = np.exp(logq[M - 1])                                # teacher softmax
        ar = np.arange(n)
        for m in range(M):
            out["lse"][m, b0:b0 + n] = lse[m]
            out["tgt"][m, b0:b0 + n] = logits[m][ar, yb]
            out["ce_lm_sum"][m] += np.sum(lse[m] - logits[m][ar, yb])
        rkl, logmix, jq, jps, accA, accB = [], [], [], [], [], []
        for m in range(M - 1):
            out["S"][m, b0:b0 + n] = np.sum(pM * logits[m], axis=1)
            q = np.exp(logq[m])
            out["R"][m, b0:b0 + n] = np.sum(q * (logits[m] - logits[M - 1]), axis=1)
            rkl.append(np.sum(q * (logq[m] - logq[M - 1]), axis=1))
            # Jensen-Shannon: log of the mixture (q + p)/2, and KL of each side against it
            logmix.append(np.logaddexp(logq[m], logq[M - 1]) - np.log(2.0))
            jq.append(np.sum(q * (logq[m] - logmix[m]), axis=1))
            jp = np.sum(pM * (logq[M - 1] - logmix[m]), axis=1)
            jps.append(jp)
            out["J"][m, b0:b0 + n] = 0.5 * jq[m]
            out["Jp"][m, b0:b0 + n] = 0.5 * jp
            # acceptance: beta = sum min(q, p) = A + B with A over q < p, B over q >= p
            below = q < pM
            accA.append(np.sum(np.where(below, q, 0.0), axis=1))
            accB.append(np.sum(np.where(below, 0.0, pM), axis=1))
            out["A"][m, b0:b0 + n] = accA[m]
            out["B"][m, b0:b0 + n] = accB[m]
            if distill == "ce":
                out["ce_kd_sum"][m] += np.sum(-np.sum(pM * logq[m], axis=1))
            elif distill == "reverse_kl":
                out["ce_kd_sum"][m] += np.sum(rkl[m])
            elif distill == "js":
                out["ce_kd_sum"][m] += np.sum(0.5 * (jq[m] + jp))
            else:
                out["ce_kd_sum"][m] += np.sum(1.0 - (accA[m] + accB[m]))
        if need_grad:
            onehot = np.zeros((n, V))
            onehot[ar, yb] = 1.0
            for m in range(M):
                q = np.exp(logq[m])
                if m < M - 1 and distill == "ce":
                    G = lam[m] * g * (q - (1.0 - alpha_d) * onehot - alpha_d * pM)
                elif m < M - 1 and distill == "reverse_kl":
                    kd = q * (logq[m] - logq[M - 1] - rkl[m][:, None])
                    G = lam[m] * g * ((1.0 - alpha_d) * (q - onehot) + alpha_d * kd)
                elif m < M - 1 and distill == "js":
                    kd = q * (0.5 * (logq[m] - logmix[m]) - 0.5 * jq[m][:, None])
                    G = lam[m] * g * ((1.0 - alpha_d) * (q - onehot) + alpha_d * kd)
                elif m < M - 1:
                    kd = q * (accA[m][:, None] - (q < pM).astype(np.float64))
                    G = lam[m] * g * ((1.0 - alpha_d) * (q - onehot) + alpha_d * kd)
                else:
                    G = lam[m] * g * (q - onehot)
                    if teacher_grad:
                        for s in range(M - 1):
                            if distill == "ce":
                                Ts = -pM * (logits[s] - np.sum(pM * logits[s], axis=1)[:, None])
                            elif distill == "reverse_kl":
                                Ts = pM - np.exp(logq[s])
                            elif distill == "js":
                                Ts = pM * (0.5 * (logq[M - 1] - logmix[s]) - 0.5 * jps[s][:, None])
                            else:
                                qs = np.exp(logq[s])
                                Ts = pM * (accB[s][:, None] - (qs >= pM).astype(np.float64))
                            G = G + lam[s] * g * alpha_d * Ts
                out["dh"][m][b0:b0 + n] = G @ Ws[m]
                out["dW"][m] += G.T @ hb[m]
    out["ce_lm"] = out["ce_lm_sum"] / T
    out["ce_kd"] = out["ce_kd_sum"] / T
    out["loss"] = float(np.sum(lam[:M - 1] * ((1.0 - alpha_d) * out["ce_lm"][:M - 1] + alpha_d * out["ce_kd"]))
                        + lam[M - 1] * out["ce_lm"][M - 1])
    return out


def multiexit_loss_vocab_rows(y, h, W, alpha_d=0.3, grad_scale=1.0, vrows=None, token_block=256):
    """Losses over all tokens and the head-gradient rows dW^m[v] for v in vrows.

    Same definitions as ``multiexit_loss``; the logits of every token are
    computed (for the softmax normalisers), but the gradient is formed only in
    the requested vocabulary columns:  dW^m[v] = sum_t G_m[t, v] h_m[t].
    Returns a dict with ce_lm, ce_kd, loss and dW_rows (list of [len(vrows), D_m]).
    """
    y = np.asarray(y, dtype=np.int64)
    vrows = np.asarray(vrows, dtype=np.int64)
    M = len(h)
    T = y.shape[0]
    Ws = [_f64(w) for w in W]
    g = grad_scale / T
    ce_lm = np.zeros(M)
    ce_kd = np.zeros(max(M - 1, 0))
    dW_rows = [np.zeros((vrows.shape[0], w.shape[1])) for w in Ws]
    for b0 in range(0, T, token_block):
        yb = y[b0:b0 + token_block]
        n = yb.shape[0]
        ar = np.arange(n)
        hb = [_f64(hm[b0:b0 + token_block]) for hm in h]
        logits = [hb[m] @ Ws[m].T for m in range(M)]
        lse = [logsumexp_rows(l) for l in logits]
        logq = [logits[m] - lse[m][:, None] for m in range(M)]
        pM = np.exp(logq[M - 1])
        for m in range(M):
            ce_lm[m] += np.sum(lse[m] - logits[m][ar, yb])
        for m in range(M - 1):
            ce_kd[m] += np.sum(-np.sum(pM * logq[m], axis=1))
        onehot = (yb[:, None] == vrows[None, :]).astype(np.float64)
        pM_sel = pM[:, vrows]
        for m in range(M):
            q_sel = np.exp(logq[m][:, vrows])
            if m < M - 1:
                G = g * (q_sel - (1.0 - alpha_d) * onehot - alpha_d * pM_sel)
            else:
                G = g * (q_sel - onehot)
            dW_rows[m] += G.T @ hb[m]
    ce_lm /= T
    ce_kd /= T
    loss = float(np.sum((1.0 - alpha_d) * ce_lm[:M - 1]) + np.sum(alpha_d * ce_kd) + ce_lm[M - 1])
    return {"ce_lm": ce_lm, "ce_kd": ce_kd, "loss": loss, "dW_rows": dW_rows}


def exit_agreement(h, W, rows=None, token_block=256):
    """Agreement of every smaller exit m with the largest exit M, per token and
    as means over the tokens.

    Definitions followed:
      * acceptance probability of a drafted token, beta = sum_v min(q_v, p_v)
        (one minus the total-variation distance between draft q and verifier p;
        "Is nesting the cheapest way to build a model suite?", section 4), with
        the draft q = q_m and the verifier p = p_M;
      * pairwise KL and top-1 next-token agreement between exits ("Matryoshka
        Language Model Suites", agihunt.info summary, alignment paragraph),
        read as KL(p_M || q_m) = sum_v p_M,v (log p_M,v - log q_m,v) and
        [argmax_v q_m = argmax_v p_M], ties going to the lowest index.

    Returns a dict with per-token beta, kl, agree [M-1, T'], top1 [M, T'] (int)
    and their means beta_mean, kl_mean, agree_mean [M-1].
    """
    M = len(h)
    Ws = [_f64(w) for w in W]
    T = h[0].shape[0]
    idx = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    Tn = idx.shape[0]
    out = {"beta": np.zeros((M - 1, Tn)), "kl": np.zeros((M - 1, Tn)), "agree": np.zeros((M - 1, Tn)),
           "top1": np.zeros((M, Tn), dtype=np.int64)}
    for b0 in range(0, Tn, token_block):
        sel = idx[b0:b0 + token_block]
        n = sel.shape[0]
        logits = [_f64(h[m][sel]) @ Ws[m].T for m in range(M)]
        logp = [l - logsumexp_rows(l)[:, None] for l in logits]
        pM = np.exp(logp[M - 1])
        for m in range(M):
            out["top1"][m, b0:b0 + n] = np.argmax(logits[m], axis=1)      # first maximum
        for m in range(M - 1):
            q = np.exp(logp[m])
            out["beta"][m, b0:b0 + n] = np.sum(np.minimum(q, pM), axis=1)
            out["kl"][m, b0:b0 + n] = np.sum(pM * (logp[M - 1] - logp[m]), axis=1)
            out["agree"][m, b0:b0 + n] = (out["top1"][m, b0:b0 + n] == out["top1"][M - 1, b0:b0 + n])
    for k in ("beta", "kl", "agree"):
        out[k + "_mean"] = out[k].mean(axis=1)
    return out
