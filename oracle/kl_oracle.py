"""CPU oracle for the full-vocabulary hidden-state distillation loss (fp64, NumPy).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import this module. The CUDA
library never calls it and shares no code with it: this file materialises full
logit rows and evaluates every quantity from its plain definition, in float64.

What it follows (page title, section):

* "Nitrobrew tweet analysis" (ricardokevins notes), section "Nitrobrew 的两个动作":
  logits are rebuilt as ``z = h @ W^T`` from the final hidden state for both
  models; a softmax / log-sum-exp and the KL terms are taken over the whole
  vocabulary.
* same page, section "仓库实现": the gradient reaches only the student hidden
  state and the student unembedding (the teacher is frozen); with p = student,
  q = teacher, the forward-KL logit gradient is ``p - q`` and the reverse-KL one
  is ``p * (log p - log q - KL)``.
* "03 White-box OPD" (ars-opd-rebuild docs), section 1, Eq. (2): the reverse KL
  ``KL(pi_theta || pi_T)`` summed per token.
* same page, section 2.3 (the beta table): beta = 0 gives ``KL(T || S)``,
  beta = 1 gives ``KL(S || T)``, beta in (0, 1) gives
  ``beta * KL(T || M) + (1 - beta) * KL(S || M)`` with ``M = (1 - beta) S + beta T``;
  the temperature divides the logits before the softmax; work in the log domain
  (the mixture via log-sum-exp); the reduction is a per-token mean over the
  positions whose label is not -100.

Readings where the pages leave a step open (each is listed in the design notes):

1. beta == 0.0 and beta == 1.0 exactly select the two KL directions; any other
   beta in (0, 1) is the mixture form (which degenerates to 0 at the ends).
2. No tau^2 factor; gradients with respect to z carry 1/tau.
3. ``lse_s`` / ``lse_t`` are natural-log LSEs of the tempered logits ``u = z / tau``.
4. ``aux`` is the per-token KL for beta in {0, 1} and ``KL(S || M)`` for the JSD.
5. No valid row (N_v = 0): loss 0 and zero gradients.
6. Masked rows: every per-token output is 0 and their gradient rows are 0.
7. Log-probabilities come from logits (``u - lse``), never from log of a
   probability, so ``0 * log 0`` never arises; a probability that underflows to
   0 contributes 0.
8. Rows are not shifted: row n of h_s, h_t and labels is one position.

Per-token side outputs of the student (``forward(..., side=True)``), from
"01 · 论文精读与参考实现全景映射" (ars-opd-rebuild docs), section 1 (Eq. 6,
the per-token entropy H_t that the peak-entropy scheduler ranks; Eq. 8, the
log-probability the student gives its own sampled token) and section 3.5:

9. Both are taken under the same tempered student distribution S = softmax(z_s / tau)
   that the loss uses (at tau = 1, the model's own distribution):
   ``entropy_s = -sum_v S log S`` and ``logp_label = log S[label]`` in nats.
10. The sampled token of row n is ``labels[n]`` (rows are not shifted, reading 8);
    masked rows get 0 for both; a label outside [0, V) gets NaN log-probability.
"""

from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

IGNORE_INDEX = -100
_V_BLOCK = 16384


def _to_f64(a: np.ndarray) -> np.ndarray:
    """float64 values of an input block; uint16 arrays are bf16 bit patterns."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


def tempered_logits(h: np.ndarray, W: np.ndarray, tau: float) -> np.ndarray:
    """u = (h @ W^T) / tau for a block of rows, full vocabulary, in float64.

    The product is evaluated one group of vocabulary rows at a time only so that
    a bf16 W is upcast piecewise; every logit is still one plain dot product.
    """
    h64 = _to_f64(h)
    V = W.shape[0]
    u = np.empty((h64.shape[0], V), dtype=np.float64)
    for v0 in range(0, V, _V_BLOCK):
        v1 = min(V, v0 + _V_BLOCK)
        u[:, v0:v1] = h64 @ _to_f64(W[v0:v1]).T
    u /= tau
    return u


def log_softmax(u: np.ndarray):
    """Row-wise log-probabilities and natural-log LSE (max-shifted, float64)."""
    m = u.max(axis=1, keepdims=True)
    lse = m + np.log(np.exp(u - m).sum(axis=1, keepdims=True))
    return u - lse, lse[:, 0]


def _kl_rows(logp: np.ndarray, logq: np.ndarray) -> np.ndarray:
    """Sum_v p (log p - log q) per row, p = exp(logp)."""
    return (np.exp(logp) * (logp - logq)).sum(axis=1)


def _log_mixture(logS: np.ndarray, logT: np.ndarray, beta: float) -> np.ndarray:
    """log M with M = (1 - beta) S + beta T, evaluated by log-sum-exp."""
    return np.logaddexp(math.log1p(-beta) + logS, math.log(beta) + logT)


def divergence_rows(logS: np.ndarray, logT: np.ndarray, beta: float):
    """Per-row generalized JSD and its auxiliary term (see readings 1 and 4)."""
    if beta == 0.0:
        loss = _kl_rows(logT, logS)
        return loss, loss.copy()
    if beta == 1.0:
        loss = _kl_rows(logS, logT)
        return loss, loss.copy()
    logM = _log_mixture(logS, logT, beta)
    k_s = _kl_rows(logS, logM)
    k_t = _kl_rows(logT, logM)
    return beta * k_t + (1.0 - beta) * k_s, k_s


def dloss_du_student(logS: np.ndarray, logT: np.ndarray, beta: float, loss: np.ndarray,
                     aux: np.ndarray) -> np.ndarray:
    """d(per-token loss)/d(u_s), u_s = z_s / tau, per element of the row block."""
    S = np.exp(logS)
    if beta == 0.0:
        return S - np.exp(logT)
    if beta == 1.0:
        return S * (logS - logT - loss[:, None])
    logM = _log_mixture(logS, logT, beta)
    return (1.0 - beta) * S * (logS - logM - aux[:, None])


def student_side_rows(logS: np.ndarray, labels: np.ndarray):
    """Entropy -sum S log S and log S[label] for a block of rows (readings 9 and 10)."""
    H = -(np.exp(logS) * logS).sum(axis=1)
    V = logS.shape[1]
    lab = np.asarray(labels, dtype=np.int64)
    inside = (lab >= 0) & (lab < V)
    logp = np.full(lab.shape[0], np.nan)
    logp[inside] = logS[np.flatnonzero(inside), lab[inside]]
    return H, logp


def _check(beta: float, tau: float):
    if not (0.0 <= beta <= 1.0):
        raise ValueError("beta must be in [0, 1]")
    if not tau > 0.0:
        raise ValueError("tau must be positive")


def _selected_rows(labels: np.ndarray, ignore_index: int, rows: Optional[Sequence[int]]):
    """Valid mask, the valid positions to evaluate (all, or those of ``rows``), and N_v.

    N_v counts every position whose label is not ``ignore_index`` ("03 White-box OPD",
    section 2.3): it is the denominator of the per-token mean whether or not ``rows``
    restricts the positions evaluated.
    """
    valid = labels != ignore_index
    n_valid = int(valid.sum())
    todo = np.flatnonzero(valid) if rows is None else np.asarray(
        [r for r in rows if valid[r]], dtype=np.int64)
    return valid, todo, n_valid


def _row_blocks(rows: np.ndarray, block: int):
    for i in range(0, len(rows), block):
        yield rows[i:i + block]


def forward(h_s, W_s, h_t, W_t, labels, beta: float, tau: float, *,
            rows: Optional[Sequence[int]] = None, ignore_index: int = IGNORE_INDEX,
            row_block: int = 256, side: bool = False) -> dict:
    """Per-token loss, both LSEs, aux, and the per-token mean.

    ``rows`` restricts the per-token outputs to those positions (the mean is then
    only returned when every valid row is among them). Returns float64 arrays of
    length N (zeros where not computed or masked). With ``side`` the student's
    per-token entropy and sampled-token log-probability are added
    (``entropy_s``, ``logp_label``).
    """
    _check(beta, tau)
    labels = np.asarray(labels)
    N = labels.shape[0]
    valid, todo, n_valid = _selected_rows(labels, ignore_index, rows)
    keys = ("loss_tok", "lse_s", "lse_t", "aux") + (("entropy_s", "logp_label") if side else ())
    out = {k: np.zeros(N) for k in keys}
    for r in _row_blocks(todo, row_block):
        logS, lse_s = log_softmax(tempered_logits(h_s[r], W_s, tau))
        logT, lse_t = log_softmax(tempered_logits(h_t[r], W_t, tau))
        loss, aux = divergence_rows(logS, logT, beta)
        out["loss_tok"][r], out["aux"][r] = loss, aux
        out["lse_s"][r], out["lse_t"][r] = lse_s, lse_t
        if side:
            out["entropy_s"][r], out["logp_label"][r] = student_side_rows(logS, labels[r])
    complete = np.unique(todo).size == n_valid   # every valid position was evaluated
    out["n_valid"] = n_valid
    if not complete:
        out["loss_mean"] = None
    elif n_valid == 0:
        out["loss_mean"] = 0.0
    else:
        out["loss_mean"] = float(out["loss_tok"][valid].sum() / n_valid)
    return out


def backward(h_s, W_s, h_t, W_t, labels, beta: float, tau: float, *, grad_out: float = 1.0,
             dW_init: Optional[np.ndarray] = None, rows: Optional[Sequence[int]] = None,
             want_dW: bool = True, dW_rows: Optional[Sequence[int]] = None,
             ignore_index: int = IGNORE_INDEX, row_block: int = 256) -> dict:
    """Gradients of ``grad_out * mean_loss`` w.r.t. h_s and W_s (the teacher is frozen).

    ``G[n, v] = grad_out / (N_v * tau) * d loss_n / d u_s[n, v]`` on valid rows,
    ``dh_s = G @ W_s`` and ``dW_s = G^T @ h_s`` (plus ``dW_init`` when given).
    With ``rows`` only those rows of ``dh_s`` are produced and ``dW_s`` is left out.
    With ``dW_rows`` only those vocabulary rows of ``dW_s`` are produced (in that order).
    """
    _check(beta, tau)
    labels = np.asarray(labels)
    N, d_s = labels.shape[0], h_s.shape[1]
    _, todo, n_valid = _selected_rows(labels, ignore_index, rows)
    want_dW = want_dW and rows is None
    dh = np.zeros((N, d_s))
    dW = None
    sel = None if dW_rows is None else np.asarray(dW_rows, dtype=np.int64)
    if want_dW:
        if sel is None:
            dW = np.zeros((W_s.shape[0], d_s)) if dW_init is None else np.array(dW_init, dtype=np.float64)
        else:
            dW = np.zeros((len(sel), d_s)) if dW_init is None else np.array(dW_init[sel], dtype=np.float64)
    if n_valid == 0:
        return {"dh_s": dh, "dW_s": dW}
    scale = grad_out / (n_valid * tau)
    for r in _row_blocks(todo, row_block):
        logS, _ = log_softmax(tempered_logits(h_s[r], W_s, tau))
        logT, _ = log_softmax(tempered_logits(h_t[r], W_t, tau))
        loss, aux = divergence_rows(logS, logT, beta)
        G = scale * dloss_du_student(logS, logT, beta, loss, aux)
        for v0 in range(0, W_s.shape[0], _V_BLOCK):
            v1 = min(W_s.shape[0], v0 + _V_BLOCK)
            dh[r] += G[:, v0:v1] @ _to_f64(W_s[v0:v1])
            if want_dW and sel is None:
                dW[v0:v1] += G[:, v0:v1].T @ _to_f64(h_s[r])
        if want_dW and sel is not None:
            dW += G[:, sel].T @ _to_f64(h_s[r])
    return {"dh_s": dh, "dW_s": dW}
