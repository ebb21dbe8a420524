"""CPU oracle of the spectral-compression front end (fp64, NumPy).

TEST INFRASTRUCTURE ONLY: like ``kl_oracle``, only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU legs may import it; the CUDA library shares no code with it.

What it follows: "Nitrobrew tweet analysis" (ricardokevins notes). The thread summary
(item 6/8) explores spectral compression, which shrinks the hidden state handed from the
teacher below d_model at the price of exactness; the evaluation table counts the floats sent
per token as V for logits, d_model for hidden states and the rank k for "SVD-Nitrobrew".
Logits are ``z = W_U h`` (item 3/8), so with the thin SVD ``W_t = U S V^T``:

* teacher side, per token: the code ``h_t' = V_k^T h_t`` (k floats, what crosses the wire);
* student side, once per teacher checkpoint: ``W_t' = U_k S_k = W_t V_k``;
* the loss then sees ``z_t' = W_t' h_t' = W_t V_k V_k^T h_t``, the logits of the best
  rank-k approximation of W_t (Eckart–Young), exact when k >= rank(W_t).

Readings (listed in the design notes): V_k are the right singular vectors of the k largest
singular values of the teacher unembedding itself (no centring, no weighting by data); the
same V_k projects every token; the compressed pair (h_t', W_t') is fed to the unchanged loss
with d_t = k.
"""

from __future__ import annotations

import numpy as np

from .kl_oracle import _to_f64


def spectral_basis(W_t: np.ndarray, k: int):
    """(V_k [d_t, k], sigma [k]): right singular vectors of the k largest singular values of
    W_t (by the thin SVD, in float64), columns ordered by decreasing singular value."""
    W = _to_f64(W_t)
    if not 1 <= k <= W.shape[1]:
        raise ValueError("rank k must be in [1, d_t]")
    _, s, vt = np.linalg.svd(W, full_matrices=False)
    return vt[:k].T.copy(), s[:k].copy()


def project(x: np.ndarray, V_k: np.ndarray) -> np.ndarray:
    """Rows of x expressed in the basis: x V_k (teacher codes h_t', or W_t' = W_t V_k)."""
    return _to_f64(x) @ _to_f64(V_k)


def compress_teacher(h_t: np.ndarray, W_t: np.ndarray, k: int):
    """(h_t', W_t', V_k): the teacher code and unembedding of rank k."""
    V_k, _ = spectral_basis(W_t, k)
    return project(h_t, V_k), project(W_t, V_k), V_k
