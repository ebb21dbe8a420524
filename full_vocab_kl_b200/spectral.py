"""Spectral-compression front end: the teacher hands over a rank-k code instead of h_t.

"Nitrobrew tweet analysis": thread item 6/8 (spectral compression of the hidden state, at the
price of exactness) and the evaluation table's "SVD-Nitrobrew" row (k floats per token).
With the thin SVD ``W_t = U S V^T`` and ``V_k`` the right singular vectors of the k largest
singular values:

* once per teacher checkpoint, :func:`spectral_factor`: the Gram matrix ``W_t^T W_t`` on the
  library's tcgen05 GEMM (``nb_kl_gram``), its eigenpairs (a d_t x d_t symmetric
  eigendecomposition, ``torch.linalg.eigh`` in float64: the one library step, off the
  per-step path), the k largest and their ``V_k`` rounded to bf16 (``nb_kl_spectral_select``),
  and ``W_t' = W_t V_k`` (``nb_kl_project``);
* every step, on the teacher's side, :func:`teacher_code`: ``h_t' = h_t V_k``
  (``nb_kl_project``), k values per token instead of d_t;
* the loss then runs unchanged on ``(h_t', W_t')`` with d_t = k.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _abi
from .api import _stream_ptr


def _check_bf16(name, t, dim=2):
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != dim:
        raise ValueError(f"{name} must be a {dim}-D bfloat16 CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _small_ws(device):
    return torch.zeros(_abi.SMALL_WORKSPACE_BYTES, dtype=torch.uint8, device=device)


def gram(X: torch.Tensor) -> torch.Tensor:
    """X^T X in fp32 for a bf16 [rows, d] matrix."""
    _check_bf16("X", X)
    rows, d = X.shape
    G = torch.empty((d, d), dtype=torch.float32, device=X.device)
    ws = _small_ws(X.device)
    code = _abi.lib().nb_kl_gram(X.data_ptr(), rows, d, G.data_ptr(), ws.data_ptr(), _stream_ptr(X.device))
    _abi.check("nb_kl_gram", code)
    return G


def project(X: torch.Tensor, basis: torch.Tensor, out: torch.Tensor = None) -> torch.Tensor:
    """X @ basis in bf16 (fp32 accumulation, round to nearest even): X [rows, d], basis [d, k]."""
    _check_bf16("X", X)
    _check_bf16("basis", basis)
    rows, d = X.shape
    if basis.shape[0] != d:
        raise ValueError("basis must have d rows")
    k = basis.shape[1]
    if out is None:
        out = torch.empty((rows, k), dtype=torch.bfloat16, device=X.device)
    _check_bf16("out", out)
    if out.shape != (rows, k):
        raise ValueError("out must be [rows, k]")
    ws = _small_ws(X.device)
    code = _abi.lib().nb_kl_project(X.data_ptr(), rows, d, basis.data_ptr(), k, out.data_ptr(), ws.data_ptr(),
                                    _stream_ptr(X.device))
    _abi.check("nb_kl_project", code)
    return out


@dataclass
class SpectralBasis:
    V_k: torch.Tensor        # [d_t, k] bf16, orthonormal columns (before rounding)
    W_code: torch.Tensor     # [V, k] bf16: W_t V_k, the student-side teacher unembedding
    sigma: torch.Tensor      # [k] float64: the kept singular values of W_t
    V_k_f64: torch.Tensor    # [d_t, k] float64 eigenvectors before rounding


def select_basis(evals: torch.Tensor, evecs: torch.Tensor, k: int):
    """(V_k bf16 [d, k], sigma float64 [k], V_k float64 [d, k]) from the eigenpairs of W_t^T W_t
    (``nb_kl_spectral_select``: the k largest eigenvalues, their eigenvectors rounded to bf16
    once, sigma = sqrt(max(lambda, 0)))."""
    d = evals.shape[0]
    for name, t, shp in (("evals", evals, (d,)), ("evecs", evecs, (d, d))):
        if not t.is_cuda or t.dtype != torch.float64 or tuple(t.shape) != shp or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous float64 CUDA tensor of shape {shp}")
    V_k = torch.empty((d, k), dtype=torch.bfloat16, device=evals.device)
    V64 = torch.empty((d, k), dtype=torch.float64, device=evals.device)
    sigma = torch.empty((k,), dtype=torch.float64, device=evals.device)
    code = _abi.lib().nb_kl_spectral_select(evals.data_ptr(), evecs.data_ptr(), d, k, V_k.data_ptr(),
                                            sigma.data_ptr(), V64.data_ptr(), _stream_ptr(evals.device))
    _abi.check("nb_kl_spectral_select", code)
    return V_k, sigma, V64


def spectral_factor(W_t: torch.Tensor, k: int) -> SpectralBasis:
    """Rank-k spectral basis of the teacher unembedding W_t [V, d_t] (bf16)."""
    _check_bf16("W_t", W_t)
    d_t = W_t.shape[1]
    if not 8 <= k <= d_t or k % 8:
        raise ValueError("k must be a multiple of 8 in [8, d_t]")
    G = gram(W_t).double()
    evals, evecs = torch.linalg.eigh(G)                # the one library step: a d_t x d_t solver
    V_k, sigma, V64 = select_basis(evals.contiguous(), evecs.contiguous(), k)
    return SpectralBasis(V_k=V_k, W_code=project(W_t, V_k), sigma=sigma, V_k_f64=V64)


def teacher_code(h_t: torch.Tensor, basis: SpectralBasis) -> torch.Tensor:
    """Per-step teacher code h_t' = h_t V_k [N, k] bf16."""
    return project(h_t, basis.V_k)
