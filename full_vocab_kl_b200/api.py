"""PyTorch-facing API over the C ABI. PyTorch only supplies device memory and streams;
every step of the loss runs in the library's CUDA kernels.

Entry points, named after the distillation pages' API ("Nitrobrew tweet analysis",
section "工程落地": ``forward_kl`` / ``reverse_kl`` taking the student and teacher
hidden states, both unembeddings and a temperature):

* :func:`kl_forward` / :func:`kl_backward` — one call each of ``nb_kl_forward`` /
  ``nb_kl_backward`` with caller-visible outputs (``side=True``: ``nb_kl_forward_side``,
  adding the student's per-token entropy and sampled-token log-probability);
* :func:`generalized_jsd`, :func:`forward_kl`, :func:`reverse_kl` — autograd-enabled
  scalar losses (gradients reach ``h_s`` and ``W_s`` only; the teacher is frozen).
"""

from __future__ import annotations

from typing import Optional

import torch

from . import _abi

IGNORE_INDEX = -100


def _stream_ptr(device: torch.device):
    return torch.cuda.current_stream(device).cuda_stream


def _check_inputs(h_s, W_s, h_t, W_t, labels):
    for name, t in (("h_s", h_s), ("W_s", W_s), ("h_t", h_t), ("W_t", W_t), ("labels", labels)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if h_s.dtype != h_t.dtype or h_s.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("h_s and h_t must both be bfloat16 or both float32")
    if W_s.dtype != torch.bfloat16 or W_t.dtype != torch.bfloat16:
        raise ValueError("W_s and W_t must be bfloat16")
    if labels.dtype != torch.int64:
        raise ValueError("labels must be int64")
    if h_s.dim() != 2 or h_t.dim() != 2 or W_s.dim() != 2 or W_t.dim() != 2 or labels.dim() != 1:
        raise ValueError("expected h [N, d], W [V, d], labels [N]")
    N = labels.shape[0]
    if h_s.shape[0] != N or h_t.shape[0] != N:
        raise ValueError("h_s, h_t and labels must have the same number of rows")
    if W_s.shape[0] != W_t.shape[0] or W_s.shape[1] != h_s.shape[1] or W_t.shape[1] != h_t.shape[1]:
        raise ValueError("inconsistent hidden widths or vocabulary sizes")


def make_shape(h_s, W_s, h_t, W_t, labels, ignore_index: int = IGNORE_INDEX, chunk_v: int = 0) -> _abi.Shape:
    return _abi.Shape(
        n_tokens=labels.shape[0], vocab=W_s.shape[0], d_s=h_s.shape[1], d_t=h_t.shape[1],
        h_dtype=_abi.NB_F32 if h_s.dtype == torch.float32 else _abi.NB_BF16, reserved=0,
        ignore_index=ignore_index, chunk_v=chunk_v)


def workspace_bytes(shape: _abi.Shape, beta: float) -> int:
    n = _abi.lib().nb_kl_workspace_size(_abi.shape_ptr(shape), float(beta))
    if n == 0:
        raise ValueError("invalid shape for the library")
    return int(n)


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]) -> torch.Tensor:
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes or not workspace.is_cuda:
            raise ValueError("workspace too small")
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def kl_forward(h_s, W_s, h_t, W_t, labels, beta: float = 1.0, tau: float = 1.0, *,
               ignore_index: int = IGNORE_INDEX, chunk_v: int = 0, workspace: Optional[torch.Tensor] = None,
               out: Optional[dict] = None, side: bool = False) -> dict:
    """Per-token loss, both tempered LSEs, aux, masked mean and N_v (device tensors).

    With ``side``, also ``entropy_s`` (entropy of the tempered student softmax) and
    ``logp_label`` (its log-probability of each row's label), fp32 [N], 0 on masked rows.
    """
    _check_inputs(h_s, W_s, h_t, W_t, labels)
    dev = h_s.device
    N = labels.shape[0]
    shape = make_shape(h_s, W_s, h_t, W_t, labels, ignore_index, chunk_v)
    ws = _workspace(workspace_bytes(shape, beta), dev, workspace)
    if out is None:
        f32 = dict(dtype=torch.float32, device=dev)
        out = {
            "loss_tok": torch.empty(N, **f32), "lse_s": torch.empty(N, **f32), "lse_t": torch.empty(N, **f32),
            "aux": torch.empty(N, **f32), "loss_mean": torch.empty((), **f32),
            "n_valid": torch.empty((), dtype=torch.int64, device=dev),
        }
        if side:
            out["entropy_s"] = torch.empty(N, **f32)
            out["logp_label"] = torch.empty(N, **f32)
    else:
        # caller-supplied outputs: device tensors of the right dtype and shape
        want = {"loss_tok": (torch.float32, (N,)), "lse_s": (torch.float32, (N,)), "lse_t": (torch.float32, (N,)),
                "aux": (torch.float32, (N,)), "loss_mean": (torch.float32, ()), "n_valid": (torch.int64, ())}
        if side:
            want.update(entropy_s=(torch.float32, (N,)), logp_label=(torch.float32, (N,)))
        for k, (dt, shp) in want.items():
            t = out.get(k)
            if not isinstance(t, torch.Tensor) or not t.is_cuda or t.device != dev or t.dtype != dt \
                    or tuple(t.shape) != shp or not t.is_contiguous():
                raise ValueError(f"out['{k}'] must be a contiguous {dt} tensor of shape {shp} on {dev}")
    common = (_abi.shape_ptr(shape), h_s.data_ptr(), W_s.data_ptr(), h_t.data_ptr(), W_t.data_ptr(),
              labels.data_ptr(), float(beta), float(tau), out["loss_tok"].data_ptr(), out["lse_s"].data_ptr(),
              out["lse_t"].data_ptr(), out["aux"].data_ptr(), out["loss_mean"].data_ptr(),
              out["n_valid"].data_ptr())
    tail = (ws.data_ptr(), ws.numel() * ws.element_size(), _stream_ptr(dev))
    if side:
        code = _abi.lib().nb_kl_forward_side(*common, out["entropy_s"].data_ptr(), out["logp_label"].data_ptr(),
                                             *tail)
        _abi.check("nb_kl_forward_side", code)
    else:
        code = _abi.lib().nb_kl_forward(*common, *tail)
        _abi.check("nb_kl_forward", code)
    out["workspace"] = ws
    return out


def kl_backward(h_s, W_s, h_t, W_t, labels, beta: float, tau: float, lse_s, lse_t, aux, grad_out, *,
                dh_s: Optional[torch.Tensor] = None, dW_s: Optional[torch.Tensor] = None,
                accumulate_dW: bool = False, ignore_index: int = IGNORE_INDEX, chunk_v: int = 0,
                workspace: Optional[torch.Tensor] = None):
    """(dh_s, dW_s) in fp32 for d(grad_out * loss_mean)."""
    _check_inputs(h_s, W_s, h_t, W_t, labels)
    dev = h_s.device
    N, d_s, V = labels.shape[0], h_s.shape[1], W_s.shape[0]
    shape = make_shape(h_s, W_s, h_t, W_t, labels, ignore_index, chunk_v)
    ws = _workspace(workspace_bytes(shape, beta), dev, workspace)
    if dh_s is None:
        dh_s = torch.empty((N, d_s), dtype=torch.float32, device=dev)
    if dW_s is None:
        if accumulate_dW:
            raise ValueError("accumulate_dW needs an existing dW_s")
        dW_s = torch.empty((V, d_s), dtype=torch.float32, device=dev)
    for name, t in (("lse_s", lse_s), ("lse_t", lse_t), ("aux", aux), ("dh_s", dh_s), ("dW_s", dW_s)):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous float32 CUDA tensor")
    if not torch.is_tensor(grad_out):
        grad_out = torch.tensor(float(grad_out), dtype=torch.float32, device=dev)
    grad_out = grad_out.to(device=dev, dtype=torch.float32).contiguous()
    code = _abi.lib().nb_kl_backward(
        _abi.shape_ptr(shape), h_s.data_ptr(), W_s.data_ptr(), h_t.data_ptr(), W_t.data_ptr(), labels.data_ptr(),
        float(beta), float(tau), lse_s.data_ptr(), lse_t.data_ptr(), aux.data_ptr(), grad_out.data_ptr(),
        dh_s.data_ptr(), dW_s.data_ptr(), 1 if accumulate_dW else 0, ws.data_ptr(),
        ws.numel() * ws.element_size(), _stream_ptr(dev))
    _abi.check("nb_kl_backward", code)
    return dh_s, dW_s


def device_status(workspace: torch.Tensor) -> int:
    return _abi.lib().nb_kl_device_status(workspace.data_ptr(), _stream_ptr(workspace.device))


class _FullVocabKL(torch.autograd.Function):
    @staticmethod
    def forward(ctx, h_s, W_s, h_t, W_t, labels, beta, tau, ignore_index, chunk_v):
        out = kl_forward(h_s, W_s, h_t, W_t, labels, beta, tau, ignore_index=ignore_index, chunk_v=chunk_v)
        ctx.save_for_backward(h_s, W_s, h_t, W_t, labels, out["lse_s"], out["lse_t"], out["aux"])
        ctx.cfg = (beta, tau, ignore_index, chunk_v)
        ctx.workspace = out["workspace"]
        return out["loss_mean"]

    @staticmethod
    def backward(ctx, grad):
        h_s, W_s, h_t, W_t, labels, lse_s, lse_t, aux = ctx.saved_tensors
        beta, tau, ignore_index, chunk_v = ctx.cfg
        dh, dW = kl_backward(h_s, W_s, h_t, W_t, labels, beta, tau, lse_s, lse_t, aux, grad,
                             ignore_index=ignore_index, chunk_v=chunk_v, workspace=ctx.workspace)
        return dh.to(h_s.dtype), dW.to(W_s.dtype), None, None, None, None, None, None, None


def generalized_jsd(h_s, h_t, W_s, W_t, labels=None, beta: float = 1.0, temperature: float = 1.0,
                    ignore_index: int = IGNORE_INDEX, chunk_v: int = 0):
    """Scalar per-token-mean generalized JSD (beta 0: forward KL, 1: reverse KL).

    h_s [..., d_s], h_t [..., d_t], W_s [V, d_s], W_t [V, d_t]; labels [...] (None: every
    position counts). Differentiable in h_s and W_s.
    """
    lead = h_s.shape[:-1]
    hs = h_s.reshape(-1, h_s.shape[-1]).contiguous()
    ht = h_t.reshape(-1, h_t.shape[-1]).contiguous()
    if labels is None:
        labels = torch.zeros(lead, dtype=torch.int64, device=h_s.device)
    lab = labels.reshape(-1).contiguous()
    return _FullVocabKL.apply(hs, W_s.contiguous(), ht, W_t.contiguous(), lab, float(beta), float(temperature),
                              int(ignore_index), int(chunk_v))


def forward_kl(xs, xt, ws, wt, temperature: float = 1.0, labels=None, **kw):
    """KL(teacher || student) with the pages' argument order (student/teacher hidden, unembeddings)."""
    return generalized_jsd(xs, xt, ws, wt, labels, beta=0.0, temperature=temperature, **kw)


def reverse_kl(xs, xt, ws, wt, temperature: float = 1.0, labels=None, **kw):
    """KL(student || teacher), the OPD objective."""
    return generalized_jsd(xs, xt, ws, wt, labels, beta=1.0, temperature=temperature, **kw)
