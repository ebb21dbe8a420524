"""Teacher -> student hand-off of final hidden states between processes and GPUs.

"Nitrobrew tweet analysis", thread items 3/8 and 4/8 and section "OPD 为什么更痛": when the
teacher runs on another GPU, the loss needs the teacher's final hidden state (d_t values per
token, or the rank-k code of the spectral front end) instead of V logits per token. The
teacher's buffer reaches this process either as a peer device's tensor (same process,
``enable_peer_access``) or through CUDA IPC (a CUDA tensor sent through a
``torch.multiprocessing`` queue arrives mapped into the receiver). ``receive_rows`` then
copies it into local memory with the library's copy kernel (plain 16-byte loads over the link,
valid rows only when labels are given), so that the loss's forward and backward both read it
locally; the loss also accepts the mapped tensor itself as h_t.
"""

from __future__ import annotations

from typing import Optional

import torch

from . import _abi
from .api import IGNORE_INDEX, _stream_ptr


def enable_peer_access(peer_device: int) -> None:
    """Let the current device read `peer_device`'s memory (idempotent)."""
    _abi.check("nb_kl_enable_peer_access", _abi.lib().nb_kl_enable_peer_access(int(peer_device)))


def receive_rows(src: torch.Tensor, labels: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                 ignore_index: int = IGNORE_INDEX, device: Optional[torch.device] = None) -> torch.Tensor:
    """Copy the teacher's [N, d] hidden rows into a local tensor on `device` (default: the
    current device). With `labels` ([N] int64 on that device) only rows whose label is not
    `ignore_index` are copied; the others keep `out`'s contents (zeros for a new tensor)."""
    if not isinstance(src, torch.Tensor) or not src.is_cuda or src.dim() != 2 or not src.is_contiguous():
        raise ValueError("src must be a contiguous 2-D CUDA tensor")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if out is None:
        out = (torch.zeros if labels is not None else torch.empty)(src.shape, dtype=src.dtype, device=dev)
    if out.shape != src.shape or out.dtype != src.dtype or not out.is_contiguous() or out.device != dev:
        raise ValueError("out must be a contiguous tensor of src's shape and dtype on the target device")
    if labels is not None and (labels.dtype != torch.int64 or labels.device != dev or labels.shape != (src.shape[0],)):
        raise ValueError("labels must be int64 [N] on the target device")
    row_bytes = src.shape[1] * src.element_size()
    with torch.cuda.device(dev):
        code = _abi.lib().nb_kl_handoff_rows(src.data_ptr(), out.data_ptr(), src.shape[0], row_bytes,
                                             labels.data_ptr() if labels is not None else None, int(ignore_index),
                                             _stream_ptr(dev))
    _abi.check("nb_kl_handoff_rows", code)
    return out
