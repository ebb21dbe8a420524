"""Vocabulary-parallel loss: the student and teacher unembeddings split by rows across ranks.

"Nitrobrew tweet analysis", section "工程落地": under tensor parallelism (or FSDP) the
unembedding is sharded, and that is where a full-vocabulary loss is hard to integrate. Here
each rank holds a contiguous row range of W_s and W_t and the full hidden states and labels.
The only exchange is the per-token online softmax state of each shard (``VP_FIELDS`` floats
per token), merged with the same log-sum-exp merge the single-GPU call applies between its
vocabulary splits; the JSD adds one more exchange of two partial sums per token. In the
backward pass each rank recomputes its own vocabulary columns with the merged LSEs: its rows
of dW_s come out exact and local, and dh_s is the sum of the ranks' terms (one all-reduce).

Every arithmetic step runs in the library's kernels (``nb_kl_vp_*`` and ``nb_kl_backward``);
this module only orders the calls and the collectives. The kernels are reached through a
``kernels`` object so that the collective plumbing can be exercised without a GPU.
"""

from __future__ import annotations

from typing import Callable, Optional

import torch

from . import _abi
from .api import IGNORE_INDEX, _check_inputs, _stream_ptr, _workspace, kl_backward, make_shape, workspace_bytes

VP_FIELDS = _abi.VP_FIELDS


def shard_range(vocab: int, rank: int, world: int, align: int = 256):
    """Rows [v0, v1) of the vocabulary held by `rank`: contiguous, in rank order, whole
    `align`-row tiles except the last shard's tail, sizes differing by at most one tile."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world size")
    tiles = -(-vocab // align)
    if tiles < world:
        raise ValueError(f"vocabulary of {vocab} rows is too small for {world} shards of {align}-row tiles")
    base, extra = divmod(tiles, world)
    t0 = rank * base + min(rank, extra)
    t1 = t0 + base + (1 if rank < extra else 0)
    return min(vocab, t0 * align), min(vocab, t1 * align)


def _dist_all_gather(group):
    import torch.distributed as dist

    def gather(t: torch.Tensor) -> torch.Tensor:
        world = dist.get_world_size(group)
        out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        dist.all_gather(list(out.unbind(0)), t.contiguous(), group=group)
        return out
    return gather


def _dist_all_reduce(group):
    import torch.distributed as dist

    def reduce(t: torch.Tensor) -> torch.Tensor:
        dist.all_reduce(t, group=group)
        return t
    return reduce


def _check_device_f32(name, t, shape):
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous float32 CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}")


def _check_labels(labels):
    if not isinstance(labels, torch.Tensor) or not labels.is_cuda or labels.dtype != torch.int64 \
            or labels.dim() != 1 or not labels.is_contiguous():
        raise ValueError("labels must be a contiguous int64 CUDA tensor [N]")


class LibraryKernels:
    """The library's calls on device tensors (the product path)."""

    def state(self, h_s, W_s, h_t, W_t, labels, beta, tau, vocab_offset, ignore_index, workspace=None):
        _check_inputs(h_s, W_s, h_t, W_t, labels)
        shape = make_shape(h_s, W_s, h_t, W_t, labels, ignore_index)
        ws = _workspace(workspace_bytes(shape, beta), h_s.device, workspace)
        st = torch.empty((VP_FIELDS, labels.shape[0]), dtype=torch.float32, device=h_s.device)
        code = _abi.lib().nb_kl_vp_state(
            _abi.shape_ptr(shape), int(vocab_offset), h_s.data_ptr(), W_s.data_ptr(), h_t.data_ptr(),
            W_t.data_ptr(), labels.data_ptr(), float(beta), float(tau), st.data_ptr(), ws.data_ptr(),
            ws.numel(), _stream_ptr(h_s.device))
        _abi.check("nb_kl_vp_state", code)
        return st, ws

    def combine(self, states, labels, beta, ignore_index, side):
        _check_labels(labels)
        n_parts, N = states.shape[0], labels.shape[0]
        _check_device_f32("states", states, (n_parts, VP_FIELDS, N))
        if states.device != labels.device:
            raise ValueError("states and labels must be on the same device")
        f32 = dict(dtype=torch.float32, device=labels.device)
        out = {k: torch.empty(N, **f32) for k in ("loss_tok", "lse_s", "lse_t", "aux")}
        if side:
            out["entropy_s"] = torch.empty(N, **f32)
            out["logp_label"] = torch.empty(N, **f32)
        out["loss_mean"] = torch.empty((), **f32)
        out["n_valid"] = torch.empty((), dtype=torch.int64, device=labels.device)
        code = _abi.lib().nb_kl_vp_combine(
            N, n_parts, states.data_ptr(), labels.data_ptr(), int(ignore_index), float(beta),
            out["loss_tok"].data_ptr(), out["lse_s"].data_ptr(), out["lse_t"].data_ptr(), out["aux"].data_ptr(),
            out["entropy_s"].data_ptr() if side else None, out["logp_label"].data_ptr() if side else None,
            out["loss_mean"].data_ptr(), out["n_valid"].data_ptr(), _stream_ptr(labels.device))
        _abi.check("nb_kl_vp_combine", code)
        return out

    def jsd_partial(self, h_s, W_s, h_t, W_t, labels, beta, tau, lse_s, lse_t, ignore_index, workspace=None):
        _check_inputs(h_s, W_s, h_t, W_t, labels)
        _check_device_f32("lse_s", lse_s, (labels.shape[0],))
        _check_device_f32("lse_t", lse_t, (labels.shape[0],))
        shape = make_shape(h_s, W_s, h_t, W_t, labels, ignore_index)
        ws = _workspace(workspace_bytes(shape, beta), h_s.device, workspace)
        part = torch.empty((2, labels.shape[0]), dtype=torch.float32, device=h_s.device)
        code = _abi.lib().nb_kl_vp_jsd_partial(
            _abi.shape_ptr(shape), h_s.data_ptr(), W_s.data_ptr(), h_t.data_ptr(), W_t.data_ptr(),
            labels.data_ptr(), float(beta), float(tau), lse_s.data_ptr(), lse_t.data_ptr(), part.data_ptr(),
            ws.data_ptr(), ws.numel(), _stream_ptr(h_s.device))
        _abi.check("nb_kl_vp_jsd_partial", code)
        return part

    def jsd_combine(self, parts, labels, ignore_index):
        _check_labels(labels)
        n_parts, N = parts.shape[0], labels.shape[0]
        _check_device_f32("parts", parts, (n_parts, 2, N))
        if parts.device != labels.device:
            raise ValueError("parts and labels must be on the same device")
        f32 = dict(dtype=torch.float32, device=labels.device)
        out = {"loss_tok": torch.empty(N, **f32), "aux": torch.empty(N, **f32),
               "loss_mean": torch.empty((), **f32),
               "n_valid": torch.empty((), dtype=torch.int64, device=labels.device)}
        code = _abi.lib().nb_kl_vp_jsd_combine(
            N, n_parts, parts.data_ptr(), labels.data_ptr(), int(ignore_index), out["loss_tok"].data_ptr(),
            out["aux"].data_ptr(), out["loss_mean"].data_ptr(), out["n_valid"].data_ptr(),
            _stream_ptr(labels.device))
        _abi.check("nb_kl_vp_jsd_combine", code)
        return out

    def backward(self, h_s, W_s, h_t, W_t, labels, beta, tau, lse_s, lse_t, aux, grad_out, ignore_index,
                 workspace=None):
        return kl_backward(h_s, W_s, h_t, W_t, labels, beta, tau, lse_s, lse_t, aux, grad_out,
                           ignore_index=ignore_index, workspace=workspace)


def vp_forward(h_s, W_s_shard, h_t, W_t_shard, labels, beta: float, tau: float, *, vocab_offset: int,
               group=None, side: bool = False, ignore_index: int = IGNORE_INDEX, kernels=None,
               all_gather: Optional[Callable] = None) -> dict:
    """Per-token outputs of the full-vocabulary loss, identical on every rank of `group`.

    W_s_shard / W_t_shard are this rank's rows [vocab_offset, vocab_offset + rows) of the
    unembeddings (``shard_range`` gives the usual split; any disjoint cover in rank order
    works). Returns the ``kl_forward`` dictionary (plus ``entropy_s`` / ``logp_label`` with
    ``side``) and this rank's workspace under ``"workspace"``.
    """
    kern = LibraryKernels() if kernels is None else kernels
    gather = _dist_all_gather(group) if all_gather is None else all_gather
    state, ws = kern.state(h_s, W_s_shard, h_t, W_t_shard, labels, beta, tau, vocab_offset, ignore_index)
    out = kern.combine(gather(state), labels, beta, ignore_index, side)
    if 0.0 < beta < 1.0:
        part = kern.jsd_partial(h_s, W_s_shard, h_t, W_t_shard, labels, beta, tau, out["lse_s"], out["lse_t"],
                                ignore_index, ws)
        out.update(kern.jsd_combine(gather(part), labels, ignore_index))
    out["workspace"] = ws
    return out


def vp_backward(h_s, W_s_shard, h_t, W_t_shard, labels, beta: float, tau: float, lse_s, lse_t, aux, grad_out, *,
                group=None, ignore_index: int = IGNORE_INDEX, kernels=None, workspace=None,
                all_reduce: Optional[Callable] = None):
    """(dh_s summed over the ranks, this rank's rows of dW_s), fp32."""
    kern = LibraryKernels() if kernels is None else kernels
    reduce = _dist_all_reduce(group) if all_reduce is None else all_reduce
    dh, dW = kern.backward(h_s, W_s_shard, h_t, W_t_shard, labels, beta, tau, lse_s, lse_t, aux, grad_out,
                           ignore_index, workspace)
    return reduce(dh), dW


class _VocabParallelKL(torch.autograd.Function):
    @staticmethod
    def forward(ctx, h_s, W_s, h_t, W_t, labels, beta, tau, vocab_offset, group, ignore_index, kernels, all_gather,
                all_reduce):
        out = vp_forward(h_s, W_s, h_t, W_t, labels, beta, tau, vocab_offset=vocab_offset, group=group,
                         ignore_index=ignore_index, kernels=kernels, all_gather=all_gather)
        ctx.save_for_backward(h_s, W_s, h_t, W_t, labels, out["lse_s"], out["lse_t"], out["aux"])
        ctx.cfg = (beta, tau, group, ignore_index, kernels, all_reduce)
        ctx.workspace = out["workspace"]
        return out["loss_mean"]

    @staticmethod
    def backward(ctx, grad):
        h_s, W_s, h_t, W_t, labels, lse_s, lse_t, aux = ctx.saved_tensors
        beta, tau, group, ignore_index, kernels, all_reduce = ctx.cfg
        dh, dW = vp_backward(h_s, W_s, h_t, W_t, labels, beta, tau, lse_s, lse_t, aux, grad, group=group,
                             ignore_index=ignore_index, kernels=kernels, workspace=ctx.workspace,
                             all_reduce=all_reduce)
        return (dh.to(h_s.dtype), dW.to(W_s.dtype)) + (None,) * 11


def vocab_parallel_jsd(h_s, h_t, W_s_shard, W_t_shard, labels, vocab_offset: int, beta: float = 1.0,
                       temperature: float = 1.0, group=None, ignore_index: int = IGNORE_INDEX, *,
                       kernels=None, all_gather: Optional[Callable] = None,
                       all_reduce: Optional[Callable] = None):
    """Scalar per-token-mean generalized JSD with row-sharded unembeddings; differentiable in
    h_s (gradient summed over the ranks) and in this rank's W_s rows. `kernels`, `all_gather`
    and `all_reduce` default to the library and torch.distributed over `group`."""
    hs = h_s.reshape(-1, h_s.shape[-1]).contiguous()
    ht = h_t.reshape(-1, h_t.shape[-1]).contiguous()
    lab = labels.reshape(-1).contiguous()
    return _VocabParallelKL.apply(hs, W_s_shard.contiguous(), ht, W_t_shard.contiguous(), lab, float(beta),
                                  float(temperature), int(vocab_offset), group, int(ignore_index), kernels,
                                  all_gather, all_reduce)
