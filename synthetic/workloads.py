"""Workload table and seeded generators for the distillation-loss inputs.

Shapes follow the workloads the distillation pages talk about (Qwen-sized
student/teacher pairs, V = 151936 or 248320, T up to 8192); there is no dataset
or trained weight here, only seeded Gaussian data with the stated statistics.

Recipe (every tensor has its own random stream ``SeedSequence([seed, id, block])``,
so the bytes do not depend on the thread count):

* hidden states: ``N(0, 1)`` rows, RMS-normalised (``x / sqrt(mean(x^2) + 1e-6)``),
  then rounded to bf16 (round-to-nearest-even) unless the workload keeps fp32;
* unembeddings: ``N(0, (c / sqrt(d))^2)`` so that logits have std about ``c``,
  rounded to bf16;
* correlated teacher: the student signal is embedded into the teacher width by a
  random signed coordinate embedding ``Q`` (an isometry, ``Q^T Q = I``):
  ``h_t = RMSnorm(0.7 * sqrt(d_t/d_s) * Q h_s + 0.3 * eps)`` and
  ``W_t = sqrt(d_s/d_t) * W_s Q^T + W_perp (I - Q Q^T)``, which makes
  ``z_t ~= 0.92 z_s + noise`` while every entry of ``W_t`` keeps variance
  ``c^2 / d_t``;
* spectral teacher: ``W_t' = U_k S_k`` of the thin SVD of a Gaussian
  ``[V, k]`` matrix (computed as ``G V`` from the eigenvectors of ``G^T G``),
  with an independent RMS-normalised ``N(0, 1)`` code ``h_t'``;
* boosted rows: ``h += a * W[v] / |W[v]|^2`` on both models at the same id, which
  raises that logit by ``a`` before the temperature;
* masks: exact counts per sequence, either a prompt prefix or a uniform subset;
  masked labels are -100, the others uniform in ``[0, V)``.

Nothing here computes any part of the loss.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

IGNORE_INDEX = -100

# tensor ids of the per-tensor random streams
_ID_HS, _ID_HT, _ID_WS, _ID_WT, _ID_EPS, _ID_Q, _ID_MASK, _ID_LABEL, _ID_BOOST, _ID_DW, _ID_SPEC = range(11)
_BLOCK_ROWS = 8192


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    d_s: int
    d_t: int
    V: int
    beta: float
    tau: float
    w_std: float                  # logit scale c: W ~ N(0, (c/sqrt(d))^2)
    h_dtype: str = "bf16"         # "bf16" or "f32"
    teacher: str = "correlated"   # "independent" | "correlated" | "spectral"
    mask: str = "random"          # "prefix" | "random"
    masked_per_seq: int = 0
    boost_frac: float = 0.0       # fraction of all positions with one boosted logit
    boost: float = 0.0            # logit increase (before the temperature)
    accumulate_dW: bool = False
    description: str = ""

    @property
    def N(self) -> int:
        return self.B * self.T

    @property
    def n_valid(self) -> int:
        return self.B * (self.T - self.masked_per_seq)


WORKLOADS = {
    "tiny": Workload(
        "tiny", 1, 128, 256, 384, 4096, 1.0, 1.0, 2.5, h_dtype="f32",
        teacher="independent", mask="prefix", masked_per_seq=32,
        description="128 tokens, d 256/384, V 4096, fp32 hidden states, reverse KL"),
    "opd_0p6b_4b": Workload(
        "opd_0p6b_4b", 4, 2048, 1024, 2560, 151936, 1.0, 1.0, 3.0,
        teacher="correlated", mask="prefix", masked_per_seq=819,
        description="Qwen3-0.6B/4B-shaped OPD, 8192 tokens, V 151936, reverse KL, 40% prompt prefix masked"),
    "long_jsd": Workload(
        "long_jsd", 1, 8192, 2048, 4096, 151936, 0.5, 2.0, 3.0,
        teacher="correlated", mask="random", masked_per_seq=2048,
        boost_frac=0.01, boost=20.0,
        description="T 8192, JSD beta 0.5, tau 2, 1% rows with a +20 logit, 25% masked"),
    "large_vocab": Workload(
        "large_vocab", 1, 8192, 5120, 5120, 248320, 0.0, 1.0, 4.0,
        teacher="correlated", mask="random", masked_per_seq=2458, accumulate_dW=True,
        description="V 248320, d 5120/5120, forward KL, 30% masked, dW_s accumulated"),
    "spectral": Workload(
        "spectral", 8, 4096, 4096, 512, 151936, 1.0, 1.0, 3.0,
        teacher="spectral", mask="random", masked_per_seq=1434,
        description="32768 tokens, rank-512 teacher code, reverse KL, 35% masked"),
}


# Same widths and statistics as a named workload but fewer tokens and a smaller vocabulary,
# so that a detailed profiler capture of one kernel stays small (the unembeddings, 543 MB,
# still exceed L2). 512 valid rows (4 token tiles) x 37 units of 2048 columns = 148 forward
# units: one per SM, so the capture shows steady-state behaviour, not a ragged last wave.
PROFILE_WORKLOADS = {
    "opd_0p6b_4b_prof": Workload(
        "opd_0p6b_4b_prof", 1, 640, 1024, 2560, 75776, 1.0, 1.0, 3.0,
        teacher="correlated", mask="prefix", masked_per_seq=128,
        description="profiling size of opd_0p6b_4b: 640 tokens (512 valid), V 75776"),
    # the OPD workload's token shape (4 x 2048 tokens, 819-token prompt prefix masked per
    # sequence, 4916 valid) with a 24576-row vocabulary: the backward's GEMM launch keeps the
    # full workload's proportions (dh_s: 20 x 2 tiles over the chunk, dW_s: 96 x 2 tiles over
    # the valid tokens) in under 1 GB on the device; the unembeddings (176 MB) exceed L2
    "opd_0p6b_4b_v24k_prof": Workload(
        "opd_0p6b_4b_v24k_prof", 4, 2048, 1024, 2560, 24576, 1.0, 1.0, 3.0,
        teacher="correlated", mask="prefix", masked_per_seq=819,
        description="profiling size of opd_0p6b_4b: its 8192 tokens (4916 valid), V 24576"),
    # the long_jsd workload's tokens, widths, mask and boosted rows with a 24576-row vocabulary
    # (unembeddings 302 MB): its three sweeps (state, JSD pass, JSD gradient) at profiling size
    "long_jsd_v24k_prof": Workload(
        "long_jsd_v24k_prof", 1, 8192, 2048, 4096, 24576, 0.5, 2.0, 3.0,
        teacher="correlated", mask="random", masked_per_seq=2048,
        boost_frac=0.01, boost=20.0,
        description="profiling size of long_jsd: its 8192 tokens (6144 valid), V 24576"),
    "spectral_prof": Workload(
        "spectral_prof", 2, 4096, 4096, 512, 32768, 1.0, 1.0, 3.0,
        teacher="spectral", mask="random", masked_per_seq=1434,
        description="profiling size of spectral: 8192 tokens, V 32768, rank-512 teacher code"),
}


# ----------------------------------------------------------------------------------------
# bf16 byte handling
# ----------------------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + (((u >> 16) & 1) + 0x7FFF)) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact float32 values of bf16 bit patterns."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------------------
# random streams
# ----------------------------------------------------------------------------------------
def _rng(seed: int, tid: int, block: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tid, block])))


def _threads() -> int:
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        n = os.cpu_count() or 1
    return max(1, min(32, n))


def _blocks(rows: int):
    return [(b, r0, min(rows, r0 + _BLOCK_ROWS)) for b, r0 in enumerate(range(0, rows, _BLOCK_ROWS))]


def _parallel(fn, jobs):
    if len(jobs) <= 1:
        for j in jobs:
            fn(*j)
        return
    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(lambda j: fn(*j), jobs))


def _rms_norm_rows(x: np.ndarray) -> np.ndarray:
    return (x / np.sqrt(np.mean(x.astype(np.float64) ** 2, axis=1, keepdims=True) + 1e-6)).astype(np.float32)


def _normal_rows_f32(seed: int, tid: int, rows: int, cols: int, std: float = 1.0) -> np.ndarray:
    out = np.empty((rows, cols), dtype=np.float32)

    def job(b, r0, r1):
        g = _rng(seed, tid, b)
        g.standard_normal((r1 - r0, cols), dtype=np.float32, out=out[r0:r1])
        if std != 1.0:
            out[r0:r1] *= np.float32(std)

    _parallel(job, _blocks(rows))
    return out


def _normal_rows_bf16(seed: int, tid: int, rows: int, cols: int, std: float) -> np.ndarray:
    out = np.empty((rows, cols), dtype=np.uint16)

    def job(b, r0, r1):
        g = _rng(seed, tid, b)
        x = g.standard_normal((r1 - r0, cols), dtype=np.float32)
        x *= np.float32(std)
        out[r0:r1] = f32_to_bf16_bits(x)

    _parallel(job, _blocks(rows))
    return out


# ----------------------------------------------------------------------------------------
# inputs
# ----------------------------------------------------------------------------------------
@dataclass
class Inputs:
    """One synthetic problem. bf16 tensors are uint16 bit patterns; fp32 hidden states stay float32."""

    workload: Workload
    seed: int
    h_s: np.ndarray
    h_t: np.ndarray
    W_s: np.ndarray
    W_t: np.ndarray
    labels: np.ndarray
    dW_init: Optional[np.ndarray] = None
    grad_out: float = 1.0
    meta: dict = field(default_factory=dict)

    @property
    def beta(self) -> float:
        return self.workload.beta

    @property
    def tau(self) -> float:
        return self.workload.tau

    @property
    def h_is_f32(self) -> bool:
        return self.h_s.dtype == np.float32

    def as_float(self, name: str) -> np.ndarray:
        """float32 values of a tensor (exact for bf16 storage)."""
        a = getattr(self, name)
        return bf16_bits_to_f32(a) if a.dtype == np.uint16 else np.asarray(a, dtype=np.float32)


def _mask_labels(w: Workload, seed: int) -> np.ndarray:
    labels = _rng(seed, _ID_LABEL).integers(0, w.V, size=w.N, dtype=np.int64)
    g = _rng(seed, _ID_MASK)
    lab = labels.reshape(w.B, w.T)
    k = w.masked_per_seq
    for b in range(w.B):
        if k <= 0:
            continue
        if w.mask == "prefix":
            lab[b, :k] = IGNORE_INDEX
        elif w.mask == "random":
            lab[b, g.choice(w.T, size=k, replace=False)] = IGNORE_INDEX
        else:
            raise ValueError(w.mask)
    return labels


def _signed_embedding(seed: int, d_s: int, d_t: int):
    g = _rng(seed, _ID_Q)
    sel = g.permutation(d_t)[:d_s]
    sign = np.where(g.integers(0, 2, size=d_s) == 1, 1.0, -1.0).astype(np.float32)
    return sel, sign


def make_inputs(name_or_workload, seed: int = 0) -> Inputs:
    """Generate the seeded inputs of a named workload (or a custom :class:`Workload`)."""
    if isinstance(name_or_workload, str):
        w = WORKLOADS.get(name_or_workload) or PROFILE_WORKLOADS[name_or_workload]
    else:
        w = name_or_workload
    N, d_s, d_t, V = w.N, w.d_s, w.d_t, w.V
    sd_s, sd_t = w.w_std / math.sqrt(d_s), w.w_std / math.sqrt(d_t)

    hs = _rms_norm_rows(_normal_rows_f32(seed, _ID_HS, N, d_s))
    W_s = _normal_rows_bf16(seed, _ID_WS, V, d_s, sd_s)
    labels = _mask_labels(w, seed)

    if w.teacher == "independent":
        ht = _rms_norm_rows(_normal_rows_f32(seed, _ID_HT, N, d_t))
        W_t = _normal_rows_bf16(seed, _ID_WT, V, d_t, sd_t)
    elif w.teacher == "correlated":
        if d_t < d_s:
            raise ValueError("correlated teacher needs d_t >= d_s")
        sel, sign = _signed_embedding(seed, d_s, d_t)
        eps = _normal_rows_f32(seed, _ID_EPS, N, d_t)
        proj = np.zeros((N, d_t), dtype=np.float32)
        proj[:, sel] = hs * sign
        ht = _rms_norm_rows(np.float32(0.7 * math.sqrt(d_t / d_s)) * proj + np.float32(0.3) * eps)
        W_t = np.empty((V, d_t), dtype=np.uint16)
        scale = np.float32(math.sqrt(d_s / d_t))

        def job(b, r0, r1):
            blk = _rng(seed, _ID_WT, b).standard_normal((r1 - r0, d_t), dtype=np.float32)
            blk *= np.float32(sd_t)
            blk[:, sel] = bf16_bits_to_f32(W_s[r0:r1]) * (sign * scale)
            W_t[r0:r1] = f32_to_bf16_bits(blk)

        _parallel(job, _blocks(V))
    elif w.teacher == "spectral":
        G = _normal_rows_f32(seed, _ID_WT, V, d_t, sd_t).astype(np.float64)
        evals, evecs = np.linalg.eigh(G.T @ G)
        Vk = evecs[:, ::-1]  # descending singular values
        W_t = f32_to_bf16_bits((G @ Vk).astype(np.float32))
        del G
        ht = _rms_norm_rows(_normal_rows_f32(seed, _ID_HT, N, d_t))
    else:
        raise ValueError(w.teacher)

    meta = {}
    if w.boost_frac > 0.0:
        g = _rng(seed, _ID_BOOST)
        valid_rows = np.flatnonzero(labels != IGNORE_INDEX)
        n_boost = min(len(valid_rows), int(round(w.boost_frac * N)))
        rows = np.sort(g.choice(valid_rows, size=n_boost, replace=False))
        ids = g.integers(0, V, size=n_boost)
        for r, v in zip(rows, ids):
            ws = bf16_bits_to_f32(W_s[v]).astype(np.float64)
            wt = bf16_bits_to_f32(W_t[v]).astype(np.float64)
            hs[r] += (w.boost * ws / np.dot(ws, ws)).astype(np.float32)
            ht[r] += (w.boost * wt / np.dot(wt, wt)).astype(np.float32)
        meta["boost_rows"] = rows
        meta["boost_ids"] = ids

    if w.h_dtype == "f32":
        h_s, h_t = hs, ht
    elif w.h_dtype == "bf16":
        h_s, h_t = f32_to_bf16_bits(hs), f32_to_bf16_bits(ht)
    else:
        raise ValueError(w.h_dtype)

    dW_init = None
    if w.accumulate_dW:
        dW_init = _normal_rows_f32(seed, _ID_DW, V, d_s, 1e-3)
    return Inputs(w, seed, h_s, h_t, W_s, W_t, labels, dW_init, 1.0, meta)


def make_custom(N: int, d_s: int, d_t: int, V: int, beta: float, tau: float, *, n_masked: int = 0,
                w_std: float = 3.0, h_dtype: str = "bf16", teacher: str = "independent",
                mask: str = "random", boost_frac: float = 0.0, boost: float = 0.0,
                accumulate_dW: bool = False, seed: int = 0) -> Inputs:
    """A one-sequence problem of arbitrary (possibly ragged) size for edge-case tests."""
    w = Workload(f"custom_N{N}_ds{d_s}_dt{d_t}_V{V}", 1, N, d_s, d_t, V, beta, tau, w_std,
                 h_dtype=h_dtype, teacher=teacher, mask=mask, masked_per_seq=n_masked,
                 boost_frac=boost_frac, boost=boost, accumulate_dW=accumulate_dW)
    return make_inputs(w, seed)


def matrix_with_spectrum(rows: int, cols: int, sigma, seed: int = 0) -> np.ndarray:
    """bf16 bits of U diag(sigma) Q^T with random orthonormal U [rows, cols] and Q [cols, cols]
    (QR of seeded Gaussians), for tests of a rank-k teacher basis. sigma has `cols` entries."""
    sigma = np.asarray(sigma, dtype=np.float64)
    if sigma.shape != (cols,):
        raise ValueError("sigma needs one value per column")
    g = _rng(seed, _ID_SPEC)
    U, _ = np.linalg.qr(g.standard_normal((rows, cols)))
    Q, _ = np.linalg.qr(g.standard_normal((cols, cols)))
    return f32_to_bf16_bits(((U * sigma) @ Q.T).astype(np.float32))


def gaussian_bf16(rows: int, cols: int, std: float, seed: int = 0, stream: int = _ID_SPEC) -> np.ndarray:
    """bf16 bits of a seeded N(0, std^2) matrix (row blocks drawn in parallel)."""
    return _normal_rows_bf16(seed, stream, rows, cols, std)
