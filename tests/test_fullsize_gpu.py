"""The five workloads at full size, in the launch configuration the benchmark times.

The oracle cannot materialise every row at these sizes in a test, so:
* loss_tok, lse_s, lse_t, aux and dh_s are compared on sampled valid rows, each of which
  the oracle computes exactly (full-vocabulary logits of that row);
* masked rows must be exactly zero, and loss_mean must equal the mean of loss_tok;
* dW_s is checked through properties that hold at any size (column sums of G vanish, so
  those of dW_s do; <dW_s, W_s> = <dh_s, h_s>) and, exactly, through a second run whose
  labels keep only the sampled rows, compared on sampled vocabulary rows.
"""

import numpy as np
import pytest

import gpu_util as gu
import oracle
from synthetic import WORKLOADS, make_inputs

pytestmark = [pytest.mark.gpu, pytest.mark.fullsize]

N_SAMPLE = 48
V_SAMPLE = 256


def _tensors(x):
    import torch
    t = gu.torch_inputs(x)
    return t


def _run(t, x, labels, dW_init):
    import torch
    import full_vocab_kl_b200 as nb
    f = nb.kl_forward(t["h_s"], t["W_s"], t["h_t"], t["W_t"], labels, x.beta, x.tau)
    dW = None
    if dW_init is not None:
        dW = torch.from_numpy(dW_init).cuda()
    dh, dW = nb.kl_backward(t["h_s"], t["W_s"], t["h_t"], t["W_t"], labels, x.beta, x.tau, f["lse_s"], f["lse_t"],
                            f["aux"], x.grad_out, dW_s=dW, accumulate_dW=dW_init is not None,
                            workspace=f["workspace"])
    torch.cuda.synchronize()
    assert nb.device_status(f["workspace"]) == 0
    return f, dh, dW


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workload_full_size(name):
    import torch
    x = make_inputs(name)
    rng = np.random.default_rng(123)
    valid = np.flatnonzero(x.labels != -100)
    sample = np.sort(rng.choice(valid, size=min(N_SAMPLE, len(valid)), replace=False))
    if "boost_rows" in x.meta:
        sample = np.union1d(sample, x.meta["boost_rows"][:16])
    t = _tensors(x)
    f, dh, dW = _run(t, x, t["labels"], x.dW_init)

    got = {k: f[k].cpu().numpy().astype(np.float64) for k in ("loss_tok", "lse_s", "lse_t", "aux")}
    got["n_valid"] = int(f["n_valid"].item())
    got["loss_mean"] = float(f["loss_mean"].item())
    ref = oracle.forward(x.h_s, x.W_s, x.h_t, x.W_t, x.labels, x.beta, x.tau, rows=sample)
    gu.check_forward(got, ref, x.labels, rows=sample)
    assert got["loss_mean"] == pytest.approx(got["loss_tok"].sum() / got["n_valid"], rel=1e-5)

    # dh_s on the sampled rows
    rb = oracle.backward(x.h_s, x.W_s, x.h_t, x.W_t, x.labels, x.beta, x.tau, grad_out=x.grad_out, rows=sample)
    dh_rows = dh[torch.from_numpy(sample).cuda()].cpu().numpy().astype(np.float64)
    e = gu.rel_l2(dh_rows, rb["dh_s"][sample])
    assert e <= gu.TOL_GRAD, f"dh_s rel L2 on sampled rows {e}"
    masked = torch.from_numpy(x.labels == -100).cuda()
    assert float(dh[masked].abs().max()) == 0.0

    # dW_s invariants of the full run
    dWd = dW.double()
    if x.dW_init is not None:
        dWd -= torch.from_numpy(x.dW_init).cuda().double()
    col = dWd.sum(0).abs()
    scale = dWd.abs().sum(0)
    assert float((col / scale.clamp_min(1e-30)).max()) < 2e-2
    Ws64 = t["W_s"].double()
    lhs = float((dWd * Ws64).sum())
    hs64 = t["h_s"].double()
    rhs = float((dh.double() * hs64).sum())
    assert lhs == pytest.approx(rhs, rel=1e-2, abs=1e-6)
    del dWd, Ws64, hs64

    # exact dW_s on a masked subset: only the sampled rows keep their labels
    sub = np.full_like(x.labels, -100)
    sub[sample] = x.labels[sample]
    _, _, dW2 = _run(t, x, torch.from_numpy(sub).cuda(), x.dW_init)
    vs = np.sort(rng.choice(x.workload.V, size=V_SAMPLE, replace=False))
    vs = np.union1d(vs, [0, x.workload.V - 1])
    ref_dW = oracle.backward(x.h_s, x.W_s, x.h_t, x.W_t, sub, x.beta, x.tau, grad_out=x.grad_out,
                             dW_init=x.dW_init, dW_rows=vs)["dW_s"]
    got_dW = dW2[torch.from_numpy(vs).cuda()].cpu().numpy().astype(np.float64)
    if x.dW_init is not None:
        ref_dW -= x.dW_init[vs]
        got_dW -= x.dW_init[vs]
    e = gu.rel_l2(got_dW, ref_dW)
    assert e <= gu.TOL_GRAD, f"dW_s rel L2 on sampled vocabulary rows {e}"
