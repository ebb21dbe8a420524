"""Helpers shared by the GPU parity tests: move synthetic inputs to the device, run the
library through its C ABI, and compare with the oracle under the stated tolerances.

Tolerances (valid rows only):
  mean loss       relative error <= 1e-3
  per-token loss  |d| <= 2e-3 |ref| + 1e-5 nats
  lse_s, lse_t    relative error <= 1e-5
  dh_s, dW_s      relative L2 error <= 1e-2
Side outputs (valid rows only):
  entropy_s       |d| <= 2e-3 |ref| + 1e-5 nats (the per-token loss bound)
  logp_label      |d| <= 1e-5 (|lse_s| + |u_label|) + 1e-5 nats (the LSE bound carried
                  through log S[y] = u_y - lse_s); NaN exactly where the label is outside [0, V)
"""

import numpy as np

import oracle

TOL_MEAN = 1e-3
TOL_TOK_REL, TOL_TOK_ABS = 2e-3, 1e-5
TOL_LSE = 1e-5
TOL_GRAD = 1e-2


def torch_inputs(x, device="cuda"):
    import torch
    t = {}
    for k in ("h_s", "h_t", "W_s", "W_t"):
        a = getattr(x, k)
        if a.dtype == np.uint16:
            t[k] = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        else:
            t[k] = torch.from_numpy(a).to(device)
    t["labels"] = torch.from_numpy(x.labels).to(device)
    return t


def run_library(x, chunk_v=0, beta=None, tau=None, labels=None, backward=True, dW_init=None):
    """Forward (+ backward with grad_out = x.grad_out) through the C ABI; numpy results."""
    import torch
    import full_vocab_kl_b200 as nb
    beta = x.beta if beta is None else beta
    tau = x.tau if tau is None else tau
    t = torch_inputs(x)
    lab = t["labels"] if labels is None else torch.from_numpy(labels).cuda()
    f = nb.kl_forward(t["h_s"], t["W_s"], t["h_t"], t["W_t"], lab, beta, tau, chunk_v=chunk_v)
    out = {k: f[k].cpu().numpy().astype(np.float64) for k in ("loss_tok", "lse_s", "lse_t", "aux")}
    out["loss_mean"] = float(f["loss_mean"].item())
    out["n_valid"] = int(f["n_valid"].item())
    assert nb.device_status(f["workspace"]) == 0
    if backward:
        dW = None
        acc = dW_init is not None
        if acc:
            dW = torch.from_numpy(np.ascontiguousarray(dW_init, dtype=np.float32)).cuda()
        dh, dW = nb.kl_backward(t["h_s"], t["W_s"], t["h_t"], t["W_t"], lab, beta, tau, f["lse_s"], f["lse_t"],
                                f["aux"], x.grad_out, dW_s=dW, accumulate_dW=acc, chunk_v=chunk_v,
                                workspace=f["workspace"])
        torch.cuda.synchronize()
        assert nb.device_status(f["workspace"]) == 0
        out["dh_s"] = dh.cpu().numpy().astype(np.float64)
        out["dW_s"] = dW.cpu().numpy().astype(np.float64)
    return out


def rel_l2(a, b):
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def check_forward(got, ref, labels, rows=None):
    valid = labels != -100
    sel = np.flatnonzero(valid) if rows is None else np.asarray([r for r in rows if valid[r]])
    assert got["n_valid"] == int(valid.sum())
    lt, rt = got["loss_tok"][sel], ref["loss_tok"][sel]
    bad = ~(np.abs(lt - rt) <= TOL_TOK_REL * np.abs(rt) + TOL_TOK_ABS)   # NaN counts as off
    assert not bad.any(), f"per-token loss: {bad.sum()} rows off, worst {np.abs(lt - rt)[bad].max()}"
    for k in ("lse_s", "lse_t"):
        err = np.abs(got[k][sel] - ref[k][sel]) / np.maximum(np.abs(ref[k][sel]), 1e-30)
        assert err.max(initial=0.0) <= TOL_LSE, f"{k}: rel err {err.max()}"
    aerr = np.abs(got["aux"][sel] - ref["aux"][sel])
    assert (aerr <= TOL_TOK_REL * np.abs(ref["aux"][sel]) + TOL_TOK_ABS).all(), f"aux: worst {aerr.max()}"
    masked = np.flatnonzero(~valid)
    for k in ("loss_tok", "lse_s", "lse_t", "aux"):
        assert (got[k][masked] == 0).all(), f"{k} not zero on masked rows"
    if ref.get("loss_mean") is not None:
        m = ref["loss_mean"]
        if m == 0.0:
            assert got["loss_mean"] == 0.0
        else:
            assert abs(got["loss_mean"] - m) <= TOL_MEAN * abs(m) + 1e-7, (got["loss_mean"], m)
    assert np.isfinite(got["loss_tok"]).all() and np.isfinite(got["loss_mean"])


def check_side(got, ref, labels, V, rows=None):
    valid = labels != -100
    sel = np.flatnonzero(valid) if rows is None else np.asarray([r for r in rows if valid[r]])
    H, Hr = got["entropy_s"][sel], ref["entropy_s"][sel]
    bad = ~(np.abs(H - Hr) <= TOL_TOK_REL * np.abs(Hr) + TOL_TOK_ABS)
    assert not bad.any(), f"entropy: {bad.sum()} rows off, worst {np.abs(H - Hr)[bad].max()}"
    lp, lpr = got["logp_label"][sel], ref["logp_label"][sel]
    inside = (labels[sel] >= 0) & (labels[sel] < V)
    assert np.isnan(lp[~inside]).all() and np.isnan(lpr[~inside]).all()
    lp, lpr = lp[inside], lpr[inside]
    lse = ref["lse_s"][sel][inside]
    bound = TOL_LSE * (np.abs(lse) + np.abs(lpr + lse)) + 1e-5
    bad = ~(np.abs(lp - lpr) <= bound)
    assert not bad.any(), f"logp_label: {bad.sum()} rows off, worst {np.abs(lp - lpr)[bad].max()}"
    masked = np.flatnonzero(~valid)
    for k in ("entropy_s", "logp_label"):
        assert (got[k][masked] == 0).all(), f"{k} not zero on masked rows"


def oracle_all(x, beta=None, tau=None, labels=None, dW_init=None):
    beta = x.beta if beta is None else beta
    tau = x.tau if tau is None else tau
    lab = x.labels if labels is None else labels
    f = oracle.forward(x.h_s, x.W_s, x.h_t, x.W_t, lab, beta, tau)
    b = oracle.backward(x.h_s, x.W_s, x.h_t, x.W_t, lab, beta, tau, grad_out=x.grad_out, dW_init=dW_init)
    f.update(b)
    return f
