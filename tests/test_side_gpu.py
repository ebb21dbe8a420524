"""Parity of the fused per-token side outputs (student entropy, sampled-token log-prob)
with the oracle, through ``nb_kl_forward_side``.

"01 · 论文精读与参考实现全景映射" (ars-opd-rebuild docs), section 1 Eq. 6 and Eq. 8: the
per-token entropy of the student and the log-probability of its own sampled token, taken
here under the same tempered softmax as the loss, from the same vocabulary sweep.
"""

import ctypes

import numpy as np
import pytest

import gpu_util as gu
import oracle
from synthetic import make_custom, make_inputs

pytestmark = pytest.mark.gpu

KEYS = ("loss_tok", "lse_s", "lse_t", "aux", "entropy_s", "logp_label")


def run_side(x, beta=None, tau=None, labels=None, side=True):
    import torch
    import full_vocab_kl_b200 as nb
    beta = x.beta if beta is None else beta
    tau = x.tau if tau is None else tau
    t = gu.torch_inputs(x)
    lab = t["labels"] if labels is None else torch.from_numpy(labels).cuda()
    f = nb.kl_forward(t["h_s"], t["W_s"], t["h_t"], t["W_t"], lab, beta, tau, side=side)
    torch.cuda.synchronize()
    assert nb.device_status(f["workspace"]) == 0
    out = {k: f[k].cpu().numpy().astype(np.float64) for k in KEYS if k in f}
    out["loss_mean"] = float(f["loss_mean"].item())
    out["n_valid"] = int(f["n_valid"].item())
    return out


def check(x, beta=None, tau=None, labels=None):
    beta = x.beta if beta is None else beta
    tau = x.tau if tau is None else tau
    lab = x.labels if labels is None else labels
    got = run_side(x, beta, tau, labels)
    ref = oracle.forward(x.h_s, x.W_s, x.h_t, x.W_t, lab, beta, tau, side=True)
    gu.check_forward(got, ref, lab)
    gu.check_side(got, ref, lab, x.W_s.shape[0])
    return got, ref


def test_tiny_workload():
    """128 tokens, fp32 hidden states (hi/lo split), V 4096: two LSE splits."""
    check(make_inputs("tiny"))


@pytest.mark.parametrize("beta", [0.0, 1.0, 0.5])
def test_ragged_with_out_of_range_labels(beta):
    x = make_custom(300, 200, 136, 1000, beta, 0.7, n_masked=37, teacher="independent")
    lab = x.labels.copy()
    valid = np.flatnonzero(lab != -100)
    lab[valid[:3]] = [1000, 123456, -5]        # outside [0, V): NaN log-probability
    check(x, labels=lab)


def test_labels_on_tile_half_and_split_boundaries():
    # V 5000: 20 tiles of 256 -> 3 units of 2048 columns, each split in two column halves
    x = make_custom(512, 256, 320, 5000, 1.0, 1.0, n_masked=40, teacher="correlated")
    lab = x.labels.copy()
    valid = np.flatnonzero(lab != -100)
    edges = [0, 31, 32, 127, 128, 255, 256, 2047, 2048, 2049, 4095, 4096, 4863, 4864, 4991, 4999]
    lab[valid[:len(edges)]] = edges
    check(x, labels=lab)


@pytest.mark.parametrize("beta", [0.0, 1.0, 0.4])
def test_side_outputs_leave_the_loss_bit_identical(beta):
    x = make_custom(384, 128, 192, 3000, beta, 1.3, n_masked=60, teacher="correlated")
    a = run_side(x, side=False)
    b = run_side(x, side=True)
    for k in ("loss_tok", "lse_s", "lse_t", "aux"):
        np.testing.assert_array_equal(a[k], b[k])
    assert a["loss_mean"] == b["loss_mean"]


def test_either_output_may_be_null():
    import torch
    import full_vocab_kl_b200 as nb
    from full_vocab_kl_b200 import _abi, api
    x = make_custom(256, 128, 128, 2048, 1.0, 1.0, n_masked=20, teacher="independent")
    t = gu.torch_inputs(x)
    ref = oracle.forward(x.h_s, x.W_s, x.h_t, x.W_t, x.labels, 1.0, 1.0, side=True)
    shape = api.make_shape(t["h_s"], t["W_s"], t["h_t"], t["W_t"], t["labels"])
    ws = torch.empty(api.workspace_bytes(shape, 1.0), dtype=torch.uint8, device="cuda")
    N = x.labels.shape[0]
    for want in ("entropy_s", "logp_label"):
        o = {k: torch.full((N,), 7.0, device="cuda") for k in KEYS}
        lm = torch.empty((), device="cuda")
        nv = torch.empty((), dtype=torch.int64, device="cuda")
        ent = o["entropy_s"].data_ptr() if want == "entropy_s" else None
        lp = o["logp_label"].data_ptr() if want == "logp_label" else None
        code = _abi.lib().nb_kl_forward_side(
            _abi.shape_ptr(shape), t["h_s"].data_ptr(), t["W_s"].data_ptr(), t["h_t"].data_ptr(),
            t["W_t"].data_ptr(), t["labels"].data_ptr(), ctypes.c_float(1.0), ctypes.c_float(1.0),
            o["loss_tok"].data_ptr(), o["lse_s"].data_ptr(), o["lse_t"].data_ptr(), o["aux"].data_ptr(),
            lm.data_ptr(), nv.data_ptr(), ent, lp, ws.data_ptr(), ws.numel(),
            torch.cuda.current_stream().cuda_stream)
        assert code == 0
        torch.cuda.synchronize()
        assert nb.device_status(ws) == 0
        other = "logp_label" if want == "entropy_s" else "entropy_s"
        assert bool((o[other] == 7.0).all()), "the NULL output's buffer must be untouched"
        got = {k: o[k].cpu().numpy().astype(np.float64) for k in KEYS}
        valid = x.labels != -100
        if want == "entropy_s":
            err = np.abs(got["entropy_s"] - ref["entropy_s"])[valid]
            assert (err <= gu.TOL_TOK_REL * np.abs(ref["entropy_s"][valid]) + gu.TOL_TOK_ABS).all()
        else:
            err = np.abs(got["logp_label"] - ref["logp_label"])[valid]
            assert (err <= 1e-4).all()


@pytest.mark.fullsize
@pytest.mark.parametrize("name", ["opd_0p6b_4b", "long_jsd", "large_vocab"])
def test_full_size_sampled_rows(name):
    """Full-size workloads (the benchmark's launch configuration with side outputs on),
    compared on sampled valid rows that the oracle evaluates exactly."""
    x = make_inputs(name)
    rng = np.random.default_rng(321)
    valid = np.flatnonzero(x.labels != -100)
    sample = np.sort(rng.choice(valid, size=min(32, len(valid)), replace=False))
    if "boost_rows" in x.meta:
        sample = np.union1d(sample, x.meta["boost_rows"][:8])
    got = run_side(x)
    ref = oracle.forward(x.h_s, x.W_s, x.h_t, x.W_t, x.labels, x.beta, x.tau, rows=sample, side=True)
    gu.check_forward(got, ref, x.labels, rows=sample)
    gu.check_side(got, ref, x.labels, x.W_s.shape[0], rows=sample)
    # properties at every valid row: 0 <= H <= ln V and log S[y] <= 0
    H = got["entropy_s"][valid]
    assert (H >= -1e-5).all() and (H <= np.log(x.W_s.shape[0]) + 1e-4).all()
    assert (got["logp_label"][valid] <= 1e-5).all()


@pytest.mark.parametrize("V", [100, 2148])
def test_side_outputs_with_empty_column_halves(V):
    x = make_custom(300, 128, 192, V, 0.5, 0.7, n_masked=40, teacher="correlated")
    check(x)
