"""Vocabulary-parallel kernels on one GPU, with the ranks emulated one after another (each
shard's calls are independent launches; nothing waits on another rank): the merged outputs
must match the oracle of the unsharded problem, and the single-GPU call.

"Nitrobrew tweet analysis", section "工程落地" (sharded unembeddings); the merge is the
split-V log-sum-exp merge of the single-GPU path applied across shards.
"""

import numpy as np
import pytest

import gpu_util as gu
import oracle
from synthetic import make_custom, make_inputs

pytestmark = pytest.mark.gpu


def emulate(x, R, beta=None, tau=None, labels=None, backward=True, side=True):
    import torch
    from full_vocab_kl_b200.vocab_parallel import LibraryKernels, shard_range
    import full_vocab_kl_b200 as nb
    beta = x.beta if beta is None else beta
    tau = x.tau if tau is None else tau
    t = gu.torch_inputs(x)
    lab = t["labels"] if labels is None else torch.from_numpy(labels).cuda()
    V = x.W_s.shape[0]
    kern = LibraryKernels()
    ranges = [shard_range(V, r, R) for r in range(R)]
    states, wss = [], []
    for v0, v1 in ranges:
        st, ws = kern.state(t["h_s"], t["W_s"][v0:v1], t["h_t"], t["W_t"][v0:v1], lab, beta, tau, v0, -100)
        states.append(st)
        wss.append(ws)
    out = kern.combine(torch.stack(states), lab, beta, -100, side)
    if 0.0 < beta < 1.0:
        parts = [kern.jsd_partial(t["h_s"], t["W_s"][v0:v1], t["h_t"], t["W_t"][v0:v1], lab, beta, tau,
                                  out["lse_s"], out["lse_t"], -100, wss[r]) for r, (v0, v1) in enumerate(ranges)]
        out.update(kern.jsd_combine(torch.stack(parts), lab, -100))
    res = {}
    if backward:
        dh = None
        dWs = []
        for r, (v0, v1) in enumerate(ranges):
            d, w = kern.backward(t["h_s"], t["W_s"][v0:v1], t["h_t"], t["W_t"][v0:v1], lab, beta, tau,
                                 out["lse_s"], out["lse_t"], out["aux"], x.grad_out, -100, wss[r])
            dh = d.clone() if dh is None else dh + d
            dWs.append(w)
        res["dh_s"] = dh.cpu().numpy().astype(np.float64)
        res["dW_s"] = torch.cat(dWs).cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    for ws in wss:
        assert nb.device_status(ws) == 0
    for k in ("loss_tok", "lse_s", "lse_t", "aux", "entropy_s", "logp_label"):
        if k in out:
            res[k] = out[k].cpu().numpy().astype(np.float64)
    res["loss_mean"] = float(out["loss_mean"].item())
    res["n_valid"] = int(out["n_valid"].item())
    return res


def check(x, R, beta=None, tau=None, labels=None):
    beta = x.beta if beta is None else beta
    tau = x.tau if tau is None else tau
    lab = x.labels if labels is None else labels
    got = emulate(x, R, beta, tau, labels)
    ref = oracle.forward(x.h_s, x.W_s, x.h_t, x.W_t, lab, beta, tau, side=True)
    ref.update(oracle.backward(x.h_s, x.W_s, x.h_t, x.W_t, lab, beta, tau, grad_out=x.grad_out))
    gu.check_forward(got, ref, lab)
    gu.check_side(got, ref, lab, x.W_s.shape[0])
    assert gu.rel_l2(got["dh_s"], ref["dh_s"]) <= gu.TOL_GRAD
    assert gu.rel_l2(got["dW_s"], ref["dW_s"]) <= gu.TOL_GRAD
    assert (got["dh_s"][lab == -100] == 0).all()
    return got


@pytest.mark.parametrize("R", [1, 2, 3])
@pytest.mark.parametrize("beta", [0.0, 1.0, 0.5])
def test_shards_match_oracle(R, beta):
    # V 5000 = 20 tiles -> shards of 7/7/6 tiles (R = 3), the last one ragged
    x = make_custom(600, 192, 256, 5000, beta, 0.8, n_masked=90, teacher="correlated")
    lab = x.labels.copy()
    valid = np.flatnonzero(lab != -100)
    lab[valid[:8]] = [0, 1791, 1792, 2559, 2560, 3583, 3584, 4999]   # around the shard edges
    check(x, R, labels=lab)


def test_matches_single_gpu_call():
    import torch
    import full_vocab_kl_b200 as nb
    x = make_custom(512, 128, 256, 4096, 1.0, 1.0, n_masked=64, teacher="correlated")
    got = emulate(x, 4, backward=False)
    t = gu.torch_inputs(x)
    f = nb.kl_forward(t["h_s"], t["W_s"], t["h_t"], t["W_t"], t["labels"], 1.0, 1.0, side=True)
    torch.cuda.synchronize()
    valid = x.labels != -100
    for k in ("loss_tok", "lse_s", "lse_t", "entropy_s", "logp_label"):
        a, b = got[k][valid], f[k].cpu().numpy().astype(np.float64)[valid]
        assert np.abs(a - b).max() <= 2e-5 * np.abs(b).max() + 2e-6, k
    assert got["loss_mean"] == pytest.approx(float(f["loss_mean"].item()), rel=1e-5)


@pytest.mark.fullsize
@pytest.mark.parametrize("name,R", [("opd_0p6b_4b", 4), ("long_jsd", 2)])
def test_full_size_sampled_rows(name, R):
    x = make_inputs(name)
    rng = np.random.default_rng(99)
    valid = np.flatnonzero(x.labels != -100)
    sample = np.sort(rng.choice(valid, size=24, replace=False))
    got = emulate(x, R, backward=False)
    ref = oracle.forward(x.h_s, x.W_s, x.h_t, x.W_t, x.labels, x.beta, x.tau, rows=sample, side=True)
    gu.check_forward(got, ref, x.labels, rows=sample)
    gu.check_side(got, ref, x.labels, x.W_s.shape[0], rows=sample)
    assert got["loss_mean"] == pytest.approx(got["loss_tok"].sum() / got["n_valid"], rel=1e-5)


@pytest.mark.parametrize("R", [2, 3])
def test_fp32_hidden_states(R):
    """The 128-token workload (fp32 hidden states carried as bf16 hi + lo) with the vocabulary
    split over R shards."""
    check(make_inputs("tiny"), R)
