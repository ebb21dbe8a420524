"""Pins of the oracle's partial paths: a subset of positions (``rows=``), the accumulated
dW_s (``dW_init=``) and a subset of vocabulary rows of dW_s (``dW_rows=``).

The full-size GPU checks only evaluate sampled positions and vocabulary rows, so these
paths are pinned on their own, against facts that do not come from the oracle:

* "03 White-box OPD", section 2.3: the loss is a per-token mean over every position whose
  label is not -100, so the gradient of one position carries 1 / N_v with N_v the count of
  ALL valid positions, however few of them are evaluated. The pin is a central finite
  difference of the full mean loss, taken only through ``forward`` over all rows.
* The accumulated dW_s (dW_s accumulation of the large-vocabulary workload) is the start
  value plus the gradient: the pin is the start value plus the same finite difference.
* Per-position values of a subset are compared with the pure-Python probability-domain
  brute force of ``test_oracle_pins``.
"""

import numpy as np
import pytest

import oracle
from test_oracle_pins import brute_row, rand_problem

GRAD_OUT = 0.7
EPS = 1e-6


def _problem(seed=200):
    rng = np.random.default_rng(seed)
    N, V = 6, 9
    h_s, W_s, h_t, W_t = rand_problem(rng, N, V, 4, 5, scale=2.0)
    labels = np.array([3, -100, 0, 8, -100, 5])        # N_v = 4
    return rng, h_s, W_s, h_t, W_t, labels


def _fd(arr, loss_of, idxs):
    """Central differences of loss_of(perturbed copy) at the given indices of `arr`."""
    out = np.zeros(arr.shape)
    for idx in idxs:
        p, m = arr.copy(), arr.copy()
        p[idx] += EPS
        m[idx] -= EPS
        out[idx] = (loss_of(p) - loss_of(m)) / (2 * EPS)
    return out


def _mean_loss(h_s, W_s, h_t, W_t, labels, beta, tau):
    return GRAD_OUT * oracle.forward(h_s, W_s, h_t, W_t, labels, beta, tau)["loss_mean"]


@pytest.mark.parametrize("beta", [0.0, 1.0, 0.35])
def test_rows_subset_forward_matches_brute_force(beta):
    _, h_s, W_s, h_t, W_t, labels = _problem()
    tau = 1.3
    rows = [5, 1, 2]                                     # 2 valid of the 4, plus a masked one
    out = oracle.forward(h_s, W_s, h_t, W_t, labels, beta, tau, rows=rows)
    assert out["n_valid"] == 4
    assert out["loss_mean"] is None                      # not every valid position was evaluated
    for r in range(len(labels)):
        if r in (5, 2):
            loss, lse_s, lse_t = brute_row(h_s[r], W_s, h_t[r], W_t, beta, tau)
            assert out["loss_tok"][r] == pytest.approx(loss, rel=1e-11, abs=1e-14)
            assert out["lse_s"][r] == pytest.approx(lse_s, rel=1e-12)
            assert out["lse_t"][r] == pytest.approx(lse_t, rel=1e-12)
        else:
            assert out["loss_tok"][r] == 0 and out["lse_s"][r] == 0 and out["aux"][r] == 0
    # every valid position, in any order and with repeats: the mean over N_v is returned
    full = oracle.forward(h_s, W_s, h_t, W_t, labels, beta, tau, rows=[5, 3, 0, 3, 2, 1])
    want = sum(brute_row(h_s[r], W_s, h_t[r], W_t, beta, tau)[0] for r in (0, 2, 3, 5)) / 4
    assert full["loss_mean"] == pytest.approx(want, rel=1e-11)


@pytest.mark.parametrize("beta", [0.0, 1.0, 0.35])
def test_rows_subset_backward_uses_all_valid_rows(beta):
    """dh_s of a sampled position is the derivative of the mean over ALL N_v positions."""
    _, h_s, W_s, h_t, W_t, labels = _problem()
    tau = 0.8
    rows = [3, 4]                                        # one valid position (N_v is 4)
    back = oracle.backward(h_s, W_s, h_t, W_t, labels, beta, tau, grad_out=GRAD_OUT, rows=rows)
    assert back["dW_s"] is None
    num = _fd(h_s, lambda hs: _mean_loss(hs, W_s, h_t, W_t, labels, beta, tau),
              [(3, j) for j in range(h_s.shape[1])])
    np.testing.assert_allclose(back["dh_s"][3], num[3], rtol=1e-6, atol=1e-9 * np.abs(num[3]).max())
    others = [r for r in range(len(labels)) if r != 3]
    assert not back["dh_s"][others].any()


@pytest.mark.parametrize("beta", [0.0, 1.0, 0.35])
def test_dW_init_is_added_to_the_gradient(beta):
    rng, h_s, W_s, h_t, W_t, labels = _problem()
    tau = 1.1
    init = rng.standard_normal(W_s.shape)
    back = oracle.backward(h_s, W_s, h_t, W_t, labels, beta, tau, grad_out=GRAD_OUT, dW_init=init)
    num = _fd(W_s, lambda ws: _mean_loss(h_s, ws, h_t, W_t, labels, beta, tau), list(np.ndindex(*W_s.shape)))
    scale = np.abs(num).max()
    np.testing.assert_allclose(back["dW_s"] - init, num, rtol=0, atol=1e-6 * scale)
    # the start value is not modified in place
    assert not np.shares_memory(back["dW_s"], init)
    # a subset of vocabulary rows, in any order and with repeats, with and without a start value
    sel = [8, 0, 4, 4]
    part = oracle.backward(h_s, W_s, h_t, W_t, labels, beta, tau, grad_out=GRAD_OUT, dW_init=init, dW_rows=sel)
    np.testing.assert_allclose(part["dW_s"] - init[sel], num[sel], rtol=0, atol=1e-6 * scale)
    part0 = oracle.backward(h_s, W_s, h_t, W_t, labels, beta, tau, grad_out=GRAD_OUT, dW_rows=sel)
    np.testing.assert_allclose(part0["dW_s"], num[sel], rtol=0, atol=1e-6 * scale)
