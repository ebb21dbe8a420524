"""Pins of the oracle's per-token side outputs: student entropy and sampled-token log-prob.

Source: "01 · 论文精读与参考实现全景映射" (ars-opd-rebuild docs), section 1 (Eq. 6: the
per-token entropy H_t of the student policy that the peak-entropy scheduler ranks; Eq. 8:
log pi_theta(y_t | x, y_<t), the student's log-probability of its own sampled token) and
section 3.5. Both are taken under the tempered student softmax S = softmax(z_s / tau).

Every expected value here comes from a definition written out independently of the
oracle (probability-domain loops, closed forms of two-level distributions, limits),
not from the oracle's own log-domain arithmetic.
"""

import math

import numpy as np
import pytest

import oracle
from test_oracle_pins import logits_problem, rand_problem

RTOL = 1e-12


def side(z_s, labels, tau=1.0):
    """Side outputs of rows whose student logits are exactly z_s (teacher irrelevant)."""
    z_s = np.atleast_2d(np.asarray(z_s, dtype=np.float64))
    args = logits_problem(z_s, np.zeros_like(z_s), labels)
    return oracle.forward(*args, 1.0, tau, side=True)


def brute_side(hs, Ws, tau, label):
    """Probability domain, explicit loops, no max shift: H = -sum p ln p, ln p[label]."""
    V = len(Ws)
    e = [math.exp(math.fsum(a * b for a, b in zip(hs, Ws[v])) / tau) for v in range(V)]
    Z = math.fsum(e)
    p = [x / Z for x in e]
    H = -math.fsum(q * math.log(q) for q in p if q > 0.0)
    return H, math.log(p[label])


@pytest.mark.parametrize("tau", [1.0, 0.7, 2.0])
@pytest.mark.parametrize("V", [12, 64])
def test_brute_force_tiny(tau, V):
    rng = np.random.default_rng(11 + V)
    N = 6
    h_s, W_s, h_t, W_t = rand_problem(rng, N, V, 8, 8, scale=3.0)
    labels = rng.integers(0, V, N)
    out = oracle.forward(h_s, W_s, h_t, W_t, labels, 1.0, tau, side=True)
    for n in range(N):
        H, lp = brute_side(h_s[n], W_s, tau, int(labels[n]))
        assert out["entropy_s"][n] == pytest.approx(H, rel=RTOL)
        assert out["logp_label"][n] == pytest.approx(lp, rel=RTOL)


def test_uniform_student():
    """W_s = 0: S is uniform, so H = ln V and every token has log-prob -ln V."""
    V = 41
    out = oracle.forward(np.ones((3, 5)), np.zeros((V, 5)), np.ones((3, 4)), np.zeros((V, 4)),
                         np.array([0, 17, 40]), 0.5, 1.7, side=True)
    np.testing.assert_allclose(out["entropy_s"], math.log(V), rtol=RTOL)
    np.testing.assert_allclose(out["logp_label"], -math.log(V), rtol=RTOL)


@pytest.mark.parametrize("k,a,b,tau", [(1, 5.0, 0.0, 1.0), (3, 2.0, -1.0, 2.0), (7, -4.0, 1.5, 0.5)])
def test_two_level_closed_form(k, a, b, tau):
    """k logits equal to a and V - k equal to b: p_a = e^(a/tau) / (k e^(a/tau) + (V-k) e^(b/tau))."""
    V = 20
    z = np.full(V, b)
    z[:k] = a
    Z = k * math.exp(a / tau) + (V - k) * math.exp(b / tau)
    pa, pb = math.exp(a / tau) / Z, math.exp(b / tau) / Z
    H = -(k * pa * math.log(pa) + (V - k) * pb * math.log(pb))
    out = side([z, z], [0, V - 1], tau)
    np.testing.assert_allclose(out["entropy_s"], H, rtol=1e-12)
    assert out["logp_label"][0] == pytest.approx(math.log(pa), rel=1e-12)
    assert out["logp_label"][1] == pytest.approx(math.log(pb), rel=1e-12)


def test_log_probs_over_all_labels_sum_to_one():
    rng = np.random.default_rng(4)
    V = 30
    z = rng.standard_normal(V) * 4
    out = side(np.tile(z, (V, 1)), np.arange(V), 0.8)
    assert math.fsum(math.exp(x) for x in out["logp_label"]) == pytest.approx(1.0, rel=1e-13)
    # and the expectation of -log p under p is the entropy
    p = np.exp(out["logp_label"])
    assert -math.fsum(p * out["logp_label"]) == pytest.approx(out["entropy_s"][0], rel=1e-12)


def test_entropy_matches_uniform_teacher_reverse_kl():
    """KL(S || uniform) = ln V - H(S): the reverse-KL path gives H independently."""
    rng = np.random.default_rng(8)
    V = 25
    z = rng.standard_normal((4, V)) * 3
    out = side(z, np.zeros(4, np.int64), 1.3)
    np.testing.assert_allclose(out["entropy_s"], math.log(V) - out["loss_tok"], rtol=1e-12)


def test_temperature_limits_and_monotonicity():
    """H(softmax(z / tau)) rises with tau, tends to ln V as tau grows and to 0 as tau shrinks."""
    z = np.array([3.0, 1.0, 0.5, -2.0, 0.0, 2.9])
    V = len(z)
    taus = [0.005, 0.05, 0.3, 1.0, 3.0, 30.0, 3000.0]
    H = [side(z, [0], t)["entropy_s"][0] for t in taus]
    assert all(H[i] < H[i + 1] for i in range(len(H) - 1))
    assert H[-1] == pytest.approx(math.log(V), rel=1e-6)
    assert H[0] < 1e-6
    # the top token's log-prob tends to 0 at small tau and to -ln V at large tau
    assert side(z, [0], 0.01)["logp_label"][0] == pytest.approx(0.0, abs=1e-3)
    assert side(z, [0], 3000.0)["logp_label"][0] == pytest.approx(-math.log(V), rel=1e-3)


def test_masked_rows_and_out_of_range_labels():
    rng = np.random.default_rng(2)
    V = 16
    z = rng.standard_normal((4, V))
    out = side(z, [3, -100, V, -1], 1.0)
    assert out["entropy_s"][1] == 0.0 and out["logp_label"][1] == 0.0
    assert math.isnan(out["logp_label"][2]) and math.isnan(out["logp_label"][3])
    assert out["entropy_s"][2] > 0.0 and out["entropy_s"][3] > 0.0
    assert math.isfinite(out["logp_label"][0])


def test_side_outputs_do_not_change_the_loss():
    rng = np.random.default_rng(6)
    h_s, W_s, h_t, W_t = rand_problem(rng, 5, 33, 8, 6, scale=2.0)
    labels = np.array([1, -100, 7, 32, 0])
    for beta in (0.0, 0.5, 1.0):
        a = oracle.forward(h_s, W_s, h_t, W_t, labels, beta, 1.4)
        b = oracle.forward(h_s, W_s, h_t, W_t, labels, beta, 1.4, side=True)
        for k in ("loss_tok", "lse_s", "lse_t", "aux"):
            np.testing.assert_array_equal(a[k], b[k])
        assert a["loss_mean"] == b["loss_mean"]
