"""Property-based checks of the oracle on random small problems (hypothesis): invariants the
mathematics fixes whatever the inputs, complementing the point pins.

"03 White-box OPD", section 2.3 (the beta table, temperature inside the softmax) and
"01 · 论文精读与参考实现全景映射", section 1 (Eq. 6 and Eq. 8, the side outputs).
"""

import math

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

# derandomized: the same examples on every run, so the CPU suite is reproducible
SETTINGS = settings(max_examples=40, deadline=None, derandomize=True)


def problem(seed, N, V, d_s, d_t, scale):
    rng = np.random.default_rng(seed)
    h_s = rng.standard_normal((N, d_s))
    h_t = rng.standard_normal((N, d_t))
    W_s = rng.standard_normal((V, d_s)) * scale / math.sqrt(d_s)
    W_t = rng.standard_normal((V, d_t)) * scale / math.sqrt(d_t)
    labels = rng.integers(0, V, N)
    labels[rng.random(N) < 0.3] = -100
    return h_s, W_s, h_t, W_t, labels


dims = st.tuples(st.integers(0, 2 ** 31 - 1), st.integers(1, 6), st.integers(2, 40), st.integers(1, 6),
                 st.integers(1, 6), st.floats(0.1, 8.0))
betas = st.one_of(st.sampled_from([0.0, 1.0]), st.floats(0.01, 0.99))
taus = st.floats(0.25, 4.0)


def binary_entropy(b):
    return -(b * math.log(b) + (1 - b) * math.log(1 - b)) if 0 < b < 1 else 0.0


@SETTINGS
@given(dims, betas, taus)
def test_divergence_bounds(d, beta, tau):
    """0 <= loss; the JSD is at most the binary entropy of beta; masked rows are 0."""
    h_s, W_s, h_t, W_t, labels = problem(*d)
    out = oracle.forward(h_s, W_s, h_t, W_t, labels, beta, tau)
    valid = labels != -100
    assert (out["loss_tok"][valid] >= -1e-12).all()
    if 0.0 < beta < 1.0:
        assert (out["loss_tok"][valid] <= binary_entropy(beta) + 1e-12).all()
    assert (out["loss_tok"][~valid] == 0).all()
    if valid.any():
        assert math.isclose(out["loss_mean"], float(np.mean(out["loss_tok"][valid])), rel_tol=1e-12)


@SETTINGS
@given(dims, betas, taus)
def test_identical_models_give_zero(d, beta, tau):
    h_s, W_s, _, _, labels = problem(*d)
    out = oracle.forward(h_s, W_s, h_s.copy(), W_s.copy(), labels, beta, tau)
    assert np.abs(out["loss_tok"]).max() <= 1e-12


@SETTINGS
@given(dims, taus, st.floats(-5.0, 5.0))
def test_lse_shift_equivariance_and_side_bounds(d, tau, c):
    """A constant logit shift c (a column of W times a fixed coordinate) moves the LSE by c/tau
    and leaves the distribution, hence entropy and label log-probabilities, unchanged;
    0 <= H <= log V and log p <= 0."""
    h_s, W_s, h_t, W_t, labels = problem(*d)
    a = oracle.forward(h_s, W_s, h_t, W_t, labels, 1.0, tau, side=True)
    # append a coordinate that is 1 in every hidden row and c in every unembedding row
    hs1 = np.hstack([h_s, np.ones((h_s.shape[0], 1))])
    Ws1 = np.hstack([W_s, np.full((W_s.shape[0], 1), c)])
    b = oracle.forward(hs1, Ws1, h_t, W_t, labels, 1.0, tau, side=True)
    valid = labels != -100
    np.testing.assert_allclose(b["lse_s"][valid], a["lse_s"][valid] + c / tau, rtol=1e-12, atol=1e-11)
    for k in ("entropy_s", "logp_label", "loss_tok"):
        np.testing.assert_allclose(b[k][valid], a[k][valid], rtol=1e-10, atol=1e-11)
    V = W_s.shape[0]
    assert (a["entropy_s"][valid] >= -1e-12).all() and (a["entropy_s"][valid] <= math.log(V) + 1e-12).all()
    assert (a["logp_label"][valid] <= 1e-12).all()


@SETTINGS
@given(dims, betas, taus, st.floats(0.1, 3.0))
def test_gradient_is_linear_in_grad_out_and_rows_sum_to_zero(d, beta, tau, g):
    """dh and dW scale with grad_out; every row of the logit gradient G sums to 0 over the
    vocabulary (it is a softmax derivative), so sum_v dW[v] = (G 1)^T h = 0."""
    h_s, W_s, h_t, W_t, labels = problem(*d)
    b1 = oracle.backward(h_s, W_s, h_t, W_t, labels, beta, tau, grad_out=1.0)
    bg = oracle.backward(h_s, W_s, h_t, W_t, labels, beta, tau, grad_out=g)
    np.testing.assert_allclose(bg["dh_s"], g * b1["dh_s"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(bg["dW_s"], g * b1["dW_s"], rtol=1e-12, atol=1e-14)
    # the row sums of G vanish only up to rounding of its terms (|G| |h| summed): an absolute
    # floor far below any gradient a slip would leave behind
    col = np.abs(b1["dW_s"].sum(axis=0)).max()
    scale = np.abs(b1["dW_s"]).sum(axis=0).max() + 1e-300
    assert col <= 1e-10 * scale + 1e-13


@SETTINGS
@given(st.integers(0, 2 ** 31 - 1), st.integers(2, 30), taus)
def test_temperature_acts_on_logits(seed, V, tau):
    """Scaling W by 1/tau at tau' = 1 equals tau on W (temperature divides the logits)."""
    h_s, W_s, h_t, W_t, labels = problem(seed, 3, V, 4, 5, 2.0)
    a = oracle.forward(h_s, W_s, h_t, W_t, labels, 1.0, tau, side=True)
    b = oracle.forward(h_s, W_s / tau, h_t, W_t / tau, labels, 1.0, 1.0, side=True)
    for k in ("loss_tok", "lse_s", "lse_t", "entropy_s", "logp_label"):
        np.testing.assert_allclose(a[k], b[k], rtol=1e-10, atol=1e-12)
