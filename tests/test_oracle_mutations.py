"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins catch each one."""

import math

import numpy as np
import pytest

import oracle
import oracle.kl_oracle as ko
import test_oracle_pins as pins


def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def test_swapped_mixture_weights_caught(monkeypatch):
    monkeypatch.setattr(ko, "_log_mixture",
                        lambda lS, lT, b: np.logaddexp(math.log(b) + lS, math.log1p(-b) + lT))
    assert _fails(pins.test_bernoulli_v2, 0.3, -1.2)


def test_swapped_jsd_term_weights_caught(monkeypatch):
    orig = ko.divergence_rows

    def bad(lS, lT, beta):
        if beta in (0.0, 1.0):
            return orig(lS, lT, beta)
        lM = ko._log_mixture(lS, lT, beta)
        ks, kt = ko._kl_rows(lS, lM), ko._kl_rows(lT, lM)
        return (1 - beta) * kt + beta * ks, ks

    monkeypatch.setattr(ko, "divergence_rows", bad)
    assert _fails(pins.test_bernoulli_v2, 0.3, -1.2)


def test_temperature_after_softmax_caught(monkeypatch):
    orig = ko.tempered_logits
    monkeypatch.setattr(ko, "tempered_logits", lambda h, W, tau: orig(h, W, 1.0))
    assert _fails(pins.test_toy_v5_temperature_inside_softmax)


def test_reversed_kl_direction_caught(monkeypatch):
    orig = ko.divergence_rows
    monkeypatch.setattr(ko, "divergence_rows",
                        lambda lS, lT, b: orig(lS, lT, 1.0 - b) if b in (0.0, 1.0) else orig(lS, lT, b))
    assert _fails(pins.test_toy_v5_tau1)


@pytest.mark.parametrize("beta", [0.0, 1.0, 0.5])
def test_gradient_slips_caught(monkeypatch, beta):
    orig = ko.dloss_du_student

    def dropped_term(lS, lT, b, loss, aux):
        S = np.exp(lS)
        if b == 0.0:
            return np.exp(lT) - S                      # sign flipped
        if b == 1.0:
            return S * (lS - lT)                       # "- KL" dropped
        return orig(lS, lT, b, loss, np.zeros_like(aux))  # "- K" dropped

    monkeypatch.setattr(ko, "dloss_du_student", dropped_term)
    assert pins._fd_check(beta, 0.7) > 1e-3


def test_missing_inverse_tau_in_gradient_caught(monkeypatch):
    orig = ko.backward

    def bad(*a, **k):
        out = orig(*a, **k)
        tau = a[6]
        out["dh_s"] *= tau
        if out["dW_s"] is not None:
            out["dW_s"] *= tau
        return out

    monkeypatch.setattr(oracle, "backward", bad)
    monkeypatch.setattr(pins.oracle, "backward", bad)
    assert pins._fd_check(1.0, 0.7) > 1e-3


def test_mean_over_all_rows_caught(monkeypatch):
    orig = ko.forward

    def bad(*a, **k):
        out = orig(*a, **k)
        if out["loss_mean"] is not None and out["n_valid"]:
            out["loss_mean"] = float(out["loss_tok"].sum() / len(a[4]))
        return out

    monkeypatch.setattr(pins.oracle, "forward", bad)
    assert _fails(pins.test_brute_force_tiny, 1.0, 1.0)


def test_lse_missing_log_caught(monkeypatch):
    def bad(u):
        m = u.max(axis=1, keepdims=True)
        lse = m + np.exp(u - m).sum(axis=1, keepdims=True)
        return u - lse, lse[:, 0]

    monkeypatch.setattr(ko, "log_softmax", bad)
    assert _fails(pins.test_lse_zero_weights_is_log_v)


# ------------------------------------------------------------------ side outputs
import test_oracle_side_pins as side_pins  # noqa: E402


def _side_mutant(monkeypatch, fn):
    orig = ko.student_side_rows
    monkeypatch.setattr(ko, "student_side_rows", lambda lS, lab: fn(orig, lS, lab))


def test_entropy_sign_slip_caught(monkeypatch):
    _side_mutant(monkeypatch, lambda o, lS, lab: (-o(lS, lab)[0], o(lS, lab)[1]))
    assert _fails(side_pins.test_uniform_student)


def test_entropy_in_bits_caught(monkeypatch):
    _side_mutant(monkeypatch, lambda o, lS, lab: (o(lS, lab)[0] / math.log(2.0), o(lS, lab)[1]))
    assert _fails(side_pins.test_two_level_closed_form, 3, 2.0, -1.0, 2.0)


def test_label_off_by_one_caught(monkeypatch):
    _side_mutant(monkeypatch, lambda o, lS, lab: o(lS, np.minimum(np.asarray(lab) + 1, lS.shape[1] - 1)))
    assert _fails(side_pins.test_brute_force_tiny, 1.0, 12)


def test_logp_without_normaliser_caught(monkeypatch):
    # log-probabilities read from the tempered logits themselves (u instead of u - lse)
    def raw(u):
        m = u.max(axis=1, keepdims=True)
        lse = m + np.log(np.exp(u - m).sum(axis=1, keepdims=True))
        return u, lse[:, 0]

    monkeypatch.setattr(ko, "log_softmax", raw)
    assert _fails(side_pins.test_two_level_closed_form, 3, 2.0, -1.0, 2.0)


def test_untempered_side_outputs_caught(monkeypatch):
    # at tau = 2: logS * 2 re-normalised is the softmax of z itself
    _side_mutant(monkeypatch, lambda o, lS, lab: o(ko.log_softmax(lS * 2.0)[0], lab))
    assert _fails(side_pins.test_two_level_closed_form, 3, 2.0, -1.0, 2.0)


# ------------------------------------------------------------------ spectral front end
import oracle.spectral as spo  # noqa: E402
import test_oracle_spectral_pins as spec_pins  # noqa: E402


def test_smallest_singular_vectors_caught(monkeypatch):
    def bad(W, k):
        W = np.asarray(W, dtype=np.float64)
        _, s, vt = np.linalg.svd(W, full_matrices=False)
        return vt[-k:][::-1].T.copy(), s[-k:][::-1].copy()
    monkeypatch.setattr(spo, "spectral_basis", bad)
    assert _fails(spec_pins.test_top_subspace_and_eckart_young)


def test_transposed_singular_factor_caught(monkeypatch):
    # columns of V^T taken where the rows were meant (a transposition slip)
    def bad(W, k):
        W = np.asarray(W, dtype=np.float64)
        _, s, vt = np.linalg.svd(W, full_matrices=False)
        return vt[:, :k].copy(), s[:k].copy()
    monkeypatch.setattr(spo, "spectral_basis", bad)
    assert _fails(spec_pins.test_top_subspace_and_eckart_young)


def test_truncated_coordinates_instead_of_projection_caught(monkeypatch):
    # keeping the first k coordinates of h instead of its coordinates in the basis
    monkeypatch.setattr(spo, "project", lambda x, Vk: np.asarray(x, dtype=np.float64)[:, :Vk.shape[1]])
    assert _fails(spec_pins.test_full_rank_and_exact_low_rank_are_lossless)


def test_unscaled_teacher_unembedding_caught(monkeypatch):
    # W_t' = U_k instead of U_k S_k: drop the singular values
    orig = spo.compress_teacher

    def bad(h, W, k):
        hp, Wp, Vk = orig(h, W, k)
        return hp, Wp / np.linalg.norm(Wp, axis=0, keepdims=True), Vk
    monkeypatch.setattr(spo, "compress_teacher", bad)
    assert _fails(spec_pins.test_closed_form_diagonal)


# ------------------------------------------------------------------ partial paths
import test_oracle_subset_pins as subset_pins  # noqa: E402


def test_dropped_dW_init_caught(monkeypatch):
    # an accumulating backward that starts dW_s from zero instead of the caller's start value
    orig = ko.backward

    def bad(*a, dW_init=None, **k):
        return orig(*a, **k)

    monkeypatch.setattr(subset_pins.oracle, "backward", bad)
    assert _fails(subset_pins.test_dW_init_is_added_to_the_gradient, 1.0)


def test_mean_over_sampled_rows_caught(monkeypatch):
    # normalising by the number of positions evaluated instead of N_v
    orig = ko._selected_rows

    def bad(labels, ignore_index, rows):
        valid, todo, _ = orig(labels, ignore_index, rows)
        return valid, todo, int(todo.size)

    monkeypatch.setattr(ko, "_selected_rows", bad)
    assert _fails(subset_pins.test_rows_subset_backward_uses_all_valid_rows, 0.35)


def test_rows_subset_ignored_caught(monkeypatch):
    # a forward that evaluates every valid position whatever `rows` says
    orig = ko._selected_rows
    monkeypatch.setattr(ko, "_selected_rows", lambda labels, ii, rows: orig(labels, ii, None))
    assert _fails(subset_pins.test_rows_subset_forward_matches_brute_force, 1.0)
