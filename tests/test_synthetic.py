"""The seeded input generator delivers the recipe the design notes state: RMS-normalised hidden
rows, logits of standard deviation about c, the correlated teacher's z_t ~ 0.92 z_s + noise,
exact mask counts, boosted logits, and the rank-k spectral teacher code."""

import math

import numpy as np
import pytest

from synthetic import bf16_bits_to_f32, make_custom


def f(a):
    return a.astype(np.float64) if a.dtype != np.uint16 else bf16_bits_to_f32(a).astype(np.float64)


def test_hidden_rows_are_rms_normalised_and_logits_have_scale_c():
    x = make_custom(256, 256, 512, 2048, 1.0, 1.0, w_std=3.0, teacher="correlated", h_dtype="f32")
    for h in (x.h_s, x.h_t):
        ms = (f(h) ** 2).mean(axis=1)
        np.testing.assert_allclose(ms, 1.0, rtol=1e-3)
    z_s = f(x.h_s) @ f(x.W_s).T
    z_t = f(x.h_t) @ f(x.W_t).T
    assert z_s.std() == pytest.approx(3.0, rel=0.08)
    assert z_t.std() == pytest.approx(3.0, rel=0.08)


def test_correlated_teacher_slope():
    """h_t = RMSnorm(0.7 sqrt(d_t/d_s) Q h_s + 0.3 eps), W_t = sqrt(d_s/d_t) W_s Q^T + W_perp:
    the regression slope of z_t on z_s is 0.7 / sqrt(0.49 + 0.09) = 0.919."""
    x = make_custom(512, 256, 640, 2048, 1.0, 1.0, w_std=3.0, teacher="correlated", h_dtype="f32")
    z_s = (f(x.h_s) @ f(x.W_s).T).ravel()
    z_t = (f(x.h_t) @ f(x.W_t).T).ravel()
    slope = np.cov(z_s, z_t)[0, 1] / z_s.var()
    assert slope == pytest.approx(0.7 / math.sqrt(0.58), abs=0.02)


@pytest.mark.parametrize("mask", ["prefix", "random"])
def test_exact_mask_counts(mask):
    x = make_custom(300, 64, 64, 512, 1.0, 1.0, n_masked=77, mask=mask)
    masked = x.labels == -100
    assert masked.sum() == 77
    if mask == "prefix":
        assert masked[:77].all() and not masked[77:].any()
    valid = x.labels[~masked]
    assert valid.min() >= 0 and valid.max() < 512


def test_boosted_rows_carry_the_boost_on_both_models():
    x = make_custom(400, 128, 192, 2048, 0.5, 2.0, w_std=3.0, teacher="correlated", n_masked=100,
                    boost_frac=0.05, boost=20.0, h_dtype="f32")
    rows, ids = x.meta["boost_rows"], x.meta["boost_ids"]
    assert len(rows) == 20 and (x.labels[rows] != -100).all()
    for h, W in ((x.h_s, x.W_s), (x.h_t, x.W_t)):
        z = f(h[rows]) @ f(W).T
        # the boosted logit is its original value (std ~3) plus 20: the row's maximum
        assert (z.argmax(axis=1) == ids).all()
        assert (z[np.arange(len(rows)), ids] > 20.0 - 5 * 3.0).all()


def test_spectral_teacher_code_is_rank_k_with_descending_columns():
    x = make_custom(64, 256, 64, 4096, 1.0, 1.0, w_std=3.0, teacher="spectral")
    Wt = f(x.W_t)
    gram = Wt.T @ Wt
    norms = np.sqrt(np.diag(gram))
    assert (np.diff(norms) <= 1e-6 * norms[0] + 1e-2 * norms[:-1]).all()   # descending up to bf16
    off = gram - np.diag(np.diag(gram))
    assert np.abs(off).max() <= 1e-2 * gram.diagonal().max()                # orthogonal columns
