"""Regression anchor: generator bytes and oracle outputs on the 128-token workload."""

import json
import os

import numpy as np
import pytest

import oracle
from synthetic import make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.json")


def test_tiny_golden():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "make_golden", os.path.join(os.path.dirname(__file__), "golden", "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    with open(GOLDEN) as f:
        g = json.load(f)
    x = make_inputs("tiny", seed=0)
    assert mg.input_hashes(x) == g["hashes"]
    fw = oracle.forward(x.h_s, x.W_s, x.h_t, x.W_t, x.labels, x.beta, x.tau, side=True)
    assert fw["n_valid"] == g["n_valid"] == 96
    np.testing.assert_allclose(fw["entropy_s"][32:40], g["entropy_s_first8_valid"], rtol=1e-12)
    np.testing.assert_allclose(fw["logp_label"][32:40], g["logp_label_first8_valid"], rtol=1e-12)
    assert fw["loss_mean"] == pytest.approx(g["loss_mean"], rel=1e-12)
    np.testing.assert_allclose(fw["loss_tok"][32:40], g["loss_tok_first8_valid"], rtol=1e-12)
    np.testing.assert_allclose(fw["lse_s"][32:40], g["lse_s_first8_valid"], rtol=1e-13)
    bw = oracle.backward(x.h_s, x.W_s, x.h_t, x.W_t, x.labels, x.beta, x.tau)
    assert np.linalg.norm(bw["dh_s"]) == pytest.approx(g["dh_s_fro"], rel=1e-11)
    assert np.linalg.norm(bw["dW_s"]) == pytest.approx(g["dW_s_fro"], rel=1e-11)


def test_generator_shapes_and_masks():
    x = make_inputs("tiny", seed=0)
    assert x.h_s.dtype == np.float32 and x.W_s.dtype == np.uint16
    assert (x.labels[:32] == -100).all() and (x.labels[32:] >= 0).all()
    y = make_inputs("tiny", seed=1)
    assert not np.array_equal(x.W_s, y.W_s)
