"""Element-by-element parity of the CUDA path with the fp64 oracle on the same seeded
inputs, at sizes the oracle finishes in seconds that still span several 128-row token
tiles, several vocabulary tiles and splits, ragged tails in every dimension, and the
degenerate cases of the method."""

import numpy as np
import pytest

import gpu_util as gu
import oracle
from synthetic import make_custom, make_inputs

pytestmark = pytest.mark.gpu


def full_check(x, chunk_v=0, beta=None, tau=None, labels=None, dW_init=None):
    got = gu.run_library(x, chunk_v=chunk_v, beta=beta, tau=tau, labels=labels, dW_init=dW_init)
    ref = gu.oracle_all(x, beta=beta, tau=tau, labels=labels, dW_init=dW_init)
    lab = x.labels if labels is None else labels
    gu.check_forward(got, ref, lab)
    e_dh = gu.rel_l2(got["dh_s"], ref["dh_s"])
    e_dw = gu.rel_l2(got["dW_s"], ref["dW_s"])
    assert e_dh <= gu.TOL_GRAD, f"dh_s rel L2 {e_dh}"
    assert e_dw <= gu.TOL_GRAD, f"dW_s rel L2 {e_dw}"
    masked = lab == -100
    assert (got["dh_s"][masked] == 0).all()
    return got, ref


def test_tiny_workload():
    """128 tokens, d 256/384, V 4096 (two splits), fp32 hidden states, reverse KL."""
    full_check(make_inputs("tiny"))


@pytest.mark.parametrize("beta", [1.0, 0.5])
def test_token_groups_of_the_work_order(beta):
    """Wide rows (d_s = d_t = 4096: 4 MB of compacted rows per 256-token tile) put the sweeps'
    work order in groups of 10 token tiles: 5400 valid rows are 22 tiles, two full groups and a
    remainder of 2; every row against the oracle, forward and backward (JSD: all three sweeps)."""
    x = make_custom(5600, 4096, 4096, 1000, beta, 1.0, n_masked=200, teacher="independent")
    full_check(x)


@pytest.mark.parametrize("beta", [0.0, 1.0, 0.5, 0.3])
def test_ragged_all_dims(beta):
    # 300 rows (tail of 44 rows), V 1000 (tail tile of 104 columns), K tails of 8 and 8
    x = make_custom(300, 200, 136, 1000, beta, 1.0, n_masked=37, teacher="independent")
    full_check(x)


@pytest.mark.parametrize("tau", [0.5, 2.0])
@pytest.mark.parametrize("beta", [0.0, 1.0, 0.5])
def test_temperatures(beta, tau):
    x = make_custom(256, 128, 192, 2048, beta, tau, n_masked=50, teacher="correlated")
    full_check(x)


@pytest.mark.parametrize("beta", [0.0, 1.0, 0.6])
def test_multi_chunk_backward(beta):
    # chunk_v 256 -> 8 chunks, the last one ragged (V = 1900)
    x = make_custom(384, 256, 256, 1900, beta, 1.0, n_masked=100, teacher="correlated")
    full_check(x, chunk_v=256)


def test_many_token_tiles_and_splits():
    # 1100 rows (800 valid: 4 pair tiles, the last ragged), V 5000 (20 vocabulary tiles, the last
    # one ragged; every tile its own split)
    x = make_custom(1100, 256, 320, 5000, 1.0, 1.0, n_masked=300, teacher="correlated")
    full_check(x)


@pytest.mark.parametrize("beta", [1.0, 0.0, 0.5])
def test_multi_tile_units_and_single_tail(beta):
    """8192 positions (32 token tiles on the host side, so the last ~160 work items are the
    last 5 vocabulary tiles of each token tile), 5192 valid rows (21 pair tiles, the last
    ragged), V 4000 (16 vocabulary tiles, the last ragged): the forward and JSD sweeps run one
    8-tile unit and then single tiles, the gradient sweep two 4-tile units and then single
    tiles; every row against the oracle."""
    x = make_custom(8192, 64, 96, 4000, beta, 1.0, n_masked=3000, teacher="correlated")
    full_check(x)


def test_no_valid_rows():
    x = make_custom(200, 128, 128, 1024, 1.0, 1.0, n_masked=200)
    got = gu.run_library(x)
    assert got["n_valid"] == 0 and got["loss_mean"] == 0.0
    for k in ("loss_tok", "lse_s", "lse_t", "aux", "dh_s", "dW_s"):
        assert not got[k].any(), k


def test_all_rows_valid():
    x = make_custom(256, 128, 128, 1536, 0.0, 1.0, n_masked=0, teacher="correlated")
    full_check(x)


@pytest.mark.parametrize("beta", [0.0, 1.0, 0.5])
def test_identical_models_give_zero(beta):
    x = make_custom(256, 192, 192, 2000, beta, 1.3, n_masked=20)
    x.h_t, x.W_t = x.h_s.copy(), x.W_s.copy()
    got = gu.run_library(x)
    valid = x.labels != -100
    assert np.abs(got["loss_tok"][valid]).max() <= 1e-5
    assert abs(got["loss_mean"]) <= 1e-5
    np.testing.assert_allclose(got["lse_s"], got["lse_t"], rtol=1e-6)
    assert np.abs(got["dh_s"]).max() <= 1e-6 and np.abs(got["dW_s"]).max() <= 1e-6


def test_boosted_rows_lse_stability():
    # one logit raised by +40 on 10% of the rows (a near one-hot peak after tau = 0.5)
    x = make_custom(512, 256, 256, 3000, 0.5, 0.5, n_masked=64, teacher="correlated",
                    boost_frac=0.1, boost=40.0)
    full_check(x)


def test_fp32_hidden_states_all_betas():
    for beta in (0.0, 0.5):
        x = make_custom(200, 128, 192, 1500, beta, 1.0, n_masked=30, h_dtype="f32")
        full_check(x)


def test_accumulate_dW():
    x = make_custom(256, 128, 128, 1100, 1.0, 1.0, n_masked=40, teacher="correlated")
    init = np.random.default_rng(5).standard_normal((1100, 128)).astype(np.float32) * 1e-3
    full_check(x, dW_init=init)


def test_spectral_shape_small():
    x = make_custom(256, 512, 64, 2048, 1.0, 1.0, n_masked=90, teacher="spectral")
    full_check(x)


def test_grad_out_scaling():
    x = make_custom(256, 128, 128, 1024, 1.0, 1.0, n_masked=40, teacher="correlated")
    x.grad_out = -2.5
    full_check(x)


def test_autograd_api_matches_oracle():
    import torch
    import full_vocab_kl_b200 as nb
    x = make_custom(256, 128, 192, 1500, 1.0, 1.0, n_masked=40, teacher="correlated")
    t = gu.torch_inputs(x)
    hs = t["h_s"].clone().requires_grad_(True)
    Ws = t["W_s"].clone().requires_grad_(True)
    loss = nb.reverse_kl(hs[None], t["h_t"][None], Ws, t["W_t"], labels=t["labels"][None])
    loss.backward()
    ref = gu.oracle_all(x)
    assert abs(loss.item() - ref["loss_mean"]) <= 1e-3 * abs(ref["loss_mean"])
    assert gu.rel_l2(hs.grad.float().cpu().numpy(), ref["dh_s"]) <= 2e-2  # bf16 cast of dh
    assert gu.rel_l2(Ws.grad.float().cpu().numpy(), ref["dW_s"]) <= 2e-2


def test_repeatable():
    x = make_custom(300, 128, 128, 1200, 0.5, 1.0, n_masked=37)
    a = gu.run_library(x)
    b = gu.run_library(x)
    for k in ("loss_tok", "lse_s", "aux", "dh_s", "dW_s"):
        np.testing.assert_array_equal(a[k], b[k])
    assert a["loss_mean"] == b["loss_mean"]


@pytest.mark.parametrize("V", [100, 2148, 4224])
@pytest.mark.parametrize("beta", [0.0, 1.0, 0.5])
def test_vocab_tail_leaves_whole_column_halves_empty(V, beta):
    # V mod 2048 <= 128 (or V <= 128): the last work unit's only tile has a column half that
    # lies entirely past the vocabulary, so some epilogue threads start on an all-masked chunk
    x = make_custom(300, 128, 192, V, beta, 0.7, n_masked=40, teacher="correlated")
    full_check(x)


def test_empty_input():
    """n_tokens = 0: loss 0, N_v 0, dW_s overwritten with zeros, no launch of a sweep."""
    import torch
    import full_vocab_kl_b200 as nb
    z = lambda *s: torch.zeros(s, dtype=torch.bfloat16, device="cuda")  # noqa: E731
    h_s, h_t, W_s, W_t = z(0, 128), z(0, 192), z(512, 128), z(512, 192)
    lab = torch.zeros(0, dtype=torch.int64, device="cuda")
    f = nb.kl_forward(h_s, W_s, h_t, W_t, lab, 0.5, 1.0, side=True)
    dW = torch.full((512, 128), 3.0, device="cuda")
    dh, dW = nb.kl_backward(h_s, W_s, h_t, W_t, lab, 0.5, 1.0, f["lse_s"], f["lse_t"], f["aux"], 1.0,
                            dW_s=dW, workspace=f["workspace"])
    torch.cuda.synchronize()
    assert float(f["loss_mean"]) == 0.0 and int(f["n_valid"]) == 0
    assert dh.shape == (0, 128) and float(dW.abs().max()) == 0.0
    assert nb.device_status(f["workspace"]) == 0


@pytest.mark.parametrize("beta,tau", [(1.0, 1.0), (0.0, 1.0), (0.5, 2.0)])
def test_one_entry_vocabulary(beta, tau):
    """V = 1: both distributions are a point mass, so every divergence is 0 and so is its gradient
    (the 255 other columns of the only vocabulary tile are masked), while each LSE is the single
    tempered logit, compared with the oracle."""
    x = make_custom(300, 64, 96, 1, beta, tau, n_masked=44, teacher="independent")
    got = gu.run_library(x)
    ref = gu.oracle_all(x)
    valid = x.labels != -100
    assert got["n_valid"] == int(valid.sum())
    assert np.abs(got["loss_tok"][valid]).max() <= 1e-5 and abs(got["loss_mean"]) <= 1e-5
    for k in ("lse_s", "lse_t"):
        np.testing.assert_allclose(got[k][valid], ref[k][valid], rtol=gu.TOL_LSE, atol=1e-6)
    assert np.abs(got["dh_s"]).max() <= 1e-6 and np.abs(got["dW_s"]).max() <= 1e-6


@pytest.mark.parametrize("beta", [1.0, 0.0, 0.5])
def test_single_token(beta):
    """One position, valid: one 256-row token tile holding a single row, every row against the
    oracle, forward and backward."""
    x = make_custom(1, 64, 128, 300, beta, 1.0, n_masked=0, teacher="independent")
    full_check(x)
