"""Spectral-compression front end on B200 against the oracle ("Nitrobrew tweet analysis":
thread item 6/8 and the "SVD-Nitrobrew" row of the evaluation table).

* nb_kl_gram (W^T W) and nb_kl_project (X B, bf16 out) element by element against float64
  products of the same bf16 inputs, on ragged shapes;
* the factor (Gram on the GPU, float64 eigendecomposition, bf16 basis): its subspace, singular
  values and compressed unembedding against the oracle's SVD of the same bf16 matrix;
* the loss on the compressed teacher: exact-input parity with the oracle, and the compressed
  logits against the oracle's rank-k teacher within the bf16 rounding of the three operands.
"""

import numpy as np
import pytest

import gpu_util as gu
import oracle
from oracle import spectral as osp
from synthetic import bf16_bits_to_f32, gaussian_bf16, make_custom, matrix_with_spectrum

pytestmark = pytest.mark.gpu


def _dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _host(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _f64(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


def _status_ok():
    import torch
    torch.cuda.synchronize()


@pytest.mark.parametrize("rows,d", [(1000, 136), (3000, 256), (20000, 520)])
def test_gram(rows, d):
    from full_vocab_kl_b200 import spectral
    X = gaussian_bf16(rows, d, 0.05, seed=rows)
    G = spectral.gram(_dev(X)).cpu().numpy().astype(np.float64)
    _status_ok()
    Xf = _f64(X)
    ref = Xf.T @ Xf
    # fp32 accumulator, one add per 16-term MMA step: worst case (K / 16 + 16) rounding
    # (truncating) errors of at most 2^-23 of the running sum of |products|
    absum = np.abs(Xf).T @ np.abs(Xf)
    bound = (rows / 16 + 16) * 2.0 ** -23 * absum
    err = np.abs(G - ref)
    assert (err <= bound).all(), (err / bound).max()
    # and in the usual sense: small relative to the row norms
    assert (err / np.sqrt(np.outer(np.diag(ref), np.diag(ref)))).max() <= 2e-4


@pytest.mark.parametrize("rows,d,k", [(300, 200, 72), (1000, 256, 8), (513, 64, 264), (4096, 2560, 512)])
def test_project(rows, d, k):
    from full_vocab_kl_b200 import spectral
    X = gaussian_bf16(rows, d, 1.0, seed=1)
    B = gaussian_bf16(d, k, 1.0 / np.sqrt(d), seed=2)
    Y = _host(spectral.project(_dev(X), _dev(B)))
    _status_ok()
    Xf, Bf = _f64(X), _f64(B)
    ref = Xf @ Bf
    got = _f64(Y)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * np.outer(np.linalg.norm(Xf, axis=1), np.linalg.norm(Bf, axis=0))
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{bad.sum()} elements off"


def _f64_to_bf16_bits(x):
    """bf16 bit patterns of float64 values rounded to nearest even in one step (normal range)."""
    b = np.ascontiguousarray(x, dtype=np.float64).view(np.uint64)
    lsb = (b >> np.uint64(45)) & np.uint64(1)
    r = (b + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    return (r.view(np.float64).astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


@pytest.mark.parametrize("d,k", [(200, 40), (64, 64), (1, 1), (520, 8)])
def test_select_basis_exact(d, k):
    """nb_kl_spectral_select against a plain host selection: the k largest eigenvalues (ties by
    index, NaN last), their eigenvector columns exactly, bf16 by one rounding, sqrt(max(l, 0))."""
    import torch
    from full_vocab_kl_b200 import spectral
    rng = np.random.default_rng(d * 1000 + k)
    evals = rng.standard_normal(d) * 5.0
    if d >= 8:
        evals[3] = evals[5]                  # a tie
        evals[6] = np.nan
        evals[7] = -abs(evals[7])            # negative: sigma clamps to 0
    evecs = rng.standard_normal((d, d))
    V_k, sigma, V64 = spectral.select_basis(torch.from_numpy(evals).cuda(), torch.from_numpy(evecs).cuda(), k)
    torch.cuda.synchronize()
    key = np.where(np.isnan(evals), -np.inf, evals)
    order = sorted(range(d), key=lambda i: (-key[i], i))[:k]
    np.testing.assert_array_equal(V64.cpu().numpy(), evecs[:, order])
    np.testing.assert_array_equal(_host(V_k), _f64_to_bf16_bits(evecs[:, order]))
    np.testing.assert_array_equal(sigma.cpu().numpy(), np.sqrt(np.maximum(evals[order], 0.0)))   # NaN stays NaN


def test_factor_matches_oracle_svd():
    from full_vocab_kl_b200 import spectral
    V, d, k = 20000, 256, 64
    sigma = np.concatenate([np.linspace(12.0, 6.0, k), np.linspace(1.0, 0.05, d - k)])
    W = matrix_with_spectrum(V, d, sigma, seed=3)
    basis = spectral.spectral_factor(_dev(W), k)
    _status_ok()
    Vref, sref = osp.spectral_basis(W, k)
    Vg = basis.V_k_f64.cpu().numpy()
    # the Gram matrix's error bound (see test_gram) carried to the factor: Weyl for the
    # eigenvalues (|d lambda| <= ||dG||_2 <= ||dG||_F, so |d sigma| <= ||dG||_F / (2 sigma)),
    # Davis-Kahan for the subspace (||dP||_F <= sqrt(2) ||dG||_F / gap)
    Wf = _f64(W)
    dG = np.linalg.norm((V / 16 + 16) * 2.0 ** -23 * (np.abs(Wf).T @ np.abs(Wf)))
    _, s_all, _ = np.linalg.svd(Wf, full_matrices=False)
    gap = s_all[k - 1] ** 2 - s_all[k] ** 2
    assert np.linalg.norm(Vg @ Vg.T - Vref @ Vref.T) <= np.sqrt(2.0) * dG / gap
    assert (np.abs(basis.sigma.cpu().numpy() - sref) <= dG / (2.0 * sref)).all()
    # the compressed unembedding is W times the (bf16) basis the GPU returned
    Vk = _host(basis.V_k)
    ref = _f64(W) @ _f64(Vk)
    got = _f64(_host(basis.W_code))
    bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * np.linalg.norm(_f64(W), axis=1)[:, None]
    assert (np.abs(got - ref) <= bound).all()


@pytest.mark.parametrize("beta,k", [(1.0, 128), (0.0, 128), (0.5, 64), (1.0, 512)])
def test_compressed_teacher_loss(beta, k):
    import torch
    import full_vocab_kl_b200 as nb
    from full_vocab_kl_b200 import spectral
    x = make_custom(512, 256, 512, 4096, beta, 1.0, n_masked=64, teacher="correlated")
    basis = spectral.spectral_factor(_dev(x.W_t), k)
    h_code = spectral.teacher_code(_dev(x.h_t), basis)
    t = gu.torch_inputs(x)
    f = nb.kl_forward(t["h_s"], t["W_s"], h_code, basis.W_code, t["labels"], beta, 1.0)
    torch.cuda.synchronize()
    assert nb.device_status(f["workspace"]) == 0
    got = {key: f[key].cpu().numpy().astype(np.float64) for key in ("loss_tok", "lse_s", "lse_t", "aux")}
    got["loss_mean"] = float(f["loss_mean"].item())
    got["n_valid"] = int(f["n_valid"].item())
    hc, Wc = _host(h_code), _host(basis.W_code)
    # 1) the loss on the compressed pair the GPU produced: ordinary parity
    ref = oracle.forward(x.h_s, x.W_s, hc, Wc, x.labels, beta, 1.0)
    gu.check_forward(got, ref, x.labels)
    # 2) the compressed teacher logits against the oracle's rank-k teacher (float64 basis):
    #    within the bf16 rounding of V_k, W_t V_k and h_t V_k (3 x 2^-9 relative)
    rows = np.flatnonzero(x.labels != -100)[:64]
    h_ref, W_ref, _ = osp.compress_teacher(x.h_t[rows], x.W_t, k)
    z_ref = h_ref @ W_ref.T
    z_got = _f64(hc[rows]) @ _f64(Wc).T
    assert np.linalg.norm(z_got - z_ref) <= 1e-2 * np.linalg.norm(z_ref)


def test_full_rank_code_is_nearly_lossless():
    from full_vocab_kl_b200 import spectral
    x = make_custom(256, 128, 256, 2048, 1.0, 1.0, n_masked=0, teacher="correlated")
    basis = spectral.spectral_factor(_dev(x.W_t), 256)
    hc = _host(spectral.teacher_code(_dev(x.h_t), basis))
    _status_ok()
    z = _f64(x.h_t) @ _f64(x.W_t).T
    zc = _f64(hc) @ _f64(_host(basis.W_code)).T
    assert np.linalg.norm(zc - z) <= 1e-2 * np.linalg.norm(z)


@pytest.mark.fullsize
def test_teacher_code_full_size():
    """The per-step projection at the spectral workload's size (32768 tokens, d_t 4096 -> 512),
    checked on sampled rows."""
    from full_vocab_kl_b200 import spectral
    N, d, k = 32768, 4096, 512
    X = gaussian_bf16(N, d, 1.0, seed=11)
    B = gaussian_bf16(d, k, 1.0 / np.sqrt(d), seed=12)
    Y = _host(spectral.project(_dev(X), _dev(B)))
    _status_ok()
    rows = np.random.default_rng(0).choice(N, 64, replace=False)
    ref = _f64(X[rows]) @ _f64(B)
    got = _f64(Y[rows])
    bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * np.outer(np.linalg.norm(_f64(X[rows]), axis=1),
                                                      np.linalg.norm(_f64(B), axis=0))
    assert (np.abs(got - ref) <= bound).all()
