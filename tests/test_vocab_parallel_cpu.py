"""Host logic of the vocabulary-parallel loss on CPU gloo ranks (world sizes 2 and 3).

Each rank holds a row shard of W_s and W_t; ``vp_forward`` / ``vp_backward`` run the real
collectives (all-gather of the shard states and JSD partials, all-reduce of dh_s) around the
CPU stand-in kernels of ``vp_cpu_kernels``; the result must equal the unsharded oracle. The
GPU kernels behind the same calls are compared with the oracle in ``test_vocab_parallel_gpu``.
"""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
from full_vocab_kl_b200.vocab_parallel import shard_range


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(seed, N=40, V=300, d_s=12, d_t=10, beta=1.0):
    rng = np.random.default_rng(seed)
    h_s = rng.standard_normal((N, d_s))
    h_t = rng.standard_normal((N, d_t))
    W_s = rng.standard_normal((V, d_s)) * 0.8
    W_t = 0.7 * W_s[:, :d_t] + 0.5 * rng.standard_normal((V, d_t))
    labels = rng.integers(0, V, N)
    labels[rng.choice(N, N // 4, replace=False)] = -100
    labels[0] = V - 1
    return h_s, W_s, h_t, W_t, labels


def _worker(rank, world, port, seed, beta, tau, align, out):
    import torch
    import torch.distributed as dist
    from vp_cpu_kernels import CpuKernels
    from full_vocab_kl_b200.vocab_parallel import vp_backward, vp_forward
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    h_s, W_s, h_t, W_t, labels = _problem(seed, beta=beta)
    v0, v1 = shard_range(W_s.shape[0], rank, world, align)
    T = torch.from_numpy
    k = CpuKernels()
    f = vp_forward(T(h_s), T(W_s[v0:v1]), T(h_t), T(W_t[v0:v1]), T(labels), beta, tau, vocab_offset=v0,
                   side=True, kernels=k)
    dh, dW = vp_backward(T(h_s), T(W_s[v0:v1]), T(h_t), T(W_t[v0:v1]), T(labels), beta, tau, f["lse_s"],
                         f["lse_t"], f["aux"], 0.8, kernels=k)
    res = {key: f[key].numpy().astype(np.float64) for key in
           ("loss_tok", "lse_s", "lse_t", "aux", "entropy_s", "logp_label")}
    res["loss_mean"] = float(f["loss_mean"])
    res["n_valid"] = int(f["n_valid"])
    res["dh"] = dh.numpy()
    res["dW"] = dW.numpy()
    res["range"] = (v0, v1)
    out[rank] = res
    dist.barrier()
    dist.destroy_process_group()


def test_shard_ranges_cover_the_vocabulary():
    for V in (256, 1000, 151936, 248320):
        for world in (1, 2, 3, 4, 8):
            if -(-V // 256) < world:
                continue
            r = [shard_range(V, k, world) for k in range(world)]
            assert r[0][0] == 0 and r[-1][1] == V
            assert all(r[k][1] == r[k + 1][0] for k in range(world - 1))
            assert all(a % 256 == 0 for a, _ in r)
            tiles = [-(-(b - a) // 256) for a, b in r]
            assert max(tiles) - min(tiles) <= 1 and min(tiles) > 0
    with pytest.raises(ValueError):
        shard_range(300, 0, 3)


@pytest.mark.parametrize("world,beta,tau", [(2, 1.0, 1.0), (2, 0.0, 0.7), (3, 0.5, 1.5), (3, 1.0, 2.0)])
def test_sharded_equals_unsharded(world, beta, tau):
    seed, align = 7, 16
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, seed, beta, tau, align, out), nprocs=world, join=True,
                       start_method="spawn")
    h_s, W_s, h_t, W_t, labels = _problem(seed, beta=beta)
    ref = oracle.forward(h_s, W_s, h_t, W_t, labels, beta, tau, side=True)
    refb = oracle.backward(h_s, W_s, h_t, W_t, labels, beta, tau, grad_out=0.8)
    valid = labels != -100
    for r in range(world):
        got = out[r]
        for key in ("loss_tok", "lse_s", "lse_t", "aux", "entropy_s", "logp_label"):
            np.testing.assert_allclose(got[key][valid], ref[key][valid], rtol=2e-5, atol=2e-6, err_msg=key)
            assert (got[key][~valid] == 0).all()
        assert got["n_valid"] == int(valid.sum())
        assert got["loss_mean"] == pytest.approx(ref["loss_mean"], rel=2e-5)
        np.testing.assert_allclose(got["dh"], refb["dh_s"], rtol=1e-4, atol=1e-7)
        # every rank holds the same per-token results (the merge runs in a fixed part order)
        for key in ("loss_tok", "lse_s", "entropy_s"):
            np.testing.assert_array_equal(got[key], out[0][key])
    dW = np.concatenate([out[r]["dW"] for r in range(world)])
    assert [out[r]["range"] for r in range(world)] == [shard_range(W_s.shape[0], r, world, align)
                                                       for r in range(world)]
    np.testing.assert_allclose(dW, refb["dW_s"], rtol=1e-4, atol=1e-7)


def test_exchange_format_composes_for_any_split():
    """The per-shard state (base-2 m, l, a, e and the label logit) merged in part order equals the
    unsharded oracle for arbitrary split points and shard counts (hypothesis over random problems);
    the CUDA combine kernel implements the same merge and is checked on the GPU."""
    from hypothesis import given, settings
    from hypothesis import strategies as st
    import torch
    from vp_cpu_kernels import CpuKernels

    @settings(max_examples=25, deadline=None, derandomize=True)
    @given(st.integers(0, 2 ** 31 - 1), st.integers(2, 60), st.integers(1, 5),
           st.sampled_from([0.0, 1.0, 0.3]), st.floats(0.3, 3.0))
    def check(seed, V, R, beta, tau):
        rng = np.random.default_rng(seed)
        N, d_s, d_t = 7, 5, 6
        h_s, h_t = rng.standard_normal((N, d_s)), rng.standard_normal((N, d_t))
        W_s, W_t = rng.standard_normal((V, d_s)), rng.standard_normal((V, d_t))
        labels = rng.integers(0, V, N)
        labels[0] = -100
        R = min(R, V)
        cuts = np.sort(rng.choice(np.arange(1, V), size=R - 1, replace=False)) if R > 1 else np.array([], int)
        edges = [0, *cuts.tolist(), V]
        k = CpuKernels()
        T = torch.from_numpy
        states = [k.state(T(h_s), T(W_s[a:b]), T(h_t), T(W_t[a:b]), T(labels), beta, tau, a, -100)[0]
                  for a, b in zip(edges[:-1], edges[1:])]
        out = k.combine(torch.stack(states), T(labels), beta, -100, True)
        if 0.0 < beta < 1.0:
            parts = [k.jsd_partial(T(h_s), T(W_s[a:b]), T(h_t), T(W_t[a:b]), T(labels), beta, tau,
                                   out["lse_s"], out["lse_t"], -100) for a, b in zip(edges[:-1], edges[1:])]
            out.update(k.jsd_combine(torch.stack(parts), T(labels), -100))
        ref = oracle.forward(h_s, W_s, h_t, W_t, labels, beta, tau, side=True)
        valid = labels != -100
        for key in ("loss_tok", "lse_s", "lse_t", "entropy_s", "logp_label"):
            np.testing.assert_allclose(out[key].numpy()[valid], ref[key][valid], rtol=3e-5, atol=3e-6,
                                       err_msg=key)

    check()


def _autograd_worker(rank, world, port, seed, beta, tau, out):
    import torch
    import torch.distributed as dist
    from vp_cpu_kernels import CpuKernels
    from full_vocab_kl_b200.vocab_parallel import vocab_parallel_jsd
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    h_s, W_s, h_t, W_t, labels = _problem(seed, beta=beta)
    v0, v1 = shard_range(W_s.shape[0], rank, world, 16)
    hs = torch.from_numpy(h_s).requires_grad_(True)
    Ws = torch.from_numpy(W_s[v0:v1].copy()).requires_grad_(True)
    loss = vocab_parallel_jsd(hs, torch.from_numpy(h_t), Ws, torch.from_numpy(W_t[v0:v1].copy()),
                              torch.from_numpy(labels), v0, beta, tau, kernels=CpuKernels())
    (0.8 * loss).backward()
    out[rank] = {"loss": float(loss), "dh": hs.grad.numpy(), "dW": Ws.grad.numpy(), "range": (v0, v1)}
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("beta", [1.0, 0.5])
def test_autograd_through_the_sharded_loss(beta):
    """loss.backward() on every rank: dh_s summed over the ranks, dW_s for the rank's own rows."""
    seed, world, tau = 3, 2, 1.3
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_autograd_worker, args=(world, port, seed, beta, tau, out), nprocs=world, join=True,
                       start_method="spawn")
    h_s, W_s, h_t, W_t, labels = _problem(seed, beta=beta)
    ref = oracle.forward(h_s, W_s, h_t, W_t, labels, beta, tau)
    refb = oracle.backward(h_s, W_s, h_t, W_t, labels, beta, tau, grad_out=0.8)
    for r in range(world):
        assert out[r]["loss"] == pytest.approx(ref["loss_mean"], rel=2e-5)
        np.testing.assert_allclose(out[r]["dh"], refb["dh_s"], rtol=1e-4, atol=1e-7)
        v0, v1 = out[r]["range"]
        np.testing.assert_allclose(out[r]["dW"], refb["dW_s"][v0:v1], rtol=1e-4, atol=1e-7)
