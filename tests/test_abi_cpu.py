"""Host-side checks of the C ABI that need no GPU: the library builds and loads, exports
every symbol the header declares, sizes its workspace O(tokens * chunk_V) and rejects bad
arguments synchronously (before touching any device)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from full_vocab_kl_b200 import build
    build.build()
    from full_vocab_kl_b200 import _abi
    return _abi


def header_functions():
    with open(os.path.join(ROOT, "include", "nb_kl.h")) as f:
        src = f.read()
    return sorted(set(re.findall(r"NB_KL_API\s+[\w\s\*]*?\b(nb_kl_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = header_functions()
    assert len(names) >= 8
    lib = L.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L.SIGNATURES)


def shape(L, N=8192, V=151936, ds=1024, dt=2560, dtype=0, chunk=0):
    return L.Shape(n_tokens=N, vocab=V, d_s=ds, d_t=dt, h_dtype=dtype, reserved=0, ignore_index=-100, chunk_v=chunk)


def ws_size(L, s, beta=1.0):
    return L.lib().nb_kl_workspace_size(L.shape_ptr(s), beta)


def test_workspace_scales_with_chunk_not_vocab(L):
    base = ws_size(L, shape(L, chunk=4096))
    assert base > 0
    # doubling V adds only the split-V state (5 floats per 2048 columns per row)
    big_v = ws_size(L, shape(L, V=2 * 151936, chunk=4096))
    assert big_v - base <= 5 * 4 * 8192 * (151936 // 2048 + 2) + 4096
    # the gradient chunk grows with chunk_v
    big_c = ws_size(L, shape(L, chunk=16384))
    assert big_c - base >= 8192 * (16384 - 4096) * 2 - 4096
    # never anywhere near N * V
    assert base < 8192 * 151936 * 2 / 4
    # JSD needs the extra partial sums
    assert ws_size(L, shape(L), 0.5) >= ws_size(L, shape(L), 1.0)


@pytest.mark.parametrize("bad", [dict(ds=100), dict(dt=12), dict(V=0), dict(N=-1), dict(dtype=3), dict(chunk=100)])
def test_invalid_shapes(L, bad):
    kw = dict(N=256, V=1000, ds=256, dt=256, dtype=0, chunk=0)
    kw.update(bad)
    assert ws_size(L, shape(L, **kw)) == 0


def test_status_strings(L):
    for code, text in ((0, "ok"), (-1, "invalid argument"), (-3, "workspace too small"), (-5, "device wait timed out")):
        assert L.status_string(code) == text


def _fwd(L, s, ptrs, beta=1.0, tau=1.0, ws_bytes=None):
    p = [ctypes.c_void_p(v) for v in ptrs]
    ws_bytes = ws_size(L, s, beta) if ws_bytes is None else ws_bytes
    return L.lib().nb_kl_forward(L.shape_ptr(s), p[0], p[1], p[2], p[3], p[4], beta, tau, p[5], p[6], p[7], p[8],
                                 p[9], p[10], p[11], ws_bytes, None)


FAKE = [0x10000 * (i + 1) for i in range(12)]  # 16-byte aligned, never dereferenced


@pytest.mark.parametrize("case", ["null_h", "misaligned_W", "beta", "tau", "tau_nan", "workspace"])
def test_forward_argument_errors(L, case):
    s = shape(L, N=256, V=1024, ds=256, dt=256)
    ptrs = list(FAKE)
    beta, tau, wsb = 1.0, 1.0, None
    if case == "null_h":
        ptrs[0] = 0
    elif case == "misaligned_W":
        ptrs[1] += 2
    elif case == "beta":
        beta = 1.5
    elif case == "tau":
        tau = 0.0
    elif case == "tau_nan":
        tau = float("nan")
    elif case == "workspace":
        wsb = 100
    code = _fwd(L, s, ptrs, beta, tau, wsb)
    assert code == (L.NB_ERR_WORKSPACE if case == "workspace" else L.NB_ERR_INVALID_ARG)


def test_backward_argument_errors(L):
    s = shape(L, N=256, V=1024, ds=256, dt=256)
    p = [ctypes.c_void_p(v) for v in FAKE]
    wsb = ws_size(L, s)
    lib = L.lib()
    # missing grad_out
    code = lib.nb_kl_backward(L.shape_ptr(s), p[0], p[1], p[2], p[3], p[4], 1.0, 1.0, p[5], p[6], p[7], None,
                              p[8], p[9], 0, p[10], wsb, None)
    assert code == L.NB_ERR_INVALID_ARG
    # beta out of range
    code = lib.nb_kl_backward(L.shape_ptr(s), p[0], p[1], p[2], p[3], p[4], -0.1, 1.0, p[5], p[6], p[7], p[11],
                              p[8], p[9], 0, p[10], wsb, None)
    assert code == L.NB_ERR_INVALID_ARG


def test_debug_entry_argument_errors(L):
    lib = L.lib()
    assert lib.nb_kl_debug_gemm(None, 0, ctypes.c_void_p(FAKE[1]), 0, 128, 128, 64, ctypes.c_void_p(FAKE[2]),
                                ctypes.c_void_p(FAKE[3]), None) == L.NB_ERR_INVALID_ARG
    assert lib.nb_kl_debug_gemm(ctypes.c_void_p(FAKE[0]), 0, ctypes.c_void_p(FAKE[1]), 0, 130, 128, 64,
                                ctypes.c_void_p(FAKE[2]), ctypes.c_void_p(FAKE[3]), None) == L.NB_ERR_INVALID_ARG
    assert lib.nb_kl_debug_wait_timeout(None, 1000, 0, None) == L.NB_ERR_INVALID_ARG
    assert lib.nb_kl_debug_wait_timeout(None, 1000, 1, None) == L.NB_ERR_INVALID_ARG


def test_python_api_refuses_cpu_tensors(L):
    import torch
    import full_vocab_kl_b200 as nb
    x = torch.zeros(4, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        nb.kl_forward(x, x, x, x, torch.zeros(4, dtype=torch.int64))


def test_vocab_parallel_argument_errors(L):
    lib = L.lib()
    s = shape(L, N=256, V=1024, ds=256, dt=256)
    p = [ctypes.c_void_p(v) for v in FAKE]
    wsb = ws_size(L, s)
    # negative shard offset
    assert lib.nb_kl_vp_state(L.shape_ptr(s), -256, p[0], p[1], p[2], p[3], p[4], 1.0, 1.0, p[5], p[6], wsb,
                              None) == L.NB_ERR_INVALID_ARG
    # missing state output
    assert lib.nb_kl_vp_state(L.shape_ptr(s), 0, p[0], p[1], p[2], p[3], p[4], 1.0, 1.0, None, p[6], wsb,
                              None) == L.NB_ERR_INVALID_ARG
    # no parts / bad beta
    assert lib.nb_kl_vp_combine(256, 0, p[0], p[1], -100, 1.0, p[2], p[3], p[4], p[5], None, None, p[6], p[7],
                                None) == L.NB_ERR_INVALID_ARG
    assert lib.nb_kl_vp_combine(256, 2, p[0], p[1], -100, 2.0, p[2], p[3], p[4], p[5], None, None, p[6], p[7],
                                None) == L.NB_ERR_INVALID_ARG
    # the second JSD pass only exists for 0 < beta < 1
    assert lib.nb_kl_vp_jsd_partial(L.shape_ptr(s), p[0], p[1], p[2], p[3], p[4], 1.0, 1.0, p[5], p[6], p[7],
                                    p[8], wsb, None) == L.NB_ERR_INVALID_ARG
    assert lib.nb_kl_vp_jsd_combine(256, 2, None, p[1], -100, p[2], p[3], p[4], p[5],
                                    None) == L.NB_ERR_INVALID_ARG


def test_spectral_argument_errors(L):
    lib = L.lib()
    p = [ctypes.c_void_p(v) for v in FAKE]
    # d not a multiple of 8, rows < 1, misaligned output, k < 8
    assert lib.nb_kl_gram(p[0], 100, 12, p[1], p[2], None) == L.NB_ERR_INVALID_ARG
    assert lib.nb_kl_gram(p[0], 0, 64, p[1], p[2], None) == L.NB_ERR_INVALID_ARG
    assert lib.nb_kl_gram(p[0], 100, 64, ctypes.c_void_p(FAKE[1] + 4), p[2], None) == L.NB_ERR_INVALID_ARG
    assert lib.nb_kl_project(p[0], 100, 64, p[1], 4, p[2], p[3], None) == L.NB_ERR_INVALID_ARG
    assert lib.nb_kl_project(p[0], 100, 64, None, 64, p[2], p[3], None) == L.NB_ERR_INVALID_ARG
    assert lib.nb_kl_project(p[0], 100, 60, p[1], 64, p[2], p[3], None) == L.NB_ERR_INVALID_ARG


def test_chunk_columns(L):
    lib = L.lib()
    # default: the vocabulary in equal chunks (multiples of 256) of at most ~24576 gradient tiles
    # of 128 x 256 (but at least 4 d_s and 2048, at most 131072 columns)
    assert lib.nb_kl_chunk_columns(L.shape_ptr(shape(L))) == 76032                  # 2 x 75968 -> 256
    assert lib.nb_kl_chunk_columns(L.shape_ptr(shape(L, N=32768, ds=4096, dt=512))) == 21760   # 7 chunks
    assert lib.nb_kl_chunk_columns(L.shape_ptr(shape(L, N=65536, ds=256, dt=256))) == 11776    # 13 chunks
    assert lib.nb_kl_chunk_columns(L.shape_ptr(shape(L, N=8192, V=248320, ds=5120, dt=5120))) == 82944
    assert lib.nb_kl_chunk_columns(L.shape_ptr(shape(L, N=256, V=1000, ds=256, dt=256))) == 1024
    # an explicit chunk is kept; an invalid shape gives 0
    assert lib.nb_kl_chunk_columns(L.shape_ptr(shape(L, chunk=4096))) == 4096
    assert lib.nb_kl_chunk_columns(L.shape_ptr(shape(L, ds=100))) == 0


def test_python_layers_refuse_host_tensors(L):
    """Every binding checks that its tensors are on the GPU before a pointer reaches the library."""
    import torch
    from full_vocab_kl_b200 import handoff, spectral
    from full_vocab_kl_b200.vocab_parallel import LibraryKernels
    k = LibraryKernels()
    lab = torch.zeros(4, dtype=torch.int64)
    with pytest.raises(ValueError):
        k.combine(torch.zeros((2, L.VP_FIELDS, 4)), lab, 1.0, -100, False)
    with pytest.raises(ValueError):
        k.jsd_combine(torch.zeros((2, 2, 4)), lab, -100)
    x = torch.zeros((4, 8), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        k.jsd_partial(x, x, x, x, lab, 0.5, 1.0, torch.zeros(4), torch.zeros(4), -100)
    with pytest.raises(ValueError):
        spectral.gram(x)
    with pytest.raises(ValueError):
        spectral.project(x, torch.zeros((8, 8), dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        handoff.receive_rows(x)


def test_forward_out_dict_is_checked(L, monkeypatch):
    """A caller-supplied output dictionary is validated before the call (here the inputs pass the
    device check through a stand-in, and the outputs are host tensors)."""
    import torch
    from full_vocab_kl_b200 import api
    monkeypatch.setattr(api, "_check_inputs", lambda *a: None)
    monkeypatch.setattr(api, "_workspace", lambda n, dev, ws: None)
    x = torch.zeros((4, 8), dtype=torch.bfloat16)
    lab = torch.zeros(4, dtype=torch.int64)
    out = {k: torch.zeros(4) for k in ("loss_tok", "lse_s", "lse_t", "aux")}
    out.update(loss_mean=torch.zeros(()), n_valid=torch.zeros((), dtype=torch.int64))
    with pytest.raises(ValueError):
        api.kl_forward(x, x, x, x, lab, 1.0, 1.0, out=out)


def test_c_program_uses_the_abi(L, tmp_path):
    """A plain C99 program compiled against include/nb_kl.h links the library and gets the
    documented host-side behaviour (tests/c/abi_check.c)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    from full_vocab_kl_b200 import build
    libdir = os.path.dirname(build.LIB)
    exe = str(tmp_path / "abi_check")
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c", "abi_check.c"), "-o", exe, "-L", libdir, "-lnbkl",
                        "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
