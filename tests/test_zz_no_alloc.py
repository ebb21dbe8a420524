"""nb_kl_forward_noalloc: the forward for callers that cannot allocate device memory
themselves (for example code under a memory manager that owns every device byte, or code
that must not call cudaMalloc/cudaFree because they can synchronise the device). Its
scratch is a fixed array inside the library, so these tests call it through the C ABI and
compare its results with nb_kl_forward given a normal workspace, on two calls in a row
(the array keeps the previous call's contents). This file is collected last on purpose."""

import ctypes

import numpy as np
import pytest

import gpu_util as gu
from synthetic import make_custom, make_inputs

pytestmark = pytest.mark.gpu


def _noalloc(x):
    import torch
    import full_vocab_kl_b200 as nb
    from full_vocab_kl_b200 import _abi
    t = gu.torch_inputs(x)
    N = x.labels.shape[0]
    f32 = dict(dtype=torch.float32, device="cuda")
    out = {"loss_tok": torch.full((N,), float("nan"), **f32), "lse_s": torch.full((N,), float("nan"), **f32),
           "lse_t": torch.full((N,), float("nan"), **f32), "aux": torch.full((N,), float("nan"), **f32),
           "loss_mean": torch.full((), float("nan"), **f32),
           "n_valid": torch.full((), -1, dtype=torch.int64, device="cuda")}
    shape = nb.make_shape(t["h_s"], t["W_s"], t["h_t"], t["W_t"], t["labels"])
    code = _abi.lib().nb_kl_forward_noalloc(
        _abi.shape_ptr(shape), t["h_s"].data_ptr(), t["W_s"].data_ptr(), t["h_t"].data_ptr(),
        t["W_t"].data_ptr(), t["labels"].data_ptr(), float(x.beta), float(x.tau), out["loss_tok"].data_ptr(),
        out["lse_s"].data_ptr(), out["lse_t"].data_ptr(), out["aux"].data_ptr(), out["loss_mean"].data_ptr(),
        out["n_valid"].data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    _abi.check("nb_kl_forward_noalloc", code)
    torch.cuda.synchronize()
    # the fixed scratch's status word: no bounded wait of this call ran out
    assert _abi.lib().nb_kl_noalloc_device_status(
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == _abi.NB_OK
    got = {k: out[k].cpu().numpy().astype(np.float64) for k in ("loss_tok", "lse_s", "lse_t", "aux")}
    got["loss_mean"] = float(out["loss_mean"].item())
    got["n_valid"] = int(out["n_valid"].item())
    return got


@pytest.mark.parametrize("case", ["tiny", "ragged_jsd", "forward_kl"])
def test_noalloc_matches_workspace_forward_twice(case):
    if case == "tiny":
        x = make_inputs("tiny")
    elif case == "ragged_jsd":
        x = make_custom(300, 200, 136, 1000, 0.5, 2.0, n_masked=37, teacher="independent")
    else:
        x = make_custom(1100, 256, 320, 5000, 0.0, 1.0, n_masked=300, teacher="correlated")
    ref = gu.run_library(x, backward=False)
    for _ in range(2):
        got = _noalloc(x)
        gu.check_forward(got, ref, x.labels)


def test_noalloc_rejects_shapes_beyond_the_fixed_scratch():
    import torch
    from full_vocab_kl_b200 import _abi
    shape = _abi.Shape(n_tokens=65536, vocab=151936, d_s=4096, d_t=4096, h_dtype=0, reserved=0,
                       ignore_index=-100, chunk_v=0)
    assert _abi.lib().nb_kl_workspace_size(_abi.shape_ptr(shape), 1.0) > _abi.NOALLOC_SCRATCH_BYTES
    # null pointers: the size check answers before any pointer is used, and if it ever did not,
    # the pointer checks would refuse the call before a launch
    null = [None] * 11
    code = _abi.lib().nb_kl_forward_noalloc(_abi.shape_ptr(shape), *null[:5], 1.0, 1.0, *null[5:11],
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == _abi.NB_ERR_WORKSPACE
