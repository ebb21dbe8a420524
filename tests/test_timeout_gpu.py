"""Bounded device waits: a wait that can never complete ends after its limit with
NB_ERR_TIMEOUT in the status word, and the context stays usable afterwards."""

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_context_survives():
    import torch
    from full_vocab_kl_b200 import _abi
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    code = _abi.lib().nb_kl_debug_wait_timeout(ws.data_ptr(), 20_000_000, torch.cuda.current_stream().cuda_stream)
    assert code == _abi.NB_OK
    assert _abi.lib().nb_kl_device_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream) == \
        _abi.NB_ERR_TIMEOUT
    # the context still works: a small loss call succeeds
    from synthetic import make_custom
    import gpu_util
    x = make_custom(130, 64, 64, 300, 1.0, 1.0, n_masked=10)
    out = gpu_util.run_library(x, backward=False)
    assert np.isfinite(out["loss_mean"])
