"""Bounded device waits: a wait that can never complete ends after its limit with
NB_ERR_TIMEOUT in the status word, and the context stays usable afterwards."""

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("sleeping", [0, 1])
def test_wait_runs_out_and_context_survives(sleeping):
    """A 20 ms limit: the polling wait and the sleeping wait of the pipeline kernels both give
    up, record the timeout, and end within the limit plus the sleeping wait's check interval
    (16 suspensions of at most 1 ms) and launch overhead."""
    import torch
    from full_vocab_kl_b200 import _abi
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    code = _abi.lib().nb_kl_debug_wait_timeout(ws.data_ptr(), 20_000_000, sleeping, stream.cuda_stream)
    e1.record(stream)
    assert code == _abi.NB_OK
    assert _abi.lib().nb_kl_device_status(ws.data_ptr(), stream.cuda_stream) == _abi.NB_ERR_TIMEOUT
    ms = e0.elapsed_time(e1)
    assert 20.0 <= ms <= 20.0 + 16.0 + 30.0, ms
    # the context still works: a small loss call succeeds
    from synthetic import make_custom
    import gpu_util
    x = make_custom(130, 64, 64, 300, 1.0, 1.0, n_masked=10)
    out = gpu_util.run_library(x, backward=False)
    assert np.isfinite(out["loss_mean"])
