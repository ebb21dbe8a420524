"""The tcgen05 GEMM mainloop on its own: every operand layout the loss kernels use
(K-major and MN-major A and B, 128-byte swizzle) against a float64 matmul of the same
bf16 values, including ragged M, N and K."""

import numpy as np
import pytest

from synthetic import bf16_bits_to_f32, f32_to_bf16_bits

pytestmark = pytest.mark.gpu


def run(A_bits, a_mn, B_bits, b_mn, M, N, K):
    import torch
    from full_vocab_kl_b200 import _abi
    A = torch.from_numpy(A_bits.view(np.int16)).view(torch.bfloat16).cuda()
    B = torch.from_numpy(B_bits.view(np.int16)).view(torch.bfloat16).cuda()
    C = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    code = _abi.lib().nb_kl_debug_gemm(A.data_ptr(), a_mn, B.data_ptr(), b_mn, M, N, K, C.data_ptr(),
                                       ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    _abi.check("nb_kl_debug_gemm", code)
    torch.cuda.synchronize()
    assert _abi.lib().nb_kl_device_status(ws.data_ptr(), None) == 0
    return C.cpu().numpy()


@pytest.mark.parametrize("a_mn", [0, 1])
@pytest.mark.parametrize("b_mn", [0, 1])
@pytest.mark.parametrize("M,N,K", [(128, 128, 64), (256, 384, 320), (136, 264, 200), (1024, 512, 1000),
                                   (304, 1288, 136), (520, 640, 512),
                                   # enough 256-row tiles for the 256 x 512 wide tiles (one per CTA pair)
                                   (19200, 512, 200), (9480, 776, 136)])
def test_gemm_layouts(a_mn, b_mn, M, N, K):
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    A = f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    B = f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32))
    ref = bf16_bits_to_f32(A).astype(np.float64) @ bf16_bits_to_f32(B).astype(np.float64).T
    As = np.ascontiguousarray(A.T) if a_mn else A
    Bs = np.ascontiguousarray(B.T) if b_mn else B
    C = run(As, a_mn, Bs, b_mn, M, N, K)
    assert np.isfinite(C).all()
    err = np.abs(C - ref).max() / np.abs(ref).max()
    assert err < 2e-6, err
