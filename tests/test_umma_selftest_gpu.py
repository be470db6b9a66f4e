"""The fused kernel's tensor-core operand encodings (128-byte swizzled
K-major and MN-major shared-memory layouts, instruction and matrix
descriptors, TMEM read-back), checked in isolation against a matmul."""
import pytest
import torch

from gated_delta_rule_156_b200 import kda as K

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("a_mn", [False, True])
@pytest.mark.parametrize("b_mn", [False, True])
@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("Kd,panel", [(64, 64), (128, 128), (64, 128)])
def test_umma_layouts(a_mn, b_mn, N, Kd, panel):
    g = torch.Generator(device="cuda").manual_seed(N + Kd + panel + 2 * a_mn + b_mn)
    A = torch.randn((128, Kd), generator=g, device="cuda").bfloat16()
    B = torch.randn((Kd, N), generator=g, device="cuda").bfloat16()
    A_in = A.t().contiguous() if a_mn else A
    B_in = B.contiguous() if b_mn else B.t().contiguous()
    D = K.selftest_umma(A_in, B_in, a_mn, b_mn, panel)
    torch.cuda.synchronize()
    ref = A.float() @ B.float()
    err = (D - ref).abs().max().item()
    assert err < 1e-3 * ref.abs().max().item(), err
