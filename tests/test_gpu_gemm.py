"""The tcgen05 projection kernel alone (through vla_gemm_bf16) against torch fp32 matmul
of the same bf16 operands: orientation, descriptors, ragged token tails, split-K fixup."""
import math

import pytest

pytestmark = pytest.mark.gpu

SHAPES = [
    # n_feat, k_dim, m_tok, split_k
    (128, 64, 1, 0),
    (128, 128, 17, 1),
    (256, 1024, 50, 0),
    (256, 1024, 50, 1),
    (256, 1024, 50, 16),
    (2560, 1024, 50, 0),
    (1024, 2048, 51, 0),
    (8192, 1024, 64, 0),
    (1024, 4096, 65, 0),
    (384, 640, 200, 3),
    (1024, 1024, 700, 0),
    (2560, 1024, 3200, 0),
    (1024, 4096, 3200, 0),
]


@pytest.mark.parametrize("n,k,m,split", SHAPES)
def test_gemm_matches_torch(n, k, m, split):
    import torch
    import flow_matching_vla_euler_b200 as V
    g = torch.Generator(device="cuda").manual_seed(n * 7 + k * 3 + m)
    W = torch.randn((n, k), device="cuda", generator=g).to(torch.bfloat16)
    X = torch.randn((m, k), device="cuda", generator=g).to(torch.bfloat16)
    Y = V.gemm(W, X, split)
    ref = X.float() @ W.float().T
    V.vla_gemm_status(V._stream())          # no bounded wait gave up
    torch.testing.assert_close(Y, ref, rtol=1e-4, atol=2e-4 * math.sqrt(k))


def test_gemm_split_k_is_deterministic():
    import torch
    import flow_matching_vla_euler_b200 as V
    g = torch.Generator(device="cuda").manual_seed(5)
    W = torch.randn((1024, 4096), device="cuda", generator=g).to(torch.bfloat16)
    X = torch.randn((50, 4096), device="cuda", generator=g).to(torch.bfloat16)
    a = V.gemm(W, X, 16)
    b = V.gemm(W, X, 16)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
