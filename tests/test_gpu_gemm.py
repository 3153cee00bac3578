"""The tcgen05 GEMM (ks_gemm_bf16) against a plain PyTorch fp32 matmul of the same
bf16 operands: ragged M (TMA zero fill, masked epilogue rows), several N/K, the
residual epilogue, and row independence (a row's result does not depend on M)."""
import pytest
import torch

from knapsack_layer_selection_b200 import binding as B
from knapsack_layer_selection_b200 import build as BUILD

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    BUILD.build()
    return B.load()


def _rand(shape, seed, scale=1.0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return (torch.randn(*shape, generator=g, device="cuda") * scale).to(torch.bfloat16)


SHAPES = [(1, 256, 64), (16, 256, 128), (127, 512, 64), (128, 256, 4096), (129, 768, 192),
          (300, 1024, 1024), (1000, 4096, 4096), (2056, 2816, 1024), (7984, 4096, 4096)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_matches_fp32_matmul(M, N, K):
    A = _rand((M, K), M * 7 + K)
    W = _rand((N, K), N * 3 + K, 0.02)
    C = torch.full((M, N), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.gemm_bf16(A, W, C, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = A.float() @ W.float().T
    err = (C - ref).abs().max().item()
    scale = ref.abs().max().item()
    assert err <= 1e-4 * scale + 1e-6, (M, N, K, err, scale)


def test_gemm_residual_epilogue():
    M, N, K = 333, 512, 256
    A = _rand((M, K), 1)
    W = _rand((N, K), 2, 0.02)
    R = torch.randn(M, N, device="cuda")
    C = torch.empty(M, N, device="cuda")
    B.gemm_bf16(A, W, C, resid=R)
    torch.cuda.synchronize()
    ref = A.float() @ W.float().T + R
    assert (C - ref).abs().max().item() < 1e-4


def test_gemm_rows_do_not_depend_on_the_batch():
    M, N, K = 517, 1024, 2048
    A = _rand((M, K), 3)
    W = _rand((N, K), 4, 0.02)
    C = torch.empty(M, N, device="cuda")
    B.gemm_bf16(A, W, C)
    for r in (0, 1, 127, 128, 300, 516):
        one = torch.empty(1, N, device="cuda")
        B.gemm_bf16(A[r:r + 1].contiguous(), W, one)
        torch.cuda.synchronize()
        assert torch.equal(one[0], C[r]), r


def test_gemm_rejects_unsupported_shapes():
    A = _rand((4, 96), 5)
    W = _rand((256, 96), 6)
    C = torch.empty(4, 256, device="cuda")
    with pytest.raises(B.KnapSpecError, match="multiple of 64"):
        B.gemm_bf16(A, W, C)
    A = _rand((4, 64), 5)
    W = _rand((200, 64), 6)
    C = torch.empty(4, 200, device="cuda")
    with pytest.raises(B.KnapSpecError, match="multiple of 256"):
        B.gemm_bf16(A, W, C)
