"""Device-side failure handling without a GPU fault: a wait that nothing
completes gives up after its bound, reports KS_ERR_TIMEOUT in the status word
the host reads, and leaves the CUDA context usable for the next launch."""
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


def test_bounded_wait_reports_timeout_and_context_survives():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    waited = torch.zeros(1, dtype=torch.int64, device="cuda")
    B.check_bounded_wait(50_000, status, waited)       # 50 ms
    torch.cuda.synchronize()
    assert status.item() == 5                           # KS_ERR_TIMEOUT
    assert 50e6 <= waited.item() < 2e9
    # the context still runs work: a tensor-core GEMM right after
    A = torch.randn(130, 128, device="cuda").to(torch.bfloat16)
    W = torch.randn(256, 128, device="cuda").to(torch.bfloat16)
    C = torch.empty(130, 256, device="cuda")
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.gemm_bf16(A, W, C, status=st2)
    torch.cuda.synchronize()
    assert st2.item() == 0
    assert (C - A.float() @ W.float().T).abs().max().item() < 1e-2


def test_bounded_wait_rejects_bad_limits():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(B.KnapSpecError):
        B.check_bounded_wait(0, status)
    with pytest.raises(B.KnapSpecError):
        B.check_bounded_wait(3_000_000, status)
