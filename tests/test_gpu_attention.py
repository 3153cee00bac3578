"""The tcgen05 attention (ks_attention_bf16) against a plain PyTorch fp32
softmax(QK^T/sqrt(hd))V of the same bf16 operands with the causal window of the
evaluation tokens: ragged row tiles, contexts that are not a multiple of the
128-key block, ctx = 0, T = 1, GQA groups, head_dim 64 and 128; and row
independence (a row's output does not depend on the batch)."""
import math

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


def _case(R, T, Hq, Hkv, hd, ctx, extra_rows=5, seed=0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = (torch.randn(R, Hq, hd, generator=g, device="cuda") * 1.3).to(torch.bfloat16)
    rows = ctx + T + extra_rows
    k = (torch.randn(rows, Hkv, hd, generator=g, device="cuda") * 1.3).to(torch.bfloat16)
    v = (torch.randn(rows, Hkv, hd, generator=g, device="cuda") * 1.3).to(torch.bfloat16)
    return q, k, v


def _reference(q, k, v, T, ctx):
    R, Hq, hd = q.shape
    Hkv = k.shape[1]
    grp = Hq // Hkv
    n = ctx + T
    kf = k[:n].float().repeat_interleave(grp, dim=1)      # [n][Hq][hd]
    vf = v[:n].float().repeat_interleave(grp, dim=1)
    s = torch.einsum("rhd,nhd->rhn", q.float(), kf) / math.sqrt(hd)
    t = torch.arange(R, device=q.device) % T
    mask = torch.arange(n, device=q.device)[None, :] <= (ctx + t)[:, None]   # [R][n]
    s = s.masked_fill(~mask[:, None, :], float("-inf"))
    return torch.einsum("rhn,nhd->rhd", torch.softmax(s, dim=-1), vf)


CASES = [(8, 8, 16, 4, 64, 2048), (296, 8, 16, 4, 64, 2048), (1, 1, 4, 4, 64, 0),
         (37, 4, 4, 1, 64, 100), (16, 16, 32, 8, 128, 8192), (300, 16, 32, 8, 128, 8192),
         (130, 16, 8, 8, 128, 127), (64, 8, 64, 8, 128, 1000), (5, 5, 2, 2, 128, 0)]


@pytest.mark.parametrize("R,T,Hq,Hkv,hd,ctx", CASES)
def test_attention_matches_fp32_reference(R, T, Hq, Hkv, hd, ctx):
    q, k, v = _case(R, T, Hq, Hkv, hd, ctx, seed=R + ctx)
    out = torch.full((R, Hq, hd), float("nan"), device="cuda").to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.attention_bf16(q, k, v, T, ctx, out, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = _reference(q, k, v, T, ctx)
    assert torch.isfinite(out.float()).all()
    rel = ((out.float() - ref).norm() / ref.norm()).item()
    worst = (out.float() - ref).abs().max().item()
    assert rel < 1e-2 and worst < 5e-2 * ref.abs().max().item(), (rel, worst)


def test_attention_rows_do_not_depend_on_the_batch():
    R, T, Hq, Hkv, hd, ctx = 259, 16, 8, 2, 128, 777
    q, k, v = _case(R, T, Hq, Hkv, hd, ctx, seed=9)
    out = torch.empty(R, Hq, hd, device="cuda", dtype=torch.bfloat16)
    B.attention_bf16(q, k, v, T, ctx, out)
    for r0 in (0, 16, 128, 240):
        sub = q[r0:r0 + 16].contiguous()          # 16 rows = one window of T tokens
        o2 = torch.empty_like(sub)
        B.attention_bf16(sub, k, v, T, ctx, o2)
        torch.cuda.synchronize()
        assert torch.equal(o2, out[r0:r0 + 16]), r0


def test_attention_is_deterministic_at_long_context():
    """Bitwise-equal outputs on reruns: at 8k context the running reference
    maximum still moves in late blocks, so the O rescale (which must wait for
    every earlier P.V to land) is exercised while the P.V chain runs behind."""
    R, T, Hq, Hkv, hd, ctx = 1024, 16, 32, 8, 128, 8192
    q, k, v = _case(R, T, Hq, Hkv, hd, ctx, seed=21)
    first = None
    for _ in range(6):
        out = torch.empty(R, Hq, hd, device="cuda", dtype=torch.bfloat16)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        B.attention_bf16(q, k, v, T, ctx, out, status)
        torch.cuda.synchronize()
        assert status.item() == 0
        if first is None:
            first = out
        else:
            assert torch.equal(first, out)


@pytest.mark.parametrize("hd", [64, 128])
def test_attention_with_a_maximum_that_keeps_growing(hd):
    """Keys whose norm grows with position: the row maximum rises block after
    block, so the reference moves often (O rescaled in place, and each softmax
    group's own row sum brought to the new reference) in both groups' blocks."""
    R, T, Hq, Hkv, ctx = 256, 16, 8, 2, 2000
    q, k, v = _case(R, T, Hq, Hkv, hd, ctx, seed=33)
    ramp = 1.0 + torch.arange(k.shape[0], device="cuda", dtype=torch.float32) / 256.0
    k = (k.float() * ramp[:, None, None]).to(torch.bfloat16)
    out = torch.empty(R, Hq, hd, device="cuda", dtype=torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.attention_bf16(q, k, v, T, ctx, out, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = _reference(q, k, v, T, ctx)
    rel = ((out.float() - ref).norm() / ref.norm()).item()
    worst = (out.float() - ref).abs().max().item()
    assert rel < 1e-2 and worst < 5e-2 * ref.abs().max().item(), (rel, worst)
