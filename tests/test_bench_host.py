"""bench.py's host-side accounting, checked by hand counts (no GPU)."""
from types import SimpleNamespace

import torch

import bench


def test_select_bytes_counts_reads_writes_and_the_next_operand():
    # T = 2 tokens x d = 4: a state is 8 fp32 values (32 bytes), an operand 8 bf16 (16 bytes)
    wl = SimpleNamespace(T=2, d_model=4, wdtype="bf16")
    bp = torch.tensor([[0, 1, 1], [0, 0, 1]], dtype=torch.uint8)   # C = 3 cells, two items
    # item 0 (w = 1): read ref + 3 skip + 2 exec = 6 states; write ref + 2 winners = 3;
    #                 next operand for 4 slots = 64 bytes
    # item 1 (w = 2): read ref + 3 skip + 1 exec = 5 states; write ref + 1 winner = 2; last item
    expect = (6 + 3) * 32 + 64 + (5 + 2) * 32
    assert bench.select_bytes(wl, 3, [1, 2], bp, keep_ref=False) == expect
    # the kept reference states add one state write per item
    assert bench.select_bytes(wl, 3, [1, 2], bp, keep_ref=True) == expect + 2 * 32
    # an fp32 model's operand is four bytes a value
    wl32 = SimpleNamespace(T=2, d_model=4, wdtype="f32")
    assert bench.select_bytes(wl32, 3, [1, 2], bp, keep_ref=False) == expect + 64
