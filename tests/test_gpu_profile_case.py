"""The profiler harness (``python -m knapsack_layer_selection_b200.profile_case``)
runs each of its cases -- one Attention item, one MLP item, whole solves of a
two-layer model spanning the full grid -- and leaves the device status clean.
It is the command the kernel profiles are taken with, so it is kept working."""
import subprocess
import sys

import pytest
import torch

from knapsack_layer_selection_b200 import build as BUILD

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("item", ["attn", "mlp", "solve"])
def test_profile_case_runs(item):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    BUILD.build()
    r = subprocess.run([sys.executable, "-m", "knapsack_layer_selection_b200.profile_case",
                        "--workload", "small", "--item", item, "--repeat", "1"],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "ok" in r.stdout
