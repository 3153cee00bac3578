"""The script that writes the large full-grid goldens (tests/golden/make_large_golden.py)
run on the tiny workload, under both key/value readings: what it stores reads back
through the loader the GPU test uses and equals a fresh oracle solve (values,
backpointers, sets, argmax), and its input digests are the seeded draws'.  CPU only."""
import dataclasses
import os
import sys

import numpy as np
import pytest

from knapsack_layer_selection_b200 import workloads as W
from oracle import ks_oracle as O
from tests._util import oracle_model, x0_np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))
import make_large_golden as MG  # noqa: E402


@pytest.mark.parametrize("kv", ["cache", "window"])
def test_golden_script_round_trip(tmp_path, monkeypatch, kv):
    out = str(tmp_path / f"tiny_{kv}_full.npz")
    monkeypatch.setattr(sys, "argv", ["make_large_golden.py", "tiny", "--kv", kv, "--out", out])
    MG.main()
    wl = W.WORKLOADS["tiny"]
    import tests.test_gpu_large as TL            # the reader the full-size GPU test uses
    z, orc = TL.load_golden(out, wl.n_items)
    inp = W.make_inputs(wl)
    assert str(z["input_sha256"]) == W.input_digest(inp)
    assert str(z["kv"]) == kv
    if kv == "window":
        ww = W.window_weights(wl, device="cpu")
        assert str(z["window_sha256"]) == W.window_digest(ww)
        inp = dataclasses.replace(inp, layers=[{**L, **x} for L, x in zip(inp.layers, ww)])
    t = wl.latencies()
    w = O.quantize_weights(t, wl.n_bins)
    ref = O.dp_solve(oracle_model(inp), x0_np(inp), wl.ctx, w, t, wl.gamma_max, kv=kv)
    assert [int(x) for x in z["w"]] == list(w)
    assert np.array_equal(orc.values, ref.values)
    assert np.array_equal(orc.dp.bp, ref.dp.bp.astype(np.uint8))
    assert orc.sets == [sorted(s) for s in ref.sets]
    assert (orc.best_b, orc.best_gamma) == (ref.best_b, ref.best_gamma)
