#!/usr/bin/env python
"""Write the oracle's full-grid DP for one large workload to tests/golden/.

Calls only the fp64 CPU oracle (``oracle/ks_oracle.py``) and the seeded input
generator; nothing here runs or reads the CUDA library.  The result is the
expected value for the full-size parity test (``tests/test_gpu_large.py``): every
budget cell's backpointers and both candidate values per item, the chosen
values, the reconstructed sets, the TPT grid and its argmax (b*, gamma*), plus a
digest of the inputs so that the GPU machine can confirm it drew the same ones.

    python tests/golden/make_large_golden.py llama3_8b_8k
    python tests/golden/make_large_golden.py llama3_8b_32k --ctx 4096
    python tests/golden/make_large_golden.py llama3_8b_8k --kv window

``--mode exact`` solves the exact-budget table, and ``--prune-tau`` / ``--skip-cap``
apply the cosine threshold and the skip cap; ``--kv window`` solves under the
window key/value reading (the oracle's R7w: the
window positions' keys and values recomputed from each candidate's state through
Wk/Wv, drawn by ``workloads.window_weights``) and records their digest as well.

The 8B shape at 8k context takes about 25 minutes on eight host cores (OpenBLAS
fp64) and 30 GB of host memory; the Qwen3-32B shape draws its layers one at a
time (``StreamedInputs``) and needs about 15 GB.
"""
from __future__ import annotations

import argparse
import dataclasses
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from knapsack_layer_selection_b200 import workloads as W  # noqa: E402
from oracle import ks_oracle as O  # noqa: E402
from tests._util import oracle_model, x0_np  # noqa: E402


def golden_path(name: str, ctx: int, kv: str = "cache", mode: str = "at_most", tau=None,
                cap=None) -> str:
    tag = "" if kv == "cache" else f"_{kv}"
    tag += "" if mode == "at_most" else f"_{mode}"
    tag += "" if tau is None else f"_tau{tau:g}"
    tag += "" if cap is None else f"_cap{cap}"
    return os.path.join(HERE, f"{name}_ctx{ctx}{tag}_full.npz")


def pack_sets(sets, n_items: int) -> np.ndarray:
    words = (n_items + 63) // 64
    out = np.zeros((len(sets), words), dtype=np.uint64)
    for b, s in enumerate(sets):
        for k in s:
            out[b, k // 64] |= np.uint64(1) << np.uint64(k % 64)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("workload", choices=["llama3_8b_8k", "llama3_8b_32k", "qwen3_32b_16k", "small",
                                         "tiny"])
    ap.add_argument("--streamed", action="store_true",
                    help="hold one layer of weights at a time (the 64 GB Qwen3-32B shape)")
    ap.add_argument("--ctx", type=int, default=None, help="context to solve at (default: the workload's)")
    ap.add_argument("--kv", choices=["cache", "window"], default="cache",
                    help="the attention's key/value reading (R7 or R7w)")
    ap.add_argument("--mode", choices=["at_most", "exact"], default="at_most")
    ap.add_argument("--prune-tau", type=float, default=None)
    ap.add_argument("--skip-cap", type=int, default=None)
    ap.add_argument("--out", default=None)
    a = ap.parse_args()

    base = W.WORKLOADS[a.workload]
    wl = base.with_ctx(a.ctx) if a.ctx is not None else base
    t0 = time.time()
    if a.streamed or a.workload == "qwen3_32b_16k":
        inp = W.StreamedInputs(base)                # layers drawn again when the oracle reads them
        digest = inp.digest
    else:
        inp = W.make_inputs(base, device="cpu")    # the cache holds the workload's largest context
        digest = W.input_digest(inp)
    print(f"{a.workload}: inputs drawn and hashed in {time.time() - t0:.0f} s, sha256 {digest}",
          flush=True)
    window_sha = ""
    if a.kv == "window":
        if isinstance(inp, W.StreamedInputs):
            raise SystemExit("the window reading is written for the fully drawn workloads only")
        ww = W.window_weights(base, device="cpu")
        window_sha = W.window_digest(ww)
        inp = dataclasses.replace(inp, layers=[{**L, **x} for L, x in zip(inp.layers, ww)])

    om = oracle_model(inp)
    x0 = x0_np(inp)
    t = wl.latencies()
    w = O.quantize_weights(t, wl.n_bins)
    t1 = time.time()
    ref = O.reference_states(om, x0, wl.ctx, kv=a.kv)
    print(f"reference chain in {time.time() - t1:.0f} s", flush=True)
    t2 = time.time()
    orc = O.dp_solve(om, x0, wl.ctx, w, t, wl.gamma_max, ref=ref, kv=a.kv, mode=a.mode,
                     prune_tau=a.prune_tau, skip_cap=a.skip_cap)
    secs = time.time() - t2
    print(f"DP over {len(orc.values)} cells x {wl.n_items} items in {secs:.0f} s; best (b={orc.best_b}, "
          f"gamma={orc.best_gamma}, TPT={orc.best_tpt:.6g}), set {orc.sets[orc.best_b]}", flush=True)

    out = a.out or golden_path(a.workload, wl.ctx, a.kv, a.mode, a.prune_tau, a.skip_cap)
    np.savez_compressed(
        out,
        workload=np.array(a.workload), ctx=np.int64(wl.ctx), T=np.int64(wl.T),
        input_sha256=np.array(digest), seed=np.int64(0), kv=np.array(a.kv),
        mode=np.array(a.mode), prune_tau=np.float64(np.nan if a.prune_tau is None else a.prune_tau),
        skip_cap=np.int64(-1 if a.skip_cap is None else a.skip_cap),
        window_sha256=np.array(window_sha),
        w=np.asarray(w, np.int32), t=np.asarray(t, np.float64),
        bp=orc.dp.bp.astype(np.uint8), cos_s=orc.dp.cos_s, cos_e=orc.dp.cos_e,
        val=orc.dp.val, valid=orc.dp.valid,
        values=orc.values, sets=pack_sets(orc.sets, wl.n_items),
        used_w=orc.used_w.astype(np.int64), t_draft=orc.t_draft, tpt=orc.tpt,
        best=np.array([orc.best_b, orc.best_gamma], np.int64), best_tpt=np.float64(orc.best_tpt),
        ref_final=ref[-1], oracle_seconds=np.float64(secs))
    print(f"wrote {out} ({os.path.getsize(out) / 1e6:.2f} MB)", flush=True)


if __name__ == "__main__":
    main()
