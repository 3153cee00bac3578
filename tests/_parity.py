"""Element-by-element comparison of a GPU solve with the oracle's.

The rule follows the tolerances stated for this build: a cell (k, b) is a
near-tie when the oracle's two candidate values differ by less than 1e-4; a
cell is tainted when it is a near-tie whose backpointer differs, or when a cell
it reads (skip source (k-1, b), execute source (k-1, b - w_k)) is tainted.  On
untainted cells backpointers are bit-exact and values agree within ``val_tol``;
final layer sets are bit-exact on untainted cells; the best (S, gamma) agrees
unless its cell is tainted or the oracle's two best distinct-set TPTs are
within 1e-6 (relative), which is reported instead.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List

import numpy as np

NEAR_TIE = 1e-4


@dataclass
class Report:
    n_cells: int
    near_ties: int = 0
    tainted: int = 0
    tainted_final: int = 0
    bp_mismatch_untainted: int = 0
    val_max_err: float = 0.0
    val_fail: int = 0
    set_mismatch_untainted: int = 0
    argmax_ok: bool = True
    argmax_note: str = ""
    notes: List[str] = field(default_factory=list)

    def assert_ok(self):
        assert self.bp_mismatch_untainted == 0, self
        assert self.val_fail == 0, self
        assert self.set_mismatch_untainted == 0, self
        assert self.argmax_ok, self


def taint_mask(w, bp_o, bp_g, cos_s_o, cos_e_o, extra=None):
    """extra [n][C]: cells tainted whatever their backpointers (e.g. values within
    the near-tie distance of a pruning threshold, whose validity may flip)."""
    n, C = bp_o.shape
    near = np.abs(np.nan_to_num(cos_e_o, nan=np.inf) - np.nan_to_num(cos_s_o, nan=-np.inf)) < NEAR_TIE
    taint = np.zeros((n, C), dtype=bool)
    prev = np.zeros(C, dtype=bool)
    for k in range(n):
        t = near[k] & (bp_o[k] != bp_g[k])
        if extra is not None:
            t |= extra[k]
        t |= prev
        wk = int(w[k])
        if wk < C:
            t[wk:] |= prev[:C - wk]
        taint[k] = t
        prev = t
    return near, taint


def compare_solve(orc, gpu, w, val_tol, n_items, sets_gpu=None, rows_val_gpu=None,
                  check_argmax=True, prune_tau=None) -> Report:
    """orc: oracle Solve; gpu: dict of numpy arrays bp [n][C], values [C], sets (lists),
    best (b, gamma), tpt grid [C][G] (optional); rows_val_gpu: [n][C] chosen values.
    With check_argmax=False (a budget prefix) the TPT choice is not compared."""
    bp_o = orc.dp.bp
    C = bp_o.shape[1]
    bp_g = gpu["bp"]
    extra = None
    if prune_tau is not None:
        kept = np.where(bp_o == 1, orc.dp.cos_e, orc.dp.cos_s)
        extra = np.abs(np.nan_to_num(kept, nan=np.inf) - prune_tau) < NEAR_TIE
    near, taint = taint_mask(w, bp_o, bp_g, orc.dp.cos_s, orc.dp.cos_e, extra)
    r = Report(n_cells=C)
    r.near_ties = int(near.sum())
    r.tainted = int(taint.sum())
    r.tainted_final = int(taint[-1].sum())
    r.bp_mismatch_untainted = int(((bp_o != bp_g) & ~taint).sum())
    # values: final row always, every row when the GPU exported them
    ok = ~taint[-1]

    def errors(g, o):
        # invalid cells (exact-budget mode) are NaN on both sides; NaN on one side only fails
        g = g.astype(np.float64)
        both = np.isnan(g) & np.isnan(o)
        e = np.where(both, 0.0, np.abs(g - o))
        return np.where(np.isnan(e), np.inf, e)

    err = errors(gpu["values"], orc.values)
    r.val_max_err = float(np.max(err[ok])) if ok.any() else 0.0
    r.val_fail = int(np.sum(err[ok] > val_tol))
    if rows_val_gpu is not None:
        e2 = errors(rows_val_gpu, orc.dp.val[1:])
        m = ~taint & orc.dp.valid[1:]
        r.val_max_err = max(r.val_max_err, float(np.max(e2[m])) if m.any() else 0.0)
        r.val_fail += int(np.sum(e2[m] > val_tol))
    sets_g = gpu["sets"]
    r.set_mismatch_untainted = int(sum(1 for b in range(C) if ok[b] and sets_g[b] != orc.sets[b]))
    if not check_argmax:
        return r
    # best (S, gamma)
    bo, go = orc.best_b, orc.best_gamma
    bg, gg = int(gpu["best"][0]), int(gpu["best"][1])
    same = (sets_g[bg] == orc.sets[bo]) and (gg == go)
    if not same:
        # second-best distinct-set TPT of the oracle
        grid = orc.tpt
        best_v = orc.best_tpt
        second = -np.inf
        for b in range(C):
            if orc.sets[b] == orc.sets[bo]:
                continue
            v = np.nanmax(grid[b]) if np.isfinite(grid[b]).any() else -np.inf
            second = max(second, v)
        gap = (best_v - second) / abs(best_v) if np.isfinite(second) else np.inf
        # gamma-only ties inside the same set are also near-ties
        row = grid[bo]
        g_sorted = np.sort(row[np.isfinite(row)])[::-1]
        ggap = (g_sorted[0] - g_sorted[1]) / abs(g_sorted[0]) if len(g_sorted) > 1 else np.inf
        if taint[-1, bo] or taint[-1, bg] or gap < 1e-6 or ggap < 1e-6:
            r.argmax_note = (f"argmax differs at a tainted or near-tied cell: oracle (b={bo}, g={go}) "
                             f"gpu (b={bg}, g={gg}), distinct-set gap {gap:.3g}, gamma gap {ggap:.3g}")
        else:
            r.argmax_ok = False
            r.argmax_note = f"oracle (b={bo}, g={go}, {orc.sets[bo]}) vs gpu (b={bg}, g={gg}, {sets_g[bg]})"
    return r
