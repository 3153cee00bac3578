"""KnapSpec knapsack layer-selection DP -- plain, slow, fp64 CPU oracle.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU
baseline leg use this module.  It shares no code with the CUDA library and
imports nothing from it; the two sides meet only in the seeded inputs.

Source of the method: the Pith review page of arXiv 2602.20217 ("KnapSpec:
Self-Speculative Decoding via Adaptive Layer Selection as a Knapsack Problem"),
which paraphrases the paper's equations:

* items and weights -- every Attention and every MLP sublayer is one item whose
  weight is its (quantised) latency; Attention latency grows with the context
  length, MLP latency is flat ("What carries the argument"; referee major 4 on
  §3.6, w_Attn ~ t_Attn / Delta);
* value -- the cosine between a draft state and X^(i), the state the
  unpruned model reaches at the same depth (Eq. 6; referee major 1 on §3.4
  Eq. 8 / Algorithm 1);
* recurrence -- one hidden state g[i, j] per (item, budget); it keeps whichever
  of "execute item i" and "skip item i" has the higher cosine to X^(i) (Eq. 7/8,
  Algorithm 1); one candidate layer set per budget is read back by walking the
  choices (Algorithm 2, referee minor 4);
* selection -- TPT(S, gamma) = ((1 - a^(gamma+1)) / (1 - a)) / (gamma t_Draft(S)
  + t_Target) maximised over the candidate pool and gamma <= D (Eq. 4, Eq. 5).

Section labels below name the steps of the solve: a0 item weights and the
budget grid, a1 reference states, a2 / a3 the Attention / MLP sublayer on a
batch of states, a4 the select with its backpointer, a5 the reconstruction,
a6 the TPT grid search.

Readings where the page is silent or ambiguous (each is one switch or one line
below and is listed with its reason in the design notes):

R1 budget = "at most b latency units used"; every cell starts from X^(0).  The
   paper's exact-budget initialisation (only g[0, 0] valid) is ``mode="exact"``.
R2 cells are indexed by used budget b: skip keeps cell b, execute reads cell
   b - w_i.
R3 execute wins only if its cosine is strictly larger (skip keeps exact ties).
R4 backtracking walks stored 1-byte backpointers (no matrix comparisons).
R5 the value of a cell is the mean over the T evaluation tokens of the
   per-token cosine.
R6 the compared state is the residual stream right after item i.
R7 a candidate's queries attend over the full model's cached keys/values of
   all ctx+T positions (the evaluation tokens are already verified); token t
   sees positions <= ctx + t.  Wk/Wv are not used by the DP.
R7w the alternative, ``kv="window"``: the keys/values of the T window
   positions ctx .. ctx+T-1 are recomputed from the candidate's own normalised
   state through the layer's Wk/Wv (keys rotated at their positions); positions
   0 .. ctx-1 still come from the full model's cache.  Token t sees the same
   positions as under R7.
R8 RoPE is the rotate-half form, theta_j = base^(-2j/hd), position ctx + t;
   only the candidate's queries are rotated (the cache holds rotated keys).
R9 RMSNorm y = x / sqrt(mean(x^2) + eps) * g.
R10 w_i = max(1, floor(t_i / Delta + 1/2)) with Delta = sum(t) / n_bins.
R11 t_Draft(S) = sum of t_i over S, t_Target = sum over all items.
R12 alpha_S = clamp((value - lo) / scale, 0, alpha_max) (a stated stand-in for
   the paper's history-based estimate, Eq. 9).
R13 TPT ties: larger TPT, then smaller b, then smaller gamma.
R14 b = 0 (the empty set) takes part in the grid search.
R15 cosine pruning (optional): a cell whose kept value is below tau is dropped.
R16 skip cap (optional): after item k the cells b < W_k - cap are dropped.

Item numbering: items k = 0 .. 2L-1; item 2l is the Attention sublayer of
layer l and item 2l+1 its MLP sublayer.  X^(0) is the evaluation tokens' input
state and X^(k+1) = item_k(X^(k)).
"""
from __future__ import annotations

import itertools
import math
from dataclasses import dataclass, field
from typing import Callable, Dict, List, Optional, Sequence, Tuple

import numpy as np

F64 = np.float64


# --------------------------------------------------------------------------
# a0: latency weights and the budget grid
# --------------------------------------------------------------------------
def quantize_weights(t: Sequence[float], n_bins: int) -> List[int]:
    """Integer item weights w_i = max(1, floor(t_i/Delta + 1/2)), Delta = sum(t)/n_bins.

    Follows the review's note that w_Attn is about t_Attn/Delta (referee major 4,
    on §3.6); the rounding rule is reading R10.  The sum runs in item order.
    """
    if n_bins <= 0:
        raise ValueError("n_bins must be positive")
    total = 0.0
    for x in t:
        if not (x > 0.0):
            raise ValueError("latencies must be positive")
        total += float(x)
    delta = total / float(n_bins)
    return [max(1, int(math.floor(float(x) / delta + 0.5))) for x in t]


# --------------------------------------------------------------------------
# a2 / a3: one sublayer applied to a batch of hidden states
# --------------------------------------------------------------------------
@dataclass
class Model:
    """Decoder weights and the full model's KV cache, as plain arrays.

    ``layers[l]`` maps attn_norm [d], wq [Hq*hd][d], wo [d][Hq*hd], mlp_norm [d],
    w_gate [F][d], w_up [F][d], w_down [d][F] to arrays (any float dtype; they
    are widened to fp64 where used), and -- only for reading R7w -- wk and wv
    [Hkv*hd][d].  ``k_cache``/``v_cache`` are sequences over layers of
    [n_pos][Hkv][hd] arrays.
    """

    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    rms_eps: float
    rope_base: float
    layers: Sequence[Dict[str, np.ndarray]]
    k_cache: Sequence[np.ndarray]
    v_cache: Sequence[np.ndarray]

    @property
    def n_items(self) -> int:
        return 2 * len(self.layers)


def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """y = x / sqrt(mean(x^2) + eps) * g over the last axis (reading R9)."""
    x = np.asarray(x, F64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, F64)


def rope_rotate_half(q: np.ndarray, positions: np.ndarray, base: float) -> np.ndarray:
    """Rotate-half RoPE of q [..., T, H, hd] at the given per-token positions [T] (R8)."""
    hd = q.shape[-1]
    half = hd // 2
    j = np.arange(half, dtype=F64)
    theta = np.power(F64(base), -2.0 * j / hd)                  # [half]
    ang = np.asarray(positions, F64)[:, None] * theta[None, :]  # [T, half]
    c = np.cos(ang)[:, None, :]                                 # [T, 1, half]
    s = np.sin(ang)[:, None, :]
    q1 = q[..., :half]
    q2 = q[..., half:]
    return np.concatenate([q1 * c - q2 * s, q2 * c + q1 * s], axis=-1)


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def attention_core(q: np.ndarray, k: np.ndarray, v: np.ndarray, ctx: int,
                   n_kv_heads: int) -> np.ndarray:
    """Causal GQA attention of the evaluation tokens' queries over the cache (R7).

    q [M, T, Hq, hd] (already rotated), k/v [n_pos, Hkv, hd]; token t attends to
    cache positions 0 .. ctx+t.  Query head h reads kv head h // (Hq / Hkv).
    Returns [M, T, Hq, hd].
    """
    M, T, Hq, hd = q.shape
    group = Hq // n_kv_heads
    n_keys = ctx + T
    if k.shape[0] < n_keys or v.shape[0] < n_keys:
        raise ValueError("the cache holds fewer than ctx + T positions")
    kf = np.asarray(k[:n_keys], F64)
    vf = np.asarray(v[:n_keys], F64)
    allowed = np.arange(n_keys)[None, :] <= (ctx + np.arange(T))[:, None]   # [T, n_keys]
    out = np.empty_like(q)
    scale = 1.0 / math.sqrt(hd)
    # bound the fp64 score block to about 256 MB
    rows_per_chunk = max(1, int(2 ** 25 // max(1, n_keys * T * group)))
    for g in range(n_kv_heads):
        kg = kf[:, g, :]                       # [n_keys, hd]
        vg = vf[:, g, :]
        for m0 in range(0, M, rows_per_chunk):
            m1 = min(M, m0 + rows_per_chunk)
            qg = q[m0:m1, :, g * group:(g + 1) * group, :]     # [m, T, group, hd]
            mm = m1 - m0
            s = (qg.reshape(-1, hd) @ kg.T).reshape(mm, T, group, n_keys) * scale
            s = np.where(allowed[None, :, None, :], s, -np.inf)
            s = s - s.max(axis=-1, keepdims=True)
            p = np.exp(s)
            p = p / p.sum(axis=-1, keepdims=True)
            out[m0:m1, :, g * group:(g + 1) * group, :] = \
                (p.reshape(-1, n_keys) @ vg).reshape(mm, T, group, hd)
    return out


def window_kv(model: Model, layer: int, xh: np.ndarray, ctx: int) -> Tuple[np.ndarray, np.ndarray]:
    """Keys and values of the T window positions from normalised states xh [M, T, d]
    (reading R7w): k = RoPE(xh Wk^T) at positions ctx + t, v = xh Wv^T; each
    [M, T, Hkv, hd]."""
    Lw = model.layers[layer]
    M, T, d = xh.shape
    shape = (M, T, model.n_kv_heads, model.head_dim)
    k = (xh.reshape(M * T, d) @ np.asarray(Lw["wk"], F64).T).reshape(shape)
    k = rope_rotate_half(k, ctx + np.arange(T), model.rope_base)
    v = (xh.reshape(M * T, d) @ np.asarray(Lw["wv"], F64).T).reshape(shape)
    return k, v


def attn_item(model: Model, layer: int, H: np.ndarray, ctx: int, kv: str = "cache") -> np.ndarray:
    """Attention sublayer on states H [M, T, d]: H + Attn(RMSNorm(H)) (R6-R9).

    ``kv="cache"`` reads every key/value from the full model's cache (R7);
    ``kv="window"`` replaces the window positions' keys/values by the
    candidate's own (R7w), so each state attends over its own key set.
    """
    Lw = model.layers[layer]
    M, T, d = H.shape
    xh = rms_norm(H, Lw["attn_norm"], model.rms_eps)
    q = xh.reshape(M * T, d) @ np.asarray(Lw["wq"], F64).T
    q = q.reshape(M, T, model.n_q_heads, model.head_dim)
    q = rope_rotate_half(q, ctx + np.arange(T), model.rope_base)
    if kv == "cache":
        o = attention_core(q, model.k_cache[layer], model.v_cache[layer], ctx, model.n_kv_heads)
    elif kv == "window":
        kw, vw = window_kv(model, layer, xh, ctx)
        kc = np.asarray(model.k_cache[layer][:ctx], F64)
        vc = np.asarray(model.v_cache[layer][:ctx], F64)
        o = np.concatenate([
            attention_core(q[m:m + 1], np.concatenate([kc, kw[m]]), np.concatenate([vc, vw[m]]),
                           ctx, model.n_kv_heads)
            for m in range(M)])
    else:
        raise ValueError(kv)
    y = o.reshape(M * T, -1) @ np.asarray(Lw["wo"], F64).T
    return H + y.reshape(M, T, d)


def mlp_item(model: Model, layer: int, H: np.ndarray) -> np.ndarray:
    """SwiGLU MLP sublayer on states H [M, T, d]: H + W_down(silu(W_gate x) * W_up x)."""
    Lw = model.layers[layer]
    M, T, d = H.shape
    xh = rms_norm(H, Lw["mlp_norm"], model.rms_eps).reshape(M * T, d)
    a = xh @ np.asarray(Lw["w_gate"], F64).T
    b = xh @ np.asarray(Lw["w_up"], F64).T
    u = silu(a) * b
    y = u @ np.asarray(Lw["w_down"], F64).T
    return H + y.reshape(M, T, d)


def apply_item(model: Model, k: int, H: np.ndarray, ctx: int, per_cell: bool = False,
               kv: str = "cache") -> np.ndarray:
    """Item k (2l = Attention of layer l, 2l+1 = MLP of layer l) on H [M, T, d].

    With ``per_cell`` each of the M states goes through its own call, so every
    state sees exactly the arithmetic of a single-state call (used where a
    bit-for-bit comparison with the reference chain is wanted).  ``kv`` picks
    reading R7 ("cache") or R7w ("window") for the Attention items.
    """
    H = np.asarray(H, F64)
    if per_cell and H.shape[0] > 1:
        return np.concatenate([apply_item(model, k, H[m:m + 1], ctx, kv=kv)
                               for m in range(H.shape[0])])
    layer = k // 2
    if k % 2 == 0:
        return attn_item(model, layer, H, ctx, kv=kv)
    return mlp_item(model, layer, H)


# --------------------------------------------------------------------------
# a1: reference states; value function
# --------------------------------------------------------------------------
def reference_states(model: Model, x0: np.ndarray, ctx: int, kv: str = "cache") -> np.ndarray:
    """X^(0) = x0 and X^(k+1) = item_k(X^(k)) for the full model: [2L+1, T, d]."""
    x = np.asarray(x0, F64)[None]
    out = [x[0]]
    for k in range(model.n_items):
        x = apply_item(model, k, x, ctx, kv=kv)
        out.append(x[0])
    return np.stack(out)


def meancos(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """Mean over tokens of the per-token cosine of A [..., T, d] with B [T, d] (R5).

    cos_t = (a_t . b_t) / sqrt((a_t . a_t)(b_t . b_t)).
    """
    A = np.asarray(A, F64)
    B = np.asarray(B, F64)
    dot = np.sum(A * B, axis=-1)
    na = np.sum(A * A, axis=-1)
    nb = np.sum(B * B, axis=-1)
    return np.mean(dot / np.sqrt(na * nb), axis=-1)


# --------------------------------------------------------------------------
# a4 / a5: the DP skeleton (select + backpointer) and reconstruction
# --------------------------------------------------------------------------
@dataclass
class DPResult:
    bp: np.ndarray            # [n_items, C] uint8, 1 = execute
    val: np.ndarray           # [n_items+1, C] value of each cell (nan where invalid)
    cos_s: np.ndarray         # [n_items, C] skip candidate's value (nan if absent)
    cos_e: np.ndarray         # [n_items, C] execute candidate's value (nan if absent)
    valid: np.ndarray         # [n_items+1, C] bool
    final_states: Optional[np.ndarray] = None


def knapsack_dp(w: Sequence[int], n_cells: int, init_states: np.ndarray,
                init_valid: np.ndarray,
                item_fn: Callable[[int, np.ndarray], np.ndarray],
                score_fn: Callable[[int, np.ndarray], np.ndarray],
                prune: Optional[Callable[[int, np.ndarray, np.ndarray], np.ndarray]] = None
                ) -> DPResult:
    """Row-by-row 0/1-knapsack DP that keeps one state per (item, budget) cell.

    Eq. 7/8 and Algorithm 1 as the review describes them (referee major 1 and
    minor 2): for item k with weight w_k and every cell b, the "skip" candidate
    is the previous row's state at b and the "execute" candidate is item_k
    applied to the previous row's state at b - w_k (reading R2); the candidate
    with the larger score is kept, execute only when strictly larger (R3), and
    the choice is stored as a backpointer (R4).  ``score_fn(k+1, states)``
    scores states against the target of row k+1.  ``prune(k+1, values,
    valid)`` may then drop cells of the new row (they become invalid: no
    later candidate reads them); it is how the review's cosine threshold and
    skipped-weight cap (R15, R16) enter.
    """
    n_items = len(w)
    C = n_cells
    prev = np.array(init_states, copy=True)
    valid = np.array(init_valid, dtype=bool, copy=True)
    bp = np.zeros((n_items, C), dtype=np.uint8)
    val = np.full((n_items + 1, C), np.nan)
    cos_s = np.full((n_items, C), np.nan)
    cos_e = np.full((n_items, C), np.nan)
    vrows = np.zeros((n_items + 1, C), dtype=bool)
    vrows[0] = valid
    s0 = score_fn(0, prev)
    val[0] = np.where(valid, s0, np.nan)
    for k in range(n_items):
        wk = int(w[k])
        skip = score_fn(k + 1, prev)
        cur = np.array(prev, copy=True)
        cur_valid = valid.copy()
        cur_val = np.where(valid, skip, np.nan)
        cos_s[k] = np.where(valid, skip, np.nan)
        if wk < C:
            src_idx = np.nonzero(valid[:C - wk])[0]           # execute sources that exist
            if src_idx.size:
                ex = item_fn(k, prev[src_idx])
                ex_score = score_fn(k + 1, ex)
                for j, e_src in enumerate(src_idx):
                    b = int(e_src) + wk
                    e = float(ex_score[j])
                    cos_e[k, b] = e
                    if (not valid[b]) or e > float(skip[b]):
                        cur[b] = ex[j]
                        cur_valid[b] = True
                        cur_val[b] = e
                        bp[k, b] = 1
        if prune is not None:
            cur_valid = np.asarray(prune(k + 1, cur_val, cur_valid), dtype=bool)
            cur_val = np.where(cur_valid, cur_val, np.nan)
        prev, valid = cur, cur_valid
        val[k + 1] = cur_val
        vrows[k + 1] = valid
    return DPResult(bp=bp, val=val, cos_s=cos_s, cos_e=cos_e, valid=vrows, final_states=prev)


def reconstruct(bp: np.ndarray, w: Sequence[int], b: int) -> Tuple[List[int], int]:
    """Walk the backpointers of cell b from the last item down (Algorithm 2, R4).

    Returns (sorted executed items, used weight).
    """
    j = int(b)
    chosen = []
    for k in range(bp.shape[0] - 1, -1, -1):
        if bp[k, j]:
            chosen.append(k)
            j -= int(w[k])
            if j < 0:
                raise AssertionError("backpointer walk left the budget grid")
    chosen.reverse()
    return chosen, int(b) - j


# --------------------------------------------------------------------------
# The full DP on a decoder
# --------------------------------------------------------------------------
@dataclass
class Solve:
    w: List[int]
    t: List[float]
    ref: np.ndarray                 # [2L+1, T, d]
    dp: DPResult
    sets: List[List[int]]           # per cell b: executed items
    used_w: np.ndarray              # [C] int
    t_draft: np.ndarray             # [C] float
    values: np.ndarray              # [C] final-row value
    best_b: int = -1
    best_gamma: int = -1
    best_tpt: float = float("nan")
    tpt: Optional[np.ndarray] = None   # [C, G]


def dp_solve(model: Model, x0: np.ndarray, ctx: int, w: Sequence[int], t: Sequence[float],
             gamma_max: int, n_cells: Optional[int] = None, mode: str = "at_most",
             per_cell: bool = False, ref: Optional[np.ndarray] = None,
             alpha_lo: float = 0.5, alpha_scale: float = 0.5, alpha_max: float = 0.99,
             keep_states: bool = False, prune_tau: Optional[float] = None,
             skip_cap: Optional[int] = None, kv: str = "cache") -> Solve:
    """KnapSpec's DP over all budget cells, reconstruction and TPT selection.

    ``n_cells`` < K+1 computes only the budgets 0 .. n_cells-1, which equal the
    full DP's cells there (every read goes to an equal or smaller budget).  The
    TPT search then runs over those cells only.

    ``prune_tau`` drops a cell whose kept value is below tau (the review's
    cosine threshold tau = 0.5, "Assumptions & free parameters" and referee
    notes on Fig. 4; reading R15); ``skip_cap`` drops, after item k, the cells
    b < W_k - cap, W_k = w_0 + .. + w_k (the skipped-weight cap K/2 of the
    review's "Reading between the lines"; reading R16).  A dropped cell is
    invalid: its value is NaN, no later candidate reads it, and a final
    invalid cell has no set.

    ``kv`` picks the attention's key/value reading for every item, the
    reference chain included: R7 ("cache") or R7w ("window").
    """
    x0 = np.asarray(x0, F64)
    n_items = model.n_items
    if len(w) != n_items or len(t) != n_items:
        raise ValueError("need one weight and one latency per item")
    K = int(sum(int(x) for x in w))
    C = K + 1 if n_cells is None else int(n_cells)
    if ref is None:
        ref = reference_states(model, x0, ctx, kv=kv)
    T, d = x0.shape
    init = np.broadcast_to(x0, (C, T, d)).copy()
    if mode == "at_most":
        init_valid = np.ones(C, dtype=bool)
    elif mode == "exact":
        init_valid = np.zeros(C, dtype=bool)
        init_valid[0] = True
    else:
        raise ValueError(mode)

    dp = knapsack_dp(w, C, init, init_valid,
                     lambda k, H: apply_item(model, k, H, ctx, per_cell=per_cell, kv=kv),
                     lambda r, H: meancos(H, ref[r]),
                     prune=pruning_rule(w, C, prune_tau, skip_cap))
    sets, used = [], np.zeros(C, dtype=np.int64)
    t_draft = np.zeros(C)
    for b in range(C):
        if not dp.valid[n_items, b]:
            sets.append([])
            used[b] = -1
            t_draft[b] = np.nan
            continue
        s, u = reconstruct(dp.bp, w, b)
        sets.append(s)
        used[b] = u
        acc = 0.0
        for k in s:
            acc += float(t[k])
        t_draft[b] = acc
    out = Solve(w=list(map(int, w)), t=list(map(float, t)), ref=ref, dp=dp, sets=sets,
                used_w=used, t_draft=t_draft, values=dp.val[n_items].copy())
    if not keep_states:
        dp.final_states = None
    t_target = 0.0
    for x in t:
        t_target += float(x)
    grid = tpt_grid(out.values, t_draft, t_target, gamma_max, alpha_lo, alpha_scale, alpha_max)
    out.tpt = grid
    out.best_b, out.best_gamma, out.best_tpt = tpt_argmax(grid)
    return out


def pruning_rule(w: Sequence[int], n_cells: int, prune_tau: Optional[float],
                 skip_cap: Optional[int]):
    """The prune callback of knapsack_dp for a cosine threshold and a skip cap.

    After item k (row r = k + 1): a cell stays valid only if its value is not
    below tau and its budget b is at least W_k - cap (a cell below that bound
    has skipped more than cap weight units whatever its exact usage).
    """
    if prune_tau is None and skip_cap is None:
        return None
    W = np.cumsum(np.asarray(w, dtype=np.int64))
    cells = np.arange(n_cells)

    def prune(r, vals, valid):
        v = np.array(valid, dtype=bool, copy=True)
        if skip_cap is not None:
            v &= cells >= W[r - 1] - int(skip_cap)
        if prune_tau is not None:
            v &= ~(np.nan_to_num(vals, nan=np.inf) < float(prune_tau))
        return v

    return prune


# --------------------------------------------------------------------------
# a6: TPT grid search
# --------------------------------------------------------------------------
def alpha_of(value: float, lo: float = 0.5, scale: float = 0.5, amax: float = 0.99) -> float:
    """Synthetic acceptance rate alpha = clamp((value - lo)/scale, 0, amax) (R12)."""
    a = (float(value) - lo) / scale
    return min(max(a, 0.0), amax)


def tpt(alpha: float, gamma: int, t_draft: float, t_target: float) -> float:
    """Tokens-per-time (Eq. 4): (sum_{k=0..gamma} alpha^k) / (gamma t_Draft + t_Target).

    The geometric sum is taken term by term, which equals (1-a^(g+1))/(1-a) and
    stays finite at a = 1.
    """
    acc = 0.0
    p = 1.0
    for _ in range(gamma + 1):
        acc += p
        p *= alpha
    return acc / (gamma * t_draft + t_target)


def tpt_grid(values: np.ndarray, t_draft: np.ndarray, t_target: float, gamma_max: int,
             lo: float = 0.5, scale: float = 0.5, amax: float = 0.99) -> np.ndarray:
    """TPT(b, gamma) for every cell b and gamma = 1..gamma_max (nan for invalid cells)."""
    C = len(values)
    g = np.full((C, gamma_max), np.nan)
    for b in range(C):
        if not np.isfinite(values[b]) or not np.isfinite(t_draft[b]):
            continue
        a = alpha_of(values[b], lo, scale, amax)
        for gam in range(1, gamma_max + 1):
            g[b, gam - 1] = tpt(a, gam, float(t_draft[b]), t_target)
    return g


def tpt_argmax(grid: np.ndarray) -> Tuple[int, int, float]:
    """Grid search of Eq. 5: largest TPT, ties to smaller b, then smaller gamma (R13)."""
    best = (-1, -1, -np.inf)
    for b in range(grid.shape[0]):
        for gi in range(grid.shape[1]):
            v = grid[b, gi]
            if np.isfinite(v) and v > best[2]:
                best = (b, gi + 1, float(v))
    return best


# --------------------------------------------------------------------------
# Checks that use the same pieces: re-running a set, exhaustive search
# --------------------------------------------------------------------------
def chain(model: Model, x0: np.ndarray, ctx: int, items: Sequence[int],
          upto: Optional[int] = None, kv: str = "cache") -> np.ndarray:
    """Run the executed items (in order) on x0; items >= upto are ignored."""
    x = np.asarray(x0, F64)[None]
    n = model.n_items if upto is None else upto
    for k in range(n):
        if k in items:
            x = apply_item(model, k, x, ctx, kv=kv)
    return x[0]


def eval_set(model: Model, x0: np.ndarray, ctx: int, items: Sequence[int],
             ref: np.ndarray, upto: Optional[int] = None, kv: str = "cache") -> float:
    """Value of a layer set re-run from scratch: meancos(chain(x0), X^(upto))."""
    n = model.n_items if upto is None else upto
    return float(meancos(chain(model, x0, ctx, set(items), n, kv=kv)[None], ref[n])[0])


def brute_force(model: Model, x0: np.ndarray, ctx: int, w: Sequence[int], ref: np.ndarray,
                n_items: Optional[int] = None,
                kv: str = "cache") -> Tuple[np.ndarray, List[Tuple[int, ...]]]:
    """Best value over all subsets of the first n_items items for every budget b.

    best[b] = max over S with sum(w_S) <= b of meancos(chain_S(x0), X^(n_items)):
    the exhaustive enumeration the review asks for ("What would settle it").
    Returns (best [K+1], argmax subsets).  Subsets are walked depth first so
    shared prefixes are computed once.
    """
    n = model.n_items if n_items is None else n_items
    K = int(sum(int(w[k]) for k in range(n)))
    best = np.full(K + 1, -np.inf)
    arg: List[Tuple[int, ...]] = [()] * (K + 1)
    x0 = np.asarray(x0, F64)

    def visit(k: int, state: np.ndarray, used: int, chosen: Tuple[int, ...]):
        if k == n:
            v = float(meancos(state[None], ref[n])[0])
            if v > best[used]:
                best[used] = v
                arg[used] = chosen
            return
        visit(k + 1, state, used, chosen)
        visit(k + 1, apply_item(model, k, state[None], ctx, kv=kv)[0], used + int(w[k]),
              chosen + (k,))

    visit(0, x0, 0, ())
    # "at most b": running maximum over budgets
    for b in range(1, K + 1):
        if best[b - 1] > best[b]:
            best[b] = best[b - 1]
            arg[b] = arg[b - 1]
    return best, arg


# --------------------------------------------------------------------------
# Scalar special case: the DP skeleton on numbers is the textbook 0/1 knapsack
# --------------------------------------------------------------------------
def scalar_knapsack_dp(w: Sequence[int], v: Sequence[int], capacity: int,
                       mode: str = "at_most", prune_tau: Optional[float] = None,
                       skip_cap: Optional[int] = None) -> Tuple[np.ndarray, DPResult]:
    """The same DP skeleton with state = running value, item(k, x) = x + v_k, score = x.

    With additive item values the keep-the-better rule is exactly the classic
    0/1 knapsack recurrence, so the result must equal the knapsack optimum for
    every capacity 0..capacity ("at most" mode) or exactly-filled capacity.
    Returns (values [capacity+1] as float, DPResult); invalid cells are -inf.
    """
    C = capacity + 1
    init = np.zeros(C, dtype=F64)
    if mode == "at_most":
        iv = np.ones(C, dtype=bool)
    else:
        iv = np.zeros(C, dtype=bool)
        iv[0] = True
    vv = np.asarray(v, F64)
    res = knapsack_dp(w, C, init, iv, lambda k, H: H + vv[k], lambda r, H: np.asarray(H, F64),
                      prune=pruning_rule(w, C, prune_tau, skip_cap))
    vals = np.where(res.valid[len(w)], res.val[len(w)], -np.inf)
    return vals, res


# --------------------------------------------------------------------------
# The full model's prefill: the KV cache "from the full model"
# --------------------------------------------------------------------------
@dataclass
class Prefill:
    k_cache: np.ndarray    # [L, n, Hkv, hd] rotated keys of every position
    v_cache: np.ndarray    # [L, n, Hkv, hd]
    hidden: np.ndarray     # [2L+1, n, d] residual stream after each item (row 0 = emb)


def prefill(model: Model, emb: np.ndarray) -> Prefill:
    """Run the full decoder over a token sequence emb [n, d] (positions 0 .. n-1)
    with causal self-attention, recording each layer's keys and values.

    This is how the workloads' "KV cache from the full model" is produced for the
    small configurations: the cache the DP reads (reading R7) holds what the
    unpruned model computed for every position, the evaluation tokens' included.
    Per layer (the same sublayer definitions as attn_item / mlp_item): x^ =
    RMSNorm(h); q = RoPE(x^ Wq^T), k = RoPE(x^ Wk^T) and v = x^ Wv^T at each
    token's own position (reading R8); position i attends to positions 0 .. i,
    query head h to kv head h // (Hq / Hkv); h += o Wo^T; then the MLP item.
    Needs Wk / Wv in every layer.
    """
    h = np.asarray(emb, F64)
    n, d = h.shape
    L = len(model.layers)
    Hq, Hkv, hd = model.n_q_heads, model.n_kv_heads, model.head_dim
    group = Hq // Hkv
    pos = np.arange(n)
    causal = pos[None, :] <= pos[:, None]                      # [query, key]
    kc = np.empty((L, n, Hkv, hd))
    vc = np.empty((L, n, Hkv, hd))
    hidden = [h]
    for l in range(L):
        Lw = model.layers[l]
        xh = rms_norm(h, Lw["attn_norm"], model.rms_eps)
        q = (xh @ np.asarray(Lw["wq"], F64).T).reshape(1, n, Hq, hd)
        k = (xh @ np.asarray(Lw["wk"], F64).T).reshape(1, n, Hkv, hd)
        v = (xh @ np.asarray(Lw["wv"], F64).T).reshape(n, Hkv, hd)
        q = rope_rotate_half(q, pos, model.rope_base)[0]
        k = rope_rotate_half(k, pos, model.rope_base)[0]
        kc[l], vc[l] = k, v
        o = np.empty((n, Hq, hd))
        for hq in range(Hq):
            g = hq // group
            sc = (q[:, hq, :] @ k[:, g, :].T) / math.sqrt(hd)
            sc = np.where(causal, sc, -np.inf)
            sc = sc - sc.max(axis=-1, keepdims=True)
            p = np.exp(sc)
            o[:, hq, :] = (p / p.sum(axis=-1, keepdims=True)) @ v[:, g, :]
        h = h + o.reshape(n, Hq * hd) @ np.asarray(Lw["wo"], F64).T
        hidden.append(h)
        h = mlp_item(model, l, h[None])[0]
        hidden.append(h)
    return Prefill(k_cache=kc, v_cache=vc, hidden=np.stack(hidden))


# --------------------------------------------------------------------------
# Lemma 4.1 checker: does cosine closeness guarantee the same greedy token?
# --------------------------------------------------------------------------
@dataclass
class LemmaCheck:
    istar: np.ndarray      # [T] greedy token of the reference state
    margin: np.ndarray     # [T] xi = z_i* - max_{j != i*} z_j
    dist: np.ndarray       # [T] D = max_j ||w_i* - w_j||
    cos: np.ndarray        # [N, T] cosine of each state's token with the reference token
    bound: np.ndarray      # [N, T] the sufficient condition ||h - h'|| < xi / D holds
    agree: np.ndarray      # [N, T] argmax W h' == i*
    state_margin: np.ndarray   # [N, T] top-1 minus top-2 logit of h'
    slack: np.ndarray      # [N, T] xi / D - ||h - h'||


def lemma_check(states: np.ndarray, ref: np.ndarray, lm_head: np.ndarray,
                final_gain: Optional[np.ndarray], eps: float) -> LemmaCheck:
    """The review's Lemma 4.1 (KnapSpec §4, referee major 2 and "What carries the
    argument") evaluated on DP states.

    h = RMSNorm(ref_t) and h' = RMSNorm(state_t) rescaled to ||h|| (the lemma's
    equal-norm premise).  With logits z = W h, i* = argmax z, margin
    xi = z_i* - max_{j != i*} z_j and D = max_j ||w_i* - w_j||, the lemma says
    ||h - h'|| < xi / D implies argmax W h' = i*: for every j,
    (w_i* - w_j).h' >= (w_i* - w_j).h - ||w_i* - w_j|| ||h' - h|| >= xi - D ||h' - h|| > 0
    (Cauchy-Schwarz).  Equal norms give ||h - h'||^2 = 2 ||h||^2 (1 - cos).
    """
    W = np.asarray(lm_head, F64)
    S = np.asarray(states, F64)
    R = np.asarray(ref, F64)
    g = np.ones(R.shape[-1]) if final_gain is None else np.asarray(final_gain, F64)
    h = rms_norm(R, g, eps)                          # [T, d]
    hp = rms_norm(S, g, eps)                         # [N, T, d]
    nh = np.linalg.norm(h, axis=-1)                  # [T]
    hp = hp * (nh / np.linalg.norm(hp, axis=-1))[..., None]
    z = h @ W.T                                      # [T, V]
    istar = np.argmax(z, axis=-1)
    top = np.sort(z, axis=-1)
    margin = top[:, -1] - top[:, -2]
    dist = np.array([np.max(np.linalg.norm(W - W[i], axis=-1)) for i in istar])
    cos = np.sum(hp * h[None], axis=-1) / (nh[None] * nh[None])
    gap = np.sqrt(np.maximum(2.0 * nh[None] ** 2 * (1.0 - cos), 0.0))   # ||h - h'||
    slack = margin[None] / dist[None] - gap
    zp = hp @ W.T                                    # [N, T, V]
    agree = np.argmax(zp, axis=-1) == istar[None]
    tp = np.sort(zp, axis=-1)
    return LemmaCheck(istar=istar, margin=margin, dist=dist, cos=cos, bound=slack > 0,
                      agree=agree, state_margin=tp[..., -1] - tp[..., -2], slack=slack)
