"""Thin ctypes binding of libknapspec.so (include/knapspec.h).

Every function here only marshals arguments: it checks tensor devices, dtypes
and shapes, turns them into pointers and calls the C ABI on the current torch
CUDA stream.  The C ABI takes bare pointers and cannot see a buffer's size, so
every shape the header fixes is checked here against the sizes passed beside
it: a wrongly sized tensor raises instead of reaching a kernel.  All arithmetic
of the DP runs in the library's CUDA kernels.  If the library has not been
built the first call raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libknapspec.so")

KS_F32, KS_BF16 = 0, 1


class KnapSpecError(RuntimeError):
    pass


class ModelDesc(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("ffn", ctypes.c_int32),
                ("rms_eps", ctypes.c_float), ("rope_base", ctypes.c_double),
                ("wdtype", ctypes.c_int32)]


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("attn_norm", "wq", "wo", "mlp_norm", "w_gate", "w_up", "w_down", "wk", "wv")]


KS_KV_CACHE, KS_KV_WINDOW = 0, 1
KV_MODES = {"cache": KS_KV_CACHE, "window": KS_KV_WINDOW}


class CacheDesc(ctypes.Structure):
    _fields_ = [("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("cache_rows", ctypes.c_int64), ("ctx", ctypes.c_int32),
                ("kv_mode", ctypes.c_int32)]


KS_BUDGET_AT_MOST, KS_BUDGET_EXACT = 0, 1


class Params(ctypes.Structure):
    _fields_ = [("gamma_max", ctypes.c_int32), ("n_bins", ctypes.c_int32),
                ("budget_mode", ctypes.c_int32),
                ("alpha_lo", ctypes.c_double), ("alpha_scale", ctypes.c_double),
                ("alpha_max", ctypes.c_double), ("prune_tau", ctypes.c_double),
                ("skip_cap", ctypes.c_int32), ("dedup", ctypes.c_int32)]


class Result(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("status", "values", "sets", "used_w", "t_draft", "bp", "cos_skip",
                 "cos_exec", "tpt", "best", "best_tpt", "ref_states", "exec_counts",
                 "final_states", "dedup_rejected")]


class KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int64),
                ("total_ms", ctypes.c_double), ("flops", ctypes.c_double),
                ("bytes", ctypes.c_double)]


EXPORTS = ["ks_version", "ks_last_error", "ks_status_string", "ks_quantize_weights",
           "ks_workspace_size", "ks_sublayer_forward", "ks_reference_forward",
           "ks_select_step", "ks_reconstruct", "ks_tpt_argmax", "ks_solve", "ks_solve_cells",
           "ks_profile_start", "ks_profile_stop", "ks_reference_forward_noalloc",
           "ks_workspace_status", "ks_gemm_bf16", "ks_attention_bf16",
           "ks_check_bounded_wait", "ks_lemma_workspace_size", "ks_lemma_check", "ks_eval_set",
           "ks_workspace_size_contexts", "ks_solve_contexts"]

_lib = None


def load() -> ctypes.CDLL:
    """Load libknapspec.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise KnapSpecError(f"{LIB_PATH} is missing: build it with "
                            "`python -m knapsack_layer_selection_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, D, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t
    sig = {
        "ks_version": ([], ctypes.c_char_p),
        "ks_last_error": ([], ctypes.c_char_p),
        "ks_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "ks_quantize_weights": ([P, I32, I32, P], ctypes.c_int),
        "ks_workspace_size": ([P, I32, I32, ctypes.POINTER(SZ)], ctypes.c_int),
        "ks_sublayer_forward": ([P, P, P, I32, I32, P, I32, P, P, SZ, P], ctypes.c_int),
        "ks_reference_forward": ([P, P, P, I32, P, P, P, SZ, P], ctypes.c_int),
        "ks_select_step": ([P, P, P, I32, I32, I32, I32, P, P, P, P, P, P], ctypes.c_int),
        "ks_reconstruct": ([P, P, P, I32, I32, P, P, P, P, P], ctypes.c_int),
        "ks_tpt_argmax": ([P, P, I32, D, P, P, P, P, P], ctypes.c_int),
        "ks_solve": ([P, P, P, I32, P, P, P, P, P, P, SZ, P, P], ctypes.c_int),
        "ks_solve_cells": ([I32, P, P, P, ctypes.POINTER(I32)], ctypes.c_int),
        "ks_profile_start": ([I32], ctypes.c_int),
        "ks_reference_forward_noalloc": ([P, P, P, I32, P, P, P], ctypes.c_int),
        "ks_workspace_status": ([P, ctypes.POINTER(I32), P], ctypes.c_int),
        "ks_gemm_bf16": ([P, P, P, P, I32, I32, I32, P, P], ctypes.c_int),
        "ks_check_bounded_wait": ([ctypes.c_uint32, P, P, P], ctypes.c_int),
        "ks_lemma_workspace_size": ([I32, I32, I32, I32, ctypes.POINTER(SZ)], ctypes.c_int),
        "ks_lemma_check": ([P, I32, P, I32, I32, P, ctypes.c_float, P, I32, P, SZ, P, P, P],
                           ctypes.c_int),
        "ks_attention_bf16": ([P, P, P, I64, I32, I32, I32, I32, I32, I32, P, P, P], ctypes.c_int),
        "ks_profile_stop": ([P, I32, ctypes.POINTER(I32)], ctypes.c_int),
        "ks_eval_set": ([P, P, P, I32, P, P, P, P, P, P, SZ, P], ctypes.c_int),
        "ks_workspace_size_contexts": ([P, I32, P, I32, ctypes.POINTER(SZ)], ctypes.c_int),
        "ks_solve_contexts": ([P, P, I32, P, I32, P, P, P, P, P, SZ, P, P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != 0:
        lib = load()
        raise KnapSpecError(f"{lib.ks_status_string(status).decode()}: "
                            f"{lib.ks_last_error().decode()}")


def _dev(t: Optional[torch.Tensor], dtype=None, name="tensor") -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise KnapSpecError(f"{name} must be a CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        raise KnapSpecError(f"{name} is on {t.device}, but calls run on the current device "
                            f"cuda:{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise KnapSpecError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise KnapSpecError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _shape(t: Optional[torch.Tensor], shape: Sequence[int], name: str) -> None:
    """Raise unless t is None or has exactly this shape."""
    if t is not None and tuple(t.shape) != tuple(shape):
        raise KnapSpecError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _rows(t: torch.Tensor, n: int, row: Sequence[int], name: str) -> None:
    """Raise unless t is [m][*row] with m >= n (a buffer of at least n rows)."""
    if t.dim() != 1 + len(row) or tuple(t.shape[1:]) != tuple(row) or t.shape[0] < n:
        raise KnapSpecError(f"{name} must have shape (>= {n}, {', '.join(map(str, row))}), "
                            f"got {tuple(t.shape)}")


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def version() -> str:
    return load().ks_version().decode()


# ---------------------------------------------------------------- descriptors
def model_desc(n_layers, d_model, n_q_heads, n_kv_heads, head_dim, ffn, rms_eps, rope_base,
               wdtype: str) -> ModelDesc:
    return ModelDesc(n_layers, d_model, n_q_heads, n_kv_heads, head_dim, ffn, rms_eps,
                     rope_base, KS_F32 if wdtype == "f32" else KS_BF16)


def _layer_shapes(m: ModelDesc) -> Dict[str, tuple]:
    d, qd, F = m.d_model, m.n_q_heads * m.head_dim, m.ffn
    kvd = m.n_kv_heads * m.head_dim
    return {"attn_norm": (d,), "wq": (qd, d), "wo": (d, qd), "mlp_norm": (d,),
            "w_gate": (F, d), "w_up": (F, d), "w_down": (d, F), "wk": (kvd, d), "wv": (kvd, d)}


OPTIONAL_WEIGHTS = ("wk", "wv")        # read only by the window key/value reading


def layer_array(layers: Sequence[Dict[str, torch.Tensor]], wdtype: torch.dtype,
                model: Optional[ModelDesc] = None):
    """Host array of the layers' device weight pointers; with a model, the
    layer count and every weight's shape are checked against it.  wk / wv are
    optional (NULL when a layer has none)."""
    if model is not None and len(layers) != model.n_layers:
        raise KnapSpecError(f"model has {model.n_layers} layers, got {len(layers)}")
    if model is not None:
        for i, L in enumerate(layers):
            for name, shape in _layer_shapes(model).items():
                if name in OPTIONAL_WEIGHTS and L.get(name) is None:
                    continue
                _shape(L[name], shape, f"layers[{i}].{name}")
    arr = (LayerWeights * len(layers))()
    for i, L in enumerate(layers):
        for name in ("attn_norm", "wq", "wo", "mlp_norm", "w_gate", "w_up", "w_down", "wk", "wv"):
            if name in OPTIONAL_WEIGHTS and L.get(name) is None:
                continue
            setattr(arr[i], name, _dev(L[name], wdtype, f"layers[{i}].{name}"))
    return arr


def cache_desc(k_cache: torch.Tensor, v_cache: torch.Tensor, ctx: int,
               model: Optional[ModelDesc] = None, kv: str = "cache") -> CacheDesc:
    """The KV cache [L][rows][Hkv][hd] of K and V; with a model, L >= n_layers,
    Hkv, hd and the dtype are checked against it.  kv: "cache" (every key and
    value from the cache) or "window" (the window's recomputed from each state)."""
    if kv not in KV_MODES:
        raise KnapSpecError(f"kv must be one of {sorted(KV_MODES)}, got {kv!r}")
    if k_cache.shape != v_cache.shape or k_cache.dim() != 4:
        raise KnapSpecError("k_cache / v_cache must both be [L][rows][Hkv][hd]")
    dt = None
    if model is not None:
        L, _, Hkv, hd = k_cache.shape
        if L < model.n_layers or Hkv != model.n_kv_heads or hd != model.head_dim:
            raise KnapSpecError(f"k_cache / v_cache must be [>= {model.n_layers}][rows]"
                                f"[{model.n_kv_heads}][{model.head_dim}], got {tuple(k_cache.shape)}")
        dt = torch.float32 if model.wdtype == KS_F32 else torch.bfloat16
    return CacheDesc(_dev(k_cache, dt, "k_cache"), _dev(v_cache, dt, "v_cache"),
                     k_cache.shape[1], ctx, KV_MODES[kv])


def params(gamma_max: int, n_bins: int = 0, alpha_lo: float = 0.5, alpha_scale: float = 0.5,
           alpha_max: float = 0.99, budget_mode: str = "at_most",
           prune_tau: Optional[float] = None, skip_cap: Optional[int] = None,
           dedup=False) -> Params:
    """dedup: False / True, or "weak" for 8-bit fingerprints (every fold then
    rests on the byte comparison; a self-test of that check)."""
    mode = {"at_most": KS_BUDGET_AT_MOST, "exact": KS_BUDGET_EXACT}[budget_mode]
    dd = 2 if dedup == "weak" else (1 if dedup else 0)
    return Params(gamma_max, n_bins, mode, alpha_lo, alpha_scale, alpha_max,
                  float("-inf") if prune_tau is None else float(prune_tau),
                  -1 if skip_cap is None else int(skip_cap), dd)


# ---------------------------------------------------------------- calls
def quantize_weights(t: Sequence[float], n_bins: int) -> List[int]:
    n = len(t)
    tt = (ctypes.c_double * n)(*t)
    w = (ctypes.c_int32 * n)()
    _check(load().ks_quantize_weights(tt, n, n_bins, w))
    return list(w)


def workspace_size(model: ModelDesc, n_cells: int, T: int) -> int:
    out = ctypes.c_size_t()
    _check(load().ks_workspace_size(ctypes.byref(model), n_cells, T, ctypes.byref(out)))
    return out.value


def workspace(model: ModelDesc, n_cells: int, T: int, device="cuda") -> torch.Tensor:
    return torch.empty(workspace_size(model, n_cells, T), dtype=torch.uint8, device=device)


def sublayer_forward(model: ModelDesc, layers, cache: CacheDesc, T: int, item: int,
                     states_in: torch.Tensor, states_out: torch.Tensor,
                     ws: torch.Tensor) -> None:
    E = states_in.shape[0] if states_in.dim() == 3 else 1
    _shape(states_in, (E, T, model.d_model) if states_in.dim() == 3 else (T, model.d_model),
           "states_in")
    _shape(states_out, tuple(states_in.shape), "states_out")
    _check(load().ks_sublayer_forward(ctypes.byref(model), layers, ctypes.byref(cache), T, item,
                                      _dev(states_in, torch.float32, "states_in"), E,
                                      _dev(states_out, torch.float32, "states_out"),
                                      _dev(ws, name="workspace"), ws.numel(), _stream()))


def _ref_shapes(model: ModelDesc, T: int, x0: torch.Tensor, ref_out: torch.Tensor) -> None:
    _shape(x0, (T, model.d_model), "x0")
    _shape(ref_out, (2 * model.n_layers + 1, T, model.d_model), "ref_out")


def reference_forward(model: ModelDesc, layers, cache: CacheDesc, T: int, x0: torch.Tensor,
                      ref_out: torch.Tensor, ws: torch.Tensor) -> None:
    _ref_shapes(model, T, x0, ref_out)
    _check(load().ks_reference_forward(ctypes.byref(model), layers, ctypes.byref(cache), T,
                                       _dev(x0, torch.float32, "x0"),
                                       _dev(ref_out, torch.float32, "ref_out"),
                                       _dev(ws, name="workspace"), ws.numel(), _stream()))


def reference_forward_noalloc(model: ModelDesc, layers, cache: CacheDesc, T: int,
                              x0: torch.Tensor, ref_out: torch.Tensor) -> None:
    """ks_reference_forward using the library's fixed scratch array (no workspace)."""
    _ref_shapes(model, T, x0, ref_out)
    _check(load().ks_reference_forward_noalloc(ctypes.byref(model), layers, ctypes.byref(cache),
                                               T, _dev(x0, torch.float32, "x0"),
                                               _dev(ref_out, torch.float32, "ref_out"),
                                               _stream()))


def set_mask(items: Sequence[int], n_items: int):
    """Host bitmask of a layer set (bit k = item k), as ks_eval_set takes it."""
    words = (ctypes.c_uint64 * ((n_items + 63) // 64))()
    for k in items:
        if not 0 <= int(k) < n_items:
            raise KnapSpecError(f"item {k} is outside 0 .. {n_items - 1}")
        words[int(k) >> 6] |= 1 << (int(k) & 63)
    return words


def eval_set(model: ModelDesc, layers, cache: CacheDesc, T: int, x0: torch.Tensor,
             target: torch.Tensor, items: Sequence[int], ws: torch.Tensor,
             value_out: torch.Tensor, state_out: Optional[torch.Tensor] = None) -> None:
    """Run only the given items on x0 and score the state against target
    (ks_eval_set): value_out [1] = meancos(state, target); state_out [T][d]."""
    d = model.d_model
    _shape(x0, (T, d), "x0")
    _shape(target, (T, d), "target")
    _shape(value_out, (1,), "value_out")
    _shape(state_out, (T, d), "state_out")
    mask = set_mask(items, 2 * model.n_layers)
    _check(load().ks_eval_set(ctypes.byref(model), layers, ctypes.byref(cache), T,
                              _dev(x0, torch.float32, "x0"), _dev(target, torch.float32, "target"),
                              mask, _dev(value_out, torch.float32, "value_out"),
                              _dev(state_out, torch.float32, "state_out"),
                              _dev(ws, name="workspace"), ws.numel(), _stream()))


def workspace_status(ws: torch.Tensor) -> int:
    """Device status word of the last sublayer/reference call on this workspace."""
    out = ctypes.c_int32()
    _check(load().ks_workspace_status(_dev(ws, name="workspace"), ctypes.byref(out), _stream()))
    return out.value


def gemm_bf16(A: torch.Tensor, Bw: torch.Tensor, C: torch.Tensor,
              resid: Optional[torch.Tensor] = None,
              status: Optional[torch.Tensor] = None) -> None:
    """C = A . Bw^T (+ resid) on the tensor cores (A [M][K], Bw [N][K] bf16; C fp32)."""
    M, K = A.shape
    N = Bw.shape[0]
    _shape(Bw, (N, K), "B")
    _shape(C, (M, N), "C")
    _shape(resid, (M, N), "resid")
    if status is not None and status.numel() < 1:
        raise KnapSpecError("status must hold one int32")
    _check(load().ks_gemm_bf16(_dev(A, torch.bfloat16, "A"), _dev(Bw, torch.bfloat16, "B"),
                               _dev(C, torch.float32, "C"), _dev(resid, torch.float32, "resid"),
                               M, N, K, _dev(status, torch.int32, "status"), _stream()))


def attention_bf16(q: torch.Tensor, k_layer: torch.Tensor, v_layer: torch.Tensor, T: int,
                   ctx: int, out: torch.Tensor, status: Optional[torch.Tensor] = None) -> None:
    """Tensor-core causal GQA attention: q/out [R][Hq][hd], k/v [rows][Hkv][hd] (bf16)."""
    R, Hq, hd = q.shape
    rows, Hkv, _ = k_layer.shape
    _shape(k_layer, (rows, Hkv, hd), "k_layer")
    _shape(v_layer, (rows, Hkv, hd), "v_layer")
    _shape(out, (R, Hq, hd), "out")
    if status is not None and status.numel() < 1:
        raise KnapSpecError("status must hold one int32")
    _check(load().ks_attention_bf16(_dev(q, torch.bfloat16, "q"), _dev(k_layer, torch.bfloat16, "k"),
                                    _dev(v_layer, torch.bfloat16, "v"), rows, R, T, Hq, Hkv, hd,
                                    ctx, _dev(out, torch.bfloat16, "out"),
                                    _dev(status, torch.int32, "status"), _stream()))


def check_bounded_wait(limit_us: int, status: torch.Tensor,
                       waited_ns: Optional[torch.Tensor] = None) -> None:
    """Run one device wait that nothing completes, bounded to limit_us."""
    _check(load().ks_check_bounded_wait(limit_us, _dev(status, torch.int32, "status"),
                                        _dev(waited_ns, torch.int64, "waited_ns"), _stream()))


def select_step(prev, exec_, target, w: int, cur, val, bp, cos_skip=None, cos_exec=None) -> None:
    C, T, d = prev.shape
    if C > w:
        _rows(exec_, C - w, (T, d), "exec")
    _shape(target, (T, d), "target")
    _shape(cur, (C, T, d), "cur")
    for t, name in ((val, "val"), (bp, "bp"), (cos_skip, "cos_skip"), (cos_exec, "cos_exec")):
        _shape(t, (C,), name)
    _check(load().ks_select_step(_dev(prev, torch.float32, "prev"),
                                 _dev(exec_, torch.float32, "exec"),
                                 _dev(target, torch.float32, "target"), C, T, d, w,
                                 _dev(cur, torch.float32, "cur"), _dev(val, torch.float32, "val"),
                                 _dev(bp, torch.uint8, "bp"),
                                 _dev(cos_skip, torch.float32, "cos_skip"),
                                 _dev(cos_exec, torch.float32, "cos_exec"), _stream()))


def reconstruct(bp: torch.Tensor, w: torch.Tensor, t: torch.Tensor, sets: torch.Tensor,
                used_w: Optional[torch.Tensor], t_draft: Optional[torch.Tensor],
                status: torch.Tensor) -> None:
    n_items, C = bp.shape
    _shape(w, (n_items,), "w")
    _shape(t, (n_items,), "t")
    _shape(sets, (C, (n_items + 63) // 64), "sets")
    _shape(used_w, (C,), "used_w")
    _shape(t_draft, (C,), "t_draft")
    if status.numel() < 1:
        raise KnapSpecError("status must hold one int32")
    _check(load().ks_reconstruct(_dev(bp, torch.uint8, "bp"), _dev(w, torch.int32, "w"),
                                 _dev(t, torch.float64, "t"), n_items, C,
                                 _dev(sets, torch.int64, "sets"),
                                 _dev(used_w, torch.int32, "used_w"),
                                 _dev(t_draft, torch.float64, "t_draft"),
                                 _dev(status, torch.int32, "status"), _stream()))


def tpt_argmax(values: torch.Tensor, t_draft: torch.Tensor, t_target: float, prm: Params,
               tpt: Optional[torch.Tensor], best: torch.Tensor,
               best_tpt: Optional[torch.Tensor]) -> None:
    C = values.numel()
    _shape(t_draft, (C,), "t_draft")
    _shape(tpt, (C, prm.gamma_max), "tpt")
    _shape(best, (2,), "best")
    if best_tpt is not None and best_tpt.numel() < 1:
        raise KnapSpecError("best_tpt must hold one float64")
    _check(load().ks_tpt_argmax(_dev(values, torch.float32, "values"),
                                _dev(t_draft, torch.float64, "t_draft"), values.numel(),
                                t_target, ctypes.byref(prm), _dev(tpt, torch.float64, "tpt"),
                                _dev(best, torch.int32, "best"),
                                _dev(best_tpt, torch.float64, "best_tpt"), _stream()))


def solve_cells(t: Sequence[float], prm: Params, w: Optional[Sequence[int]] = None) -> int:
    n = len(t)
    tt = (ctypes.c_double * n)(*t)
    ww = (ctypes.c_int32 * n)(*w) if w is not None else None
    out = ctypes.c_int32()
    _check(load().ks_solve_cells(n, ww, tt, ctypes.byref(prm), ctypes.byref(out)))
    return out.value


@dataclass
class SolveOutputs:
    status: torch.Tensor
    values: torch.Tensor
    sets: torch.Tensor
    used_w: torch.Tensor
    t_draft: torch.Tensor
    best: torch.Tensor
    best_tpt: torch.Tensor
    bp: Optional[torch.Tensor] = None
    cos_skip: Optional[torch.Tensor] = None
    cos_exec: Optional[torch.Tensor] = None
    tpt: Optional[torch.Tensor] = None
    ref_states: Optional[torch.Tensor] = None
    exec_counts: Optional[torch.Tensor] = None
    final_states: Optional[torch.Tensor] = None
    dedup_rejected: Optional[torch.Tensor] = None


class Solver:
    """Owns the device workspace and result buffers for repeated ks_solve calls."""

    def __init__(self, model: ModelDesc, layers: Sequence[Dict[str, torch.Tensor]],
                 k_cache: torch.Tensor, v_cache: torch.Tensor, ctx: int, T: int,
                 t: Sequence[float], prm: Params, w: Optional[Sequence[int]] = None,
                 keep_bp: bool = True, keep_cos: bool = False, keep_tpt: bool = True,
                 keep_ref: bool = True, keep_final: bool = False, device="cuda",
                 kv: str = "cache"):
        self.model = model
        self.wdtype = torch.float32 if model.wdtype == KS_F32 else torch.bfloat16
        self._layers_keep = layers
        self.layers = layer_array(layers, self.wdtype, model)
        self._cache_keep = (k_cache, v_cache)
        self.cache = cache_desc(k_cache, v_cache, ctx, model, kv=kv)
        self.T = T
        self.t = list(map(float, t))
        self.prm = prm
        self.n_items = 2 * model.n_layers
        if len(self.t) != self.n_items:
            raise KnapSpecError("need one latency per item")
        self.w = list(w) if w is not None else quantize_weights(self.t, prm.n_bins)
        self.C = solve_cells(self.t, prm, self.w)
        self.ws = workspace(model, self.C, T, device)
        self.device = self.ws.device
        C, n, words = self.C, self.n_items, (self.n_items + 63) // 64
        z = lambda *s, dt: torch.zeros(*s, dtype=dt, device=device)
        self.out = SolveOutputs(
            status=z(1, dt=torch.int32), values=z(C, dt=torch.float32),
            sets=z(C, words, dt=torch.int64), used_w=z(C, dt=torch.int32),
            t_draft=z(C, dt=torch.float64), best=z(2, dt=torch.int32),
            best_tpt=z(1, dt=torch.float64),
            bp=z(n, C, dt=torch.uint8) if keep_bp else None,
            cos_skip=z(n, C, dt=torch.float32) if keep_cos else None,
            cos_exec=z(n, C, dt=torch.float32) if keep_cos else None,
            tpt=z(C, prm.gamma_max, dt=torch.float64) if keep_tpt else None,
            ref_states=z(n + 1, T, model.d_model, dt=torch.float32) if keep_ref else None,
            exec_counts=z(n, dt=torch.int32),
            final_states=z(C, T, model.d_model, dt=torch.float32) if keep_final else None,
            dedup_rejected=z(n, dt=torch.int32) if prm.dedup else None)
        o = self.out
        p = lambda x: None if x is None else x.data_ptr()
        self.result = Result(p(o.status), p(o.values), p(o.sets), p(o.used_w), p(o.t_draft),
                             p(o.bp), p(o.cos_skip), p(o.cos_exec), p(o.tpt), p(o.best),
                             p(o.best_tpt), p(o.ref_states), p(o.exec_counts),
                             p(o.final_states), p(o.dedup_rejected))
        self._t_arr = (ctypes.c_double * n)(*self.t)
        self._w_arr = (ctypes.c_int32 * n)(*self.w)

    def solve(self, x0: torch.Tensor, ref: Optional[torch.Tensor] = None) -> SolveOutputs:
        """Enqueue one solve on the current stream of the solver's device (results
        valid after a sync)."""
        _shape(x0, (self.T, self.model.d_model), "x0")
        _shape(ref, (self.n_items + 1, self.T, self.model.d_model), "ref")
        with torch.cuda.device(self.device):
            _check(load().ks_solve(ctypes.byref(self.model), self.layers,
                                   ctypes.byref(self.cache), self.T,
                                   _dev(x0, torch.float32, "x0"),
                                   _dev(ref, torch.float32, "ref"), self._w_arr, self._t_arr,
                                   ctypes.byref(self.prm), _dev(self.ws), self.ws.numel(),
                                   ctypes.byref(self.result), _stream()))
        return self.out

    def check_status(self) -> None:
        s = int(self.out.status.item())
        if s != 0:
            raise KnapSpecError(f"device status {s}: {load().ks_status_string(s).decode()}")


class SolverContexts:
    """The DP of one model at several contexts in one pass (ks_solve_contexts):
    per context a KV cache view and context length, latencies (and optionally
    weights); each context keeps its own result buffers (``outs[j]``, shaped as
    a Solver's)."""

    def __init__(self, model: ModelDesc, layers: Sequence[Dict[str, torch.Tensor]],
                 caches: Sequence[tuple], T: int, ts: Sequence[Sequence[float]], prm: Params,
                 ws: Optional[Sequence[Sequence[int]]] = None, keep_bp: bool = True,
                 keep_cos: bool = False, keep_tpt: bool = True, keep_ref: bool = True,
                 device="cuda", kv: str = "cache"):
        """caches: per context (k_cache, v_cache, ctx)."""
        n = len(caches)
        if not 1 <= n <= 4:
            raise KnapSpecError("1 to 4 contexts")
        if len(ts) != n or (ws is not None and len(ws) != n):
            raise KnapSpecError("one latency list (and weight list) per context")
        self.model = model
        self.wdtype = torch.float32 if model.wdtype == KS_F32 else torch.bfloat16
        self._layers_keep = layers
        self.layers = layer_array(layers, self.wdtype, model)
        self._cache_keep = list(caches)
        self.caches = (CacheDesc * n)(*[cache_desc(k, v, ctx, model, kv=kv) for k, v, ctx in caches])
        self.n_ctx, self.T = n, T
        self.n_items = 2 * model.n_layers
        self.t = [list(map(float, t)) for t in ts]
        for t in self.t:
            if len(t) != self.n_items:
                raise KnapSpecError("need one latency per item")
        self.prm = prm
        self.w = [list(ws[j]) if ws is not None else quantize_weights(self.t[j], prm.n_bins)
                  for j in range(n)]
        self.C = [solve_cells(self.t[j], prm, self.w[j]) for j in range(n)]
        size = ctypes.c_size_t()
        cells = (ctypes.c_int32 * n)(*self.C)
        _check(load().ks_workspace_size_contexts(ctypes.byref(model), n, cells, T,
                                                 ctypes.byref(size)))
        self.ws = torch.empty(size.value, dtype=torch.uint8, device=device)
        self.device = self.ws.device
        words = (self.n_items + 63) // 64
        z = lambda *s, dt: torch.zeros(*s, dtype=dt, device=device)
        self.outs = []
        for C in self.C:
            ni = self.n_items
            self.outs.append(SolveOutputs(
                status=z(1, dt=torch.int32), values=z(C, dt=torch.float32),
                sets=z(C, words, dt=torch.int64), used_w=z(C, dt=torch.int32),
                t_draft=z(C, dt=torch.float64), best=z(2, dt=torch.int32),
                best_tpt=z(1, dt=torch.float64),
                bp=z(ni, C, dt=torch.uint8) if keep_bp else None,
                cos_skip=z(ni, C, dt=torch.float32) if keep_cos else None,
                cos_exec=z(ni, C, dt=torch.float32) if keep_cos else None,
                tpt=z(C, prm.gamma_max, dt=torch.float64) if keep_tpt else None,
                ref_states=z(ni + 1, T, model.d_model, dt=torch.float32) if keep_ref else None,
                exec_counts=z(ni, dt=torch.int32)))
        p = lambda x: None if x is None else x.data_ptr()
        self.results = (Result * n)(*[
            Result(p(o.status), p(o.values), p(o.sets), p(o.used_w), p(o.t_draft), p(o.bp),
                   p(o.cos_skip), p(o.cos_exec), p(o.tpt), p(o.best), p(o.best_tpt),
                   p(o.ref_states), p(o.exec_counts), None, None) for o in self.outs])
        self._t_arrs = [(ctypes.c_double * self.n_items)(*t) for t in self.t]
        self._w_arrs = [(ctypes.c_int32 * self.n_items)(*w) for w in self.w]
        self._t_ptrs = (ctypes.c_void_p * n)(*[ctypes.cast(a, ctypes.c_void_p) for a in self._t_arrs])
        self._w_ptrs = (ctypes.c_void_p * n)(*[ctypes.cast(a, ctypes.c_void_p) for a in self._w_arrs])

    def solve(self, x0s: Sequence[torch.Tensor]) -> List[SolveOutputs]:
        """Enqueue the solve of every context on the current stream (x0s: one
        [T][d] fp32 tensor per context)."""
        if len(x0s) != self.n_ctx:
            raise KnapSpecError("one x0 per context")
        for x in x0s:
            _shape(x, (self.T, self.model.d_model), "x0")
        ptrs = (ctypes.c_void_p * self.n_ctx)(*[_dev(x, torch.float32, "x0") for x in x0s])
        with torch.cuda.device(self.device):
            _check(load().ks_solve_contexts(ctypes.byref(self.model), self.layers, self.n_ctx,
                                            self.caches, self.T, ptrs, self._w_ptrs, self._t_ptrs,
                                            ctypes.byref(self.prm), _dev(self.ws), self.ws.numel(),
                                            self.results, _stream()))
        return self.outs

    def check_status(self) -> None:
        for j, o in enumerate(self.outs):
            s = int(o.status.item())
            if s != 0:
                raise KnapSpecError(f"context {j}: device status {s}: "
                                    f"{load().ks_status_string(s).decode()}")


def profile_start(timing: bool = True) -> None:
    """Reset the library's launch accounting; with timing, record event pairs."""
    _check(load().ks_profile_start(1 if timing else 0))


def profile_stop() -> List[dict]:
    """Per kernel kind: launches, event time (ms), algorithmic FLOPs and bytes."""
    arr = (KernelStat * 64)()
    n = ctypes.c_int32()
    _check(load().ks_profile_stop(arr, 64, ctypes.byref(n)))
    return [{"name": arr[i].name.decode(), "launches": arr[i].launches,
             "total_ms": arr[i].total_ms, "flops": arr[i].flops, "bytes": arr[i].bytes}
            for i in range(min(n.value, 64))]


class LemmaResult(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("istar", "margin", "dist", "cos", "bound", "agree", "counts")]


def lemma_check(states: torch.Tensor, ref: torch.Tensor, lm_head: torch.Tensor,
                final_norm: Optional[torch.Tensor] = None, eps: float = 1e-6,
                status: Optional[torch.Tensor] = None) -> dict:
    """Lemma 4.1 checker on N states [N][T][d] against ref [T][d] (see knapspec.h)."""
    N, T, d = states.shape
    V = lm_head.shape[0]
    _shape(ref, (T, d), "ref")
    _shape(lm_head, (V, d), "lm_head")
    _shape(final_norm, (d,), "final_norm")
    if status is not None and status.numel() < 1:
        raise KnapSpecError("status must hold one int32")
    size = ctypes.c_size_t()
    _check(load().ks_lemma_workspace_size(N, T, d, V, ctypes.byref(size)))
    ws = torch.empty(size.value, dtype=torch.uint8, device=states.device)
    dev = states.device
    out = {"istar": torch.empty(T, dtype=torch.int32, device=dev),
           "margin": torch.empty(T, dtype=torch.float32, device=dev),
           "dist": torch.empty(T, dtype=torch.float32, device=dev),
           "cos": torch.empty(N, T, dtype=torch.float32, device=dev),
           "bound": torch.empty(N, T, dtype=torch.uint8, device=dev),
           "agree": torch.empty(N, T, dtype=torch.uint8, device=dev),
           "counts": torch.empty(3, dtype=torch.int32, device=dev)}
    res = LemmaResult(*[out[k].data_ptr() for k in
                        ("istar", "margin", "dist", "cos", "bound", "agree", "counts")])
    _check(load().ks_lemma_check(_dev(states, torch.float32, "states"), N,
                                 _dev(ref, torch.float32, "ref"), T, d,
                                 _dev(final_norm, torch.bfloat16, "final_norm"), eps,
                                 _dev(lm_head, torch.bfloat16, "lm_head"), V, ws.data_ptr(),
                                 ws.numel(), ctypes.byref(res), _dev(status, torch.int32, "status"),
                                 _stream()))
    out["_ws"] = ws
    return out


def sets_to_lists(sets: torch.Tensor, n_items: int) -> List[List[int]]:
    """Decode the [C][words] bitmask tensor into sorted item lists (host)."""
    s = sets.cpu().numpy().view("uint64")
    out = []
    for row in s:
        items = [k for k in range(n_items) if (int(row[k >> 6]) >> (k & 63)) & 1]
        out.append(items)
    return out
