"""Synthetic KnapSpec workloads: configuration records and seeded input draws.

This module only describes shapes and draws seeded random numbers.  It holds no
arithmetic of the method (no norm, attention, MLP, cosine, quantisation, DP or
TPT); both the CUDA library's callers and the CPU oracle's callers take their
inputs from here, and nothing else is shared between the two sides.

Workloads follow the KnapSpec setting (arXiv 2602.20217, "KnapSpec:
Self-Speculative Decoding via Adaptive Layer Selection as a Knapsack Problem",
§3.1/§3.3 on the Pith review page): every Attention and every MLP sublayer of a
decoder is one knapsack item, Attention latency grows linearly with context and
MLP latency is flat.  The trained Qwen3/Llama3 weights and the benchmark texts
the paper uses are not available, so every tensor here is drawn at random:

* linear weights ~ N(0, 0.02^2), stored as ``[out_features][in_features]``
  (bf16, or fp32 for the tiny model); RMSNorm gains are ones;
* the key/value cache ~ N(0, (0.02*sqrt(d_model))^2) per entry -- the per-entry
  spread that projecting a unit-RMS hidden state through N(0, 0.02^2) weights
  gives -- laid out ``[layer][position][kv_head][head_dim]``;
* the T evaluation tokens' input hidden states x0 ~ N(0, 1), ``[T][d_model]`` fp32.

Draw order (one ``torch.Generator`` seeded with ``seed`` on ``device``): for each
layer in order Wq, Wo, W_gate, W_up, W_down; then the K cache, the V cache, then
x0.  Each tensor is drawn in fp32 and then rounded to the storage dtype.  Every
workload is drawn on the CPU generator, so that a machine without a GPU can
reproduce the inputs exactly; ``input_digest`` fingerprints a draw so that two
machines can confirm they hold the same values, and ``StreamedInputs`` holds
only one layer at a time of a model too large for host memory (the 64 GB
Qwen3-32B shape).
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Dict, List, Optional, Sequence

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decoder + DP problem."""

    name: str
    n_layers: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    rms_eps: float
    rope_base: float
    ctx: int                 # context tokens already in the cache
    T: int                   # evaluation tokens (the DP's r / m window)
    wdtype: str              # "f32" or "bf16" (weights and KV cache)
    n_bins: int              # budget-grid bins used by the latency quantiser
    gamma_max: int           # largest draft length in the TPT grid search
    gen_device: str          # device whose RNG defines the values ("cpu"/"cuda")
    contexts: Sequence[int] = ()   # extra contexts a re-solve sweep visits
    attn_latency: str = "1+ctx/256"  # latency model (stated by the workload)
    mlp_latency: float = 4.0

    @property
    def n_items(self) -> int:
        return 2 * self.n_layers

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def n_positions(self) -> int:
        return self.ctx + self.T

    def with_ctx(self, ctx: int) -> "Workload":
        return dataclasses.replace(self, ctx=ctx)

    def latencies(self, ctx: Optional[int] = None) -> List[float]:
        """Raw per-item latencies t_i (item 2l = Attn of layer l, 2l+1 = MLP).

        These are the workload's stated latency model (synthetic stand-ins for
        the paper's pre-profiled hardware latencies): an Attention sublayer costs
        an affine function of the context length, an MLP sublayer a constant.
        """
        c = self.ctx if ctx is None else ctx
        if self.attn_latency == "2+ceil(ctx/64)":
            ta = 2.0 + float(-(-c // 64))
        elif self.attn_latency == "1+ctx/256":
            ta = 1.0 + c / 256.0
        else:
            raise ValueError(self.attn_latency)
        out: List[float] = []
        for _ in range(self.n_layers):
            out += [ta, float(self.mlp_latency)]
        return out


WORKLOADS: Dict[str, Workload] = {
    # Tiny Llama-style decoder, fp32: small enough for exhaustive subset search.
    "tiny": Workload("tiny", n_layers=4, d_model=256, n_q_heads=4, n_kv_heads=4,
                     head_dim=64, ffn=688, rms_eps=1e-6, rope_base=1e4, ctx=128, T=4,
                     wdtype="f32", n_bins=28, gamma_max=8, gen_device="cpu",
                     attn_latency="2+ceil(ctx/64)", mlp_latency=3.0),
    # Small GQA decoder, bf16.
    "small": Workload("small", n_layers=16, d_model=1024, n_q_heads=16, n_kv_heads=4,
                      head_dim=64, ffn=2816, rms_eps=1e-6, rope_base=1e4, ctx=2048, T=8,
                      wdtype="bf16", n_bins=256, gamma_max=8, gen_device="cpu"),
    # Llama-3-8B shape at 8k context.
    "llama3_8b_8k": Workload("llama3_8b_8k", n_layers=32, d_model=4096, n_q_heads=32,
                             n_kv_heads=8, head_dim=128, ffn=14336, rms_eps=1e-6,
                             rope_base=5e5, ctx=8192, T=16, wdtype="bf16", n_bins=512,
                             gamma_max=10, gen_device="cpu"),
    # Llama-3-8B shape, long context, re-solved at 4k / 16k / 32k.
    "llama3_8b_32k": Workload("llama3_8b_32k", n_layers=32, d_model=4096, n_q_heads=32,
                              n_kv_heads=8, head_dim=128, ffn=14336, rms_eps=1e-6,
                              rope_base=5e5, ctx=32768, T=16, wdtype="bf16", n_bins=1024,
                              gamma_max=10, gen_device="cpu",
                              contexts=(4096, 16384, 32768)),
    # Qwen3-32B shape at 16k context (q-dim 8192 differs from d_model 5120).
    "qwen3_32b_16k": Workload("qwen3_32b_16k", n_layers=64, d_model=5120, n_q_heads=64,
                              n_kv_heads=8, head_dim=128, ffn=25600, rms_eps=1e-6,
                              rope_base=1e6, ctx=16384, T=8, wdtype="bf16", n_bins=1024,
                              gamma_max=10, gen_device="cpu"),
}

# Order of the five workloads as the build's configuration list names them.
WORKLOAD_ORDER = ["tiny", "small", "llama3_8b_8k", "llama3_8b_32k", "qwen3_32b_16k"]

LINEAR_STD = 0.02


def kv_std(wl: Workload) -> float:
    """Per-entry standard deviation of the synthetic K/V cache."""
    return LINEAR_STD * math.sqrt(wl.d_model)


def torch_dtype(wl: Workload) -> torch.dtype:
    return torch.float32 if wl.wdtype == "f32" else torch.bfloat16


@dataclasses.dataclass
class Inputs:
    """Seeded inputs of one workload, all on one device."""

    wl: Workload
    layers: List[Dict[str, torch.Tensor]]   # per layer: attn_norm, wq, wo, mlp_norm, w_gate, w_up, w_down
    k_cache: torch.Tensor                    # [L][ctx+T][Hkv][hd]
    v_cache: torch.Tensor                    # [L][ctx+T][Hkv][hd]
    x0: torch.Tensor                         # [T][d] fp32

    def first_layers(self, n: int) -> "Inputs":
        """The sub-problem made of the first ``n`` layers (same cache rows and x0)."""
        return Inputs(dataclasses.replace(self.wl, n_layers=n), self.layers[:n],
                      self.k_cache[:n], self.v_cache[:n], self.x0)

    def to(self, device) -> "Inputs":
        mv = lambda t: t.to(device)
        return Inputs(self.wl, [{k: mv(v) for k, v in l.items()} for l in self.layers],
                      mv(self.k_cache), mv(self.v_cache), mv(self.x0))


def _randn(shape, std, dtype, gen, device):
    t = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


LAYER_KEYS = ("wq", "wo", "w_gate", "w_up", "w_down", "attn_norm", "mlp_norm")


def _draw_layer(wl: Workload, gen, dev) -> Dict[str, torch.Tensor]:
    """One layer's weights, drawn in the stated order."""
    dt = torch_dtype(wl)
    d, qd, F = wl.d_model, wl.q_dim, wl.ffn
    layer = {
        "wq": _randn((qd, d), LINEAR_STD, dt, gen, dev),
        "wo": _randn((d, qd), LINEAR_STD, dt, gen, dev),
        "w_gate": _randn((F, d), LINEAR_STD, dt, gen, dev),
        "w_up": _randn((F, d), LINEAR_STD, dt, gen, dev),
        "w_down": _randn((d, F), LINEAR_STD, dt, gen, dev),
    }
    layer["attn_norm"] = torch.ones(d, dtype=dt, device=dev)
    layer["mlp_norm"] = torch.ones(d, dtype=dt, device=dev)
    return layer


def _draw_tail(wl: Workload, gen, dev):
    """The K cache, the V cache and x0, drawn after every layer."""
    dt = torch_dtype(wl)
    kvshape = (wl.n_layers, wl.n_positions, wl.n_kv_heads, wl.head_dim)
    k_cache = _randn(kvshape, kv_std(wl), dt, gen, dev)
    v_cache = _randn(kvshape, kv_std(wl), dt, gen, dev)
    x0 = _randn((wl.T, wl.d_model), 1.0, torch.float32, gen, dev)
    return k_cache, v_cache, x0


def make_inputs(wl: Workload, seed: int = 0, device: Optional[str] = None) -> Inputs:
    """Draw the workload's inputs (see the module docstring for the recipe)."""
    dev = device or wl.gen_device
    if dev == "cuda" and not torch.cuda.is_available():
        raise RuntimeError(f"workload {wl.name} is drawn on CUDA, which is not available")
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    layers = [_draw_layer(wl, gen, dev) for _ in range(wl.n_layers)]
    k_cache, v_cache, x0 = _draw_tail(wl, gen, dev)
    return Inputs(wl, layers, k_cache, v_cache, x0)


class StreamedInputs:
    """The CPU-generator inputs of a workload too large to hold at once.

    The draw runs once in the stated order, keeping only the K/V cache and x0
    and recording the generator's state at the start of every layer; a layer's
    weights are drawn again from that state when asked for (``layers[l]``), so
    they equal make_inputs(wl, seed, "cpu")'s.  ``digest`` equals input_digest
    of that full draw, computed on the way.  ``to(device)`` places the whole
    set on a device one layer at a time; with ``device`` given, each layer is
    copied there as it is drawn, and ``to(device)`` then draws nothing again."""

    def __init__(self, wl: Workload, seed: int = 0, device: Optional[str] = None):
        gen = torch.Generator(device="cpu")
        gen.manual_seed(seed)
        h = hashlib.sha256()
        self.wl = wl
        self._states = []
        self._device = device
        self._dev_layers = []
        for _ in range(wl.n_layers):
            self._states.append(gen.get_state())
            layer = _draw_layer(wl, gen, "cpu")
            for k in LAYER_KEYS:
                _hash_update(h, layer[k])
            if device is not None:
                self._dev_layers.append({k: v.to(device) for k, v in layer.items()})
            del layer
        self.k_cache, self.v_cache, self.x0 = _draw_tail(wl, gen, "cpu")
        for l in range(wl.n_layers):
            _hash_update(h, self.k_cache[l])
        for l in range(wl.n_layers):
            _hash_update(h, self.v_cache[l])
        _hash_update(h, self.x0)
        self.digest = h.hexdigest()
        self.layers = _StreamedLayers(self)

    def layer(self, l: int) -> Dict[str, torch.Tensor]:
        gen = torch.Generator(device="cpu")
        gen.set_state(self._states[l])
        return _draw_layer(self.wl, gen, "cpu")

    def to(self, device) -> Inputs:
        if self._device is not None and torch.device(device) == torch.device(self._device):
            layers = self._dev_layers
        else:
            layers = [{k: v.to(device) for k, v in self.layer(l).items()}
                      for l in range(self.wl.n_layers)]
        return Inputs(self.wl, layers, self.k_cache.to(device), self.v_cache.to(device),
                      self.x0.to(device))


class _StreamedLayers:
    def __init__(self, src: StreamedInputs):
        self._src = src

    def __len__(self):
        return self._src.wl.n_layers

    def __getitem__(self, l):
        return self._src.layer(l)


def window_weights(wl: Workload, seed: int = 2, device: Optional[str] = None
                   ) -> List[Dict[str, torch.Tensor]]:
    """Per layer the key/value projections Wk, Wv [Hkv*hd][d] ~ N(0, 0.02^2) in the
    workload's weight dtype, from their own generator and seed (drawn in layer
    order, Wk then Wv), so the main draw order above is unchanged.  Only the
    attention reading that recomputes the window's keys/values uses them."""
    dev = device or wl.gen_device
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    dt = torch_dtype(wl)
    kvd = wl.n_kv_heads * wl.head_dim
    return [{"wk": _randn((kvd, wl.d_model), LINEAR_STD, dt, gen, dev),
             "wv": _randn((kvd, wl.d_model), LINEAR_STD, dt, gen, dev)}
            for _ in range(wl.n_layers)]


def sequence_embeddings(wl: Workload, seed: int = 3, device: Optional[str] = None) -> torch.Tensor:
    """N(0, 1) input embeddings [ctx + T][d] fp32 of a whole token sequence, from
    their own generator and seed: the input of a full-model prefill, whose last T
    rows are then the evaluation tokens' x0."""
    dev = device or wl.gen_device
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    return _randn((wl.n_positions, wl.d_model), 1.0, torch.float32, gen, dev)


def truncated(wl: Workload, n_layers: int, ctx: Optional[int] = None) -> Workload:
    """The same workload shape with fewer layers (and optionally another context)."""
    return dataclasses.replace(wl, n_layers=n_layers, ctx=wl.ctx if ctx is None else ctx)


# Vocabulary sizes of the synthetic LM heads used by the Lemma 4.1 checker
# (the 8B and 32B shapes use Llama-3's and a 256-aligned Qwen3-like size).
VOCAB = {"tiny": 1024, "small": 8192, "llama3_8b_8k": 128256, "llama3_8b_32k": 128256,
         "qwen3_32b_16k": 151808}


def lm_head(wl: Workload, seed: int = 1, device: Optional[str] = None,
            vocab: Optional[int] = None) -> torch.Tensor:
    """A random LM head W [V][d] ~ N(0, 0.02^2) in bf16 (its own generator and seed)."""
    dev = device or wl.gen_device
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    V = vocab or VOCAB[wl.name]
    return _randn((V, wl.d_model), LINEAR_STD, torch.bfloat16, gen, dev)


def random_states(shape: Sequence[int], seed: int, device: str = "cpu",
                  dtype: torch.dtype = torch.float32) -> torch.Tensor:
    """N(0,1) tensor of the given shape (for kernel-level tests of one step)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32).to(dtype)


def _hash_update(h, t: torch.Tensor) -> None:
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        t = t.view(torch.int16)
    h.update(t.numpy().tobytes())


def window_digest(ww: Sequence[Dict[str, torch.Tensor]]) -> str:
    """SHA-256 of window_weights' tensors in draw order (per layer Wk then Wv)."""
    h = hashlib.sha256()
    for layer in ww:
        _hash_update(h, layer["wk"])
        _hash_update(h, layer["wv"])
    return h.hexdigest()


def input_digest(inp: Inputs) -> str:
    """SHA-256 of every input tensor's bytes, in draw order (weights layer by layer,
    then the K cache, the V cache and x0).  Two draws hold the same values iff
    their digests agree (up to hash collisions)."""
    h = hashlib.sha256()
    for layer in inp.layers:
        for k in LAYER_KEYS:
            _hash_update(h, layer[k])
    for l in range(inp.k_cache.shape[0]):
        _hash_update(h, inp.k_cache[l])
    for l in range(inp.v_cache.shape[0]):
        _hash_update(h, inp.v_cache[l])
    _hash_update(h, inp.x0)
    return h.hexdigest()
