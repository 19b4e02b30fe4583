"""Seeded synthetic inputs for attention-map reuse (sender Q/K, receiver V, head map W, logit biases).

This module only draws and rounds random inputs. It holds none of the method's arithmetic
(no logits, softmax, masses, selection or retrieval), so the CUDA path and the fp64 oracle can
both be fed from it without sharing any computation.

Workload shapes follow the settings the MapFlow page describes (sender model prefills a shared
context, a receiver with a different head count reuses the sender's maps: "Accelerating
Cross-Model LLM Inference via Attention Map Reuse", sections 4 and 5).  The structured logit
biases stand in for the attention sinks, local windows and retrieval heads that the AttnCache
page lists as the recurring patterns of real maps ("AttnCache Guide", section "The Attention Map
Redundancy Discovery"); no dataset or trained weight is used anywhere.

Recipe (all draws from ``numpy.random.default_rng(seed)``, float32, in this order):
  per layer -> per sender head (Q then K) -> bias draws -> per receiver head V -> W logits.
bf16 workloads round every Q/K/V value to bf16 with round-to-nearest-even; the float32 arrays
returned here hold exactly the bf16 values, and ``to_bf16_bits`` gives the 16-bit patterns.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import List, Optional

import numpy as np

NEG_INF = float("-inf")


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32 holding bf16 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32)
    rounded = (bits + np.uint32(0x7FFF) + ((bits >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return rounded.view(np.float32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-representable."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


@dataclass
class Bias:
    """Structured causal logit bias for one layer (all values are inputs, not computed).

    b(h, i, j) for a causal pair j <= i is the MAXIMUM of the biases that apply to it, or 0 when
    none applies:
      * ``sink_bias``   applies when j < sink_len;
      * ``window_bias`` applies when i - window < j (a local window of ``window`` keys ending at i);
      * ``kb_bias[h, j // kb_block]`` applies when that entry is finite (-inf marks "no bias").
    ``kb_bias`` rows are per sender head; a layer whose key-block bias is shared by all heads
    simply repeats the row.
    """
    sink_len: int = 0
    sink_bias: float = 0.0
    window: int = 0
    window_bias: float = 0.0
    kb_bias: Optional[np.ndarray] = None  # float32 [H][n_kb], -inf = none
    kb_block: int = 0

    def for_heads(self, heads: np.ndarray) -> "Bias":
        kb = None if self.kb_bias is None else np.ascontiguousarray(self.kb_bias[heads])
        return replace(self, kb_bias=kb)


@dataclass
class Spec:
    """Shape and distribution of one workload."""
    name: str
    H_s: int
    H_r: int
    L: int
    d: int
    d_v: int
    block: int
    p: float
    dtype: str  # "bf16" or "f32"
    n_layers: int = 1
    qk_std: float = 1.0
    sink_len: int = 0
    sink_bias: float = 0.0
    window: int = 0
    window_bias: float = 0.0
    kb_per_head: int = 0          # distinct random key-blocks per sender head with bias kb_value
    kb_value: float = 0.0
    kb_per_layer: int = 0         # distinct random key-blocks per layer, shared by heads, bias ~U(0, kb_max)
    kb_max: float = 0.0
    w_kind: str = "softmax"       # "softmax" or "diag" (softmax of N(0,1) + diag_boost on s = r mod H_s)
    diag_boost: float = 0.0
    seed: int = 0
    # multi-request batch (shared prefix of length L, ragged suffixes)
    n_req: int = 0
    suffix_min: int = 0
    suffix_max: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def n_blocks(self) -> int:
        return self.L // self.block


def config(n: int) -> Spec:
    """The five benchmark workloads at full size."""
    if n == 1:
        return Spec("toy_L512_d64_f32", H_s=4, H_r=4, L=512, d=64, d_v=64, block=64, p=0.95,
                    dtype="f32", qk_std=1.0, sink_len=16, sink_bias=4.0, window=128,
                    window_bias=4.0, seed=1000)
    if n == 2:
        return Spec("L4096_32to40_d128_bf16", H_s=32, H_r=40, L=4096, d=128, d_v=128, block=64,
                    p=0.9, dtype="bf16", qk_std=4.0 / math.sqrt(128), sink_len=16, sink_bias=3.0,
                    window=128, window_bias=3.0, seed=2000)
    if n == 3:
        return Spec("L8192_28layers_32to28_d128_bf16", H_s=32, H_r=28, L=8192, d=128, d_v=128,
                    block=64, p=0.9, dtype="bf16", n_layers=28, qk_std=4.0 / math.sqrt(128),
                    kb_per_layer=8, kb_max=4.0, w_kind="diag", diag_boost=3.0, seed=3000)
    if n == 4:
        return Spec("L32768_32to64_d128_bf16_B128", H_s=32, H_r=64, L=32768, d=128, d_v=128,
                    block=128, p=0.9, dtype="bf16", qk_std=4.0 / math.sqrt(128), sink_len=16,
                    sink_bias=3.0, window=128, window_bias=3.0, kb_per_head=32, kb_value=2.0,
                    seed=4000)
    if n == 5:
        return Spec("prefix4096_16req_suffix512to2048_32to32_d128_bf16", H_s=32, H_r=32, L=4096,
                    d=128, d_v=128, block=64, p=0.9, dtype="bf16", qk_std=4.0 / math.sqrt(128),
                    sink_len=16, sink_bias=3.0, window=128, window_bias=3.0, seed=5000,
                    n_req=16, suffix_min=512, suffix_max=2048)
    raise ValueError(f"no workload {n}")


def shrink(spec: Spec, **kw) -> Spec:
    """Same distributions, smaller shapes (for parity cases the oracle finishes in seconds)."""
    s = replace(spec, **kw)
    if s.L % s.block:
        raise ValueError("L must be a multiple of the block size")
    return s


def _normal(rng, shape, std, dtype):
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return round_to_bf16(x) if dtype == "bf16" else x


def _row_softmax(logits: np.ndarray) -> np.ndarray:
    # W rows on the simplex (an input distribution, drawn once per layer)
    z = logits.astype(np.float64)
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    return (e / e.sum(axis=1, keepdims=True)).astype(np.float32)


def _bias(spec: Spec, rng, H: int, n_kb: int) -> Bias:
    kb = None
    if spec.kb_per_head > 0:
        kb = np.full((H, n_kb), NEG_INF, dtype=np.float32)
        for h in range(H):
            idx = rng.choice(n_kb, size=min(spec.kb_per_head, n_kb), replace=False)
            kb[h, idx] = np.float32(spec.kb_value)
    elif spec.kb_per_layer > 0:
        row = np.full((n_kb,), NEG_INF, dtype=np.float32)
        idx = rng.choice(n_kb, size=min(spec.kb_per_layer, n_kb), replace=False)
        row[idx] = rng.uniform(0.0, spec.kb_max, size=idx.shape[0]).astype(np.float32)
        kb = np.repeat(row[None, :], H, axis=0)
    return Bias(sink_len=spec.sink_len, sink_bias=spec.sink_bias, window=spec.window,
                window_bias=spec.window_bias, kb_bias=kb, kb_block=spec.block if kb is not None else 0)


def _W(spec: Spec, rng) -> np.ndarray:
    logits = rng.standard_normal((spec.H_r, spec.H_s), dtype=np.float32)
    if spec.w_kind == "diag":
        for r in range(spec.H_r):
            logits[r, r % spec.H_s] += np.float32(spec.diag_boost)
    return _row_softmax(logits)


@dataclass
class Layer:
    Q: np.ndarray          # [H_s][L][d]   sender queries (float32 holding dtype-rounded values)
    K: np.ndarray          # [H_s][L][d]   sender keys
    V: np.ndarray          # [H_r][L][d_v] receiver values
    W: np.ndarray          # [H_r][H_s]    head map, rows on the simplex
    bias: Bias


def iter_layers(spec: Spec):
    """Yield every layer of the workload in order, drawn from one stream (the same values as
    draw_layers), so a caller can move each layer to the device before the next is drawn."""
    rng = np.random.default_rng(spec.seed)
    n_kb = spec.L // spec.block
    for _ in range(spec.n_layers):
        Q = np.empty((spec.H_s, spec.L, spec.d), np.float32)
        K = np.empty_like(Q)
        for h in range(spec.H_s):
            Q[h] = _normal(rng, (spec.L, spec.d), spec.qk_std, spec.dtype)
            K[h] = _normal(rng, (spec.L, spec.d), spec.qk_std, spec.dtype)
        bias = _bias(spec, rng, spec.H_s, n_kb)
        V = np.empty((spec.H_r, spec.L, spec.d_v), np.float32)
        for r in range(spec.H_r):
            V[r] = _normal(rng, (spec.L, spec.d_v), 1.0, spec.dtype)
        W = _W(spec, rng)
        yield Layer(Q=Q, K=K, V=V, W=W, bias=bias)


def draw_layers(spec: Spec, layers: Optional[List[int]] = None) -> List[Layer]:
    """Draw the requested layers (all by default), consuming the stream in layer order."""
    want = set(range(spec.n_layers) if layers is None else layers)
    out: List[Layer] = []
    for layer, lay in enumerate(iter_layers(spec)):
        if layer in want:
            out.append(lay)
        if layer >= max(want):
            break
    return out


@dataclass
class Request:
    Q: np.ndarray   # [H_r][P + s][d]   receiver queries over prefix + suffix
    K: np.ndarray   # [H_r][P + s][d]
    V: np.ndarray   # [H_r][P + s][d_v]
    suffix: int


@dataclass
class Batch:
    Qs: np.ndarray          # [H_s][P][d] sender prefix queries
    Ks: np.ndarray          # [H_s][P][d] sender prefix keys
    W: np.ndarray           # [H_r][H_s]
    bias: Bias              # over the prefix key blocks (sender heads)
    requests: List[Request] = field(default_factory=list)


def draw_batch(spec: Spec) -> Batch:
    """Multi-request batch: one shared prefix of length ``spec.L`` and ``spec.n_req`` ragged suffixes."""
    rng = np.random.default_rng(spec.seed)
    P = spec.L
    suffix = rng.integers(spec.suffix_min, spec.suffix_max + 1, size=spec.n_req)
    Qs = np.empty((spec.H_s, P, spec.d), np.float32)
    Ks = np.empty_like(Qs)
    for h in range(spec.H_s):
        Qs[h] = _normal(rng, (P, spec.d), spec.qk_std, spec.dtype)
        Ks[h] = _normal(rng, (P, spec.d), spec.qk_std, spec.dtype)
    bias = _bias(spec, rng, spec.H_s, P // spec.block)
    reqs = []
    for s in suffix:
        n = P + int(s)
        Q = np.empty((spec.H_r, n, spec.d), np.float32)
        K = np.empty_like(Q)
        V = np.empty((spec.H_r, n, spec.d_v), np.float32)
        for r in range(spec.H_r):
            Q[r] = _normal(rng, (n, spec.d), spec.qk_std, spec.dtype)
            K[r] = _normal(rng, (n, spec.d), spec.qk_std, spec.dtype)
            V[r] = _normal(rng, (n, spec.d_v), 1.0, spec.dtype)
        reqs.append(Request(Q=Q, K=K, V=V, suffix=int(s)))
    W = _W(spec, rng)
    return Batch(Qs=Qs, Ks=Ks, W=W, bias=bias, requests=reqs)
