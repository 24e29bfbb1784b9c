"""Seeded synthetic inputs for the ViT encoder hot path.

This module is shared by the fp64 oracle (``oracle/``) and by the GPU path's
tests and benchmark.  It holds shapes, seeds, the random draw order and the
storage rounding of the inputs, and nothing of the method's arithmetic: no
normalisation, contraction, rotation, softmax or merge is computed here.

Workloads (KLiteInfer README, sections "精度与性能" and "架构": the SigLIP encoder
of PaddleOCR-VL run over batched patch tokens; shapes are the five workloads
this library is measured on):

* ``c0``  1 layer, hidden 256, 4 x 64 heads, MLP 1024, 16x16 grid, fp32.
* ``c1``  1 layer, hidden 1152, 16 x 72 heads, MLP 4304, 30x32 grid, bf16.
* ``c2``  27 layers of the c1 layer over 3900 patches, then the 2x2 merge
          to 975 x 4608.  The stated 60x65 grid has an odd width, which no
          2x2 merge can consume; the merge workload therefore runs on a
          50x78 grid (also 3900 tokens, merging to exactly 975 tokens).
          ``c2_60x65`` keeps the literal grid for the encoder alone.
* ``c3``  27 layers over 5 packed images (780+888+960+3900+4408 tokens).
* ``c4``  attention half-layer of a DiT block: 2 x 4096 tokens (64x64),
          hidden 3072, 24 x 128 heads, each sequence with its own 1024-token
          prefix K/V in layout [2, P, kv_heads, d].

Draw order (one ``numpy.random.Generator(PCG64(seed))`` per workload, all
``standard_normal`` in fp64): x; then per layer ln1_g, ln1_b, w_qkv, b_qkv,
w_o, b_o, ln2_g, ln2_b, w_fc1, b_fc1, w_fc2, b_fc2; then prefix_kv.
Scales: x, prefix ~ N(0,1); weights ~ N(0,0.02); biases ~ N(0,0.01);
LayerNorm gamma = 1 + N(0,0.02), beta ~ N(0,0.01).

Storage rounding: fp64 -> fp32 (round to nearest even) and, for bf16
workloads, fp32 -> bf16 (round to nearest even).  bf16 tensors are carried as
``uint16`` bit patterns; ``to_f64`` widens them exactly.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "get", "make_inputs", "make_layer_weights",
    "round_bf16_bits", "bf16_bits_to_f64", "to_f64", "from_f64",
    "grid_tokens", "LAYER_KEYS", "make_projector_weights",
]

LAYER_KEYS = ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o",
              "ln2_g", "ln2_b", "w_fc1", "b_fc1", "w_fc2", "b_fc2")


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    dtype: str                      # "f32" or "bf16"
    hidden: int
    heads: int
    head_dim: int
    mlp: int
    layers: int
    grids: Tuple[Tuple[int, int], ...]   # (rows, cols) per image
    merge: bool = False
    prefix_len: int = 0             # prefix K/V tokens per sequence (0: none)
    kv_heads: int = 0               # heads of the prefix K/V (0: = heads)
    attn_only: bool = False         # attention half-layer (no MLP)
    ln_eps: float = 1e-6
    rope_theta: float = 10000.0
    rope: bool = True

    @property
    def tokens(self) -> int:
        return grid_tokens(self.grids)

    @property
    def n_seqs(self) -> int:
        return len(self.grids)

    @property
    def prefix_heads(self) -> int:
        return self.kv_heads if self.kv_heads else self.heads

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)

    def flops(self) -> Dict[str, float]:
        """Algorithmic FLOP count at 2 FLOP per multiply-add (head_dim as
        stated, no padding)."""
        T, C, F = self.tokens, self.hidden, self.mlp
        gemm = 2.0 * T * C * 3 * C + 2.0 * T * C * C
        if not self.attn_only:
            gemm += 2.0 * 2 * T * C * F
        attn = 0.0
        for (h, w) in self.grids:
            n = h * w
            attn += 4.0 * n * (n + self.prefix_len) * C
        return {"gemm": gemm * self.layers, "attn": attn * self.layers,
                "total": (gemm + attn) * self.layers}


def grid_tokens(grids) -> int:
    return int(sum(int(h) * int(w) for (h, w) in grids))


WORKLOADS: Dict[str, Workload] = {
    "c0": Workload("c0", 0, "f32", 256, 4, 64, 1024, 1, ((16, 16),), merge=True),
    "c1": Workload("c1", 1, "bf16", 1152, 16, 72, 4304, 1, ((30, 32),)),
    "c2": Workload("c2", 2, "bf16", 1152, 16, 72, 4304, 27, ((50, 78),), merge=True),
    "c2_60x65": Workload("c2_60x65", 2, "bf16", 1152, 16, 72, 4304, 27, ((60, 65),)),
    "c3": Workload("c3", 3, "bf16", 1152, 16, 72, 4304, 27,
                   ((26, 30), (24, 37), (30, 32), (60, 65), (76, 58))),
    "c4": Workload("c4", 4, "bf16", 3072, 24, 128, 0, 1, ((64, 64), (64, 64)),
                   prefix_len=1024, kv_heads=24, attn_only=True),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


# ---------------------------------------------------------------- rounding
def round_bf16_bits(a) -> np.ndarray:
    """fp64/fp32 values -> bf16 bit patterns (uint16), via fp32, both steps
    round-to-nearest-even.  Finite inputs only."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def from_f64(a, dtype: str) -> np.ndarray:
    """Quantise fp64 values to the storage type of a workload."""
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32)
    if dtype == "bf16":
        return round_bf16_bits(a)
    raise ValueError(dtype)


def to_f64(a, dtype: str) -> np.ndarray:
    """Exact widening of stored values to fp64."""
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        return bf16_bits_to_f64(a)
    raise ValueError(dtype)


# ---------------------------------------------------------------- draws
def _layer_shapes(wl: Workload):
    C, F = wl.hidden, wl.mlp
    shapes = {
        "ln1_g": (C,), "ln1_b": (C,),
        "w_qkv": (3 * C, C), "b_qkv": (3 * C,),
        "w_o": (C, C), "b_o": (C,),
        "ln2_g": (C,), "ln2_b": (C,),
        "w_fc1": (F, C), "b_fc1": (F,),
        "w_fc2": (C, F), "b_fc2": (C,),
    }
    return shapes


def _layer_scale(key: str):
    if key.startswith("w_"):
        return 0.0, 0.02
    if key.startswith("b_") or key.endswith("_b"):
        return 0.0, 0.01
    return 1.0, 0.02      # LayerNorm gamma


def make_layer_weights(wl: Workload, rng: np.random.Generator) -> Dict[str, np.ndarray]:
    """Draws one layer's parameters in the fixed key order.  Attention-only
    workloads draw zero-sized MLP / LN2 tensors so the draw order is the same
    rule for every workload."""
    out = {}
    shapes = _layer_shapes(wl)
    for k in LAYER_KEYS:
        shp = shapes[k]
        if wl.attn_only and k in ("ln2_g", "ln2_b", "w_fc1", "b_fc1", "w_fc2", "b_fc2"):
            out[k] = from_f64(np.zeros((0,)), wl.dtype)
            continue
        off, sd = _layer_scale(k)
        out[k] = from_f64(off + sd * rng.standard_normal(shp), wl.dtype)
    return out


@dataclass
class Inputs:
    workload: Workload
    x: np.ndarray                         # [T, C] storage dtype
    layers: List[Dict[str, np.ndarray]]   # per layer, storage dtype
    prefix_kv: Optional[np.ndarray] = None   # [S, 2, P, Hkv, d] storage dtype
    extra: Dict[str, np.ndarray] = field(default_factory=dict)


def make_inputs(wl: Workload, layers: Optional[int] = None) -> Inputs:
    """All inputs of a workload, in the fixed draw order.  ``layers`` limits
    how many layers are drawn (the first ones of the same stream)."""
    rng = np.random.Generator(np.random.PCG64(wl.seed))
    T, C = wl.tokens, wl.hidden
    x = from_f64(rng.standard_normal((T, C)), wl.dtype)
    nl = wl.layers if layers is None else min(layers, wl.layers)
    lw = [make_layer_weights(wl, rng) for _ in range(nl)]
    pkv = None
    if wl.prefix_len:
        if nl != wl.layers:
            for _ in range(wl.layers - nl):
                make_layer_weights(wl, rng)
        pkv = from_f64(rng.standard_normal(
            (wl.n_seqs, 2, wl.prefix_len, wl.prefix_heads, wl.head_dim)), wl.dtype)
    return Inputs(wl, x, lw, pkv)


def random_tensor(shape, seed: int, dtype: str, scale: float = 1.0) -> np.ndarray:
    """A standalone seeded N(0, scale^2) tensor in storage dtype, for unit
    tests of single steps."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return from_f64(scale * rng.standard_normal(shape), dtype)


def make_projector_weights(d_in: int, d_hidden: int, d_out: int, seed: int,
                           dtype: str) -> Dict[str, np.ndarray]:
    """Seeded weights of a LayerNorm + two-layer MLP projector (draw order
    ln_g, ln_b, w1, b1, w2, b2; scales as for the encoder layers:
    gamma = 1 + N(0, 0.02), beta and biases N(0, 0.01), weights N(0, 0.02))."""
    rng = np.random.Generator(np.random.PCG64(seed))
    shapes = {"ln_g": (d_in,), "ln_b": (d_in,), "w1": (d_hidden, d_in), "b1": (d_hidden,),
              "w2": (d_out, d_hidden), "b2": (d_out,)}
    out = {}
    for k, shp in shapes.items():
        z = rng.standard_normal(shp)
        if k == "ln_g":
            v = 1.0 + 0.02 * z
        elif k in ("ln_b", "b1", "b2"):
            v = 0.01 * z
        else:
            v = 0.02 * z
        out[k] = from_f64(v, dtype)
    return out


@dataclass
class EmbedInputs:
    """Inputs of the patch embedding (the step before the encoder)."""
    grids: List[Tuple[int, int]]
    patch: int
    images: List[np.ndarray]   # per image [3, rows*patch, cols*patch], storage dtype
    w_pe: np.ndarray           # [C, 3*patch*patch]
    b_pe: np.ndarray           # [C]
    table: np.ndarray          # [table_h, table_w, C]


def make_embed_inputs(wl: Workload, patch: int = 14, table_hw: Tuple[int, int] = (27, 27),
                      seed: Optional[int] = None) -> EmbedInputs:
    """Seeded synthetic pixels (N(0, 1), as normalised images) and a random
    patch projection (N(0, 0.02), bias N(0, 0.01)) and position table
    (N(0, 0.02)) for the workload's image grids; draw order: images, w_pe,
    b_pe, table."""
    rng = np.random.Generator(np.random.PCG64(wl.seed + 1000 if seed is None else seed))
    C = wl.hidden
    imgs = [from_f64(rng.standard_normal((3, r * patch, c * patch)), wl.dtype) for r, c in wl.grids]
    w = from_f64(0.02 * rng.standard_normal((C, 3 * patch * patch)), wl.dtype)
    b = from_f64(0.01 * rng.standard_normal(C), wl.dtype)
    t = from_f64(0.02 * rng.standard_normal((table_hw[0], table_hw[1], C)), wl.dtype)
    return EmbedInputs(list(wl.grids), patch, imgs, w, b, t)
