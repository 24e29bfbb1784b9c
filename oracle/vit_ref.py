"""fp64 CPU oracle of the ViT encoder hot path.  TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import or run this module.  The CUDA library never calls it
and shares no code with it; the only common module is ``synth`` (seeded input
generation, no arithmetic of the method).

Every function is the plain definition of one step, written in fp64 NumPy with
no blocking, fusion or reordering, following the KLiteInfer README
(PaddleOCR-VL SigLIP vision tower):

* intro bullet "多模态全流程自研": a 27-layer SigLIP ViT with 2D RoPE and
  bidirectional attention, followed by a 2x2 spatial merge;
* section "架构", paragraph "视觉算子": row-major batched-token vision ops --
  GEMM + bias, bidirectional attention (two batched GEMMs around a softmax),
  LayerNorm, 2D RoPE, 2x2 spatial merge;
* section "精度与性能": the encoder is 27 layers over 3900 tokens of batched
  GEMMs and carries most of the inference compute.

Points the pages leave open and the reading taken here (each is listed in the
design notes):

1. Layer order is pre-LN:  x1 = x + Wo·Attn(RoPE(QKV(LN1 x))) + bo,
   y = x1 + fc2(GELU(fc1(LN2 x1))).  No final LayerNorm after the stack.
2. LayerNorm uses the biased variance (divide by C) and eps = 1e-6.
3. Attention scale is 1/sqrt(head_dim).
4. 2D RoPE: head dims [0, d/2) rotate by the token's row, dims [d/2, d) by
   its column; inside each half of width h = d/2, dim j pairs with j + h/2
   (j < h/2), frequency w_j = theta^(-2j/h), and the pair (a, b) becomes
   (a cos(p w_j) - b sin(p w_j), b cos(p w_j) + a sin(p w_j)).
5. Tokens are row-major within an image (t = r*W + c) and positions restart
   at (0, 0) for every image.
6. The 2x2 merge concatenates each window in row-major order (top-left,
   top-right, bottom-left, bottom-right); merged tokens are row-major over
   the merged grid; images are merged independently, in order.
7. Prefix K/V (DiT conditioning) is used as given (no RoPE) and precedes the
   sequence's own keys; layout per sequence [2 (K,V), P, kv_heads, d].
8. GELU is the tanh form.

Parity status: every function here is pinned by tests/test_oracle.py
(closed forms, invariants, brute force on tiny inputs, library routines and
hand-written fixtures in tests/golden/).  Agreement with the trained
PaddleOCR-VL encoder itself is not pinned: no weights or tensor dumps exist.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "layernorm", "linear", "gelu_tanh", "rope2d_frequencies", "rope2d",
    "attention", "attention_segment", "layer_forward", "encoder_forward",
    "spatial_merge_2x2", "positions_from_grids", "split_qkv", "projector",
]


# ------------------------------------------------------------------ LayerNorm
def layernorm(x, gamma, beta, eps=1e-6):
    """Per-token LayerNorm over the feature axis ("视觉算子": LayerNorm).

    y = (x - mean) / sqrt(var + eps) * gamma + beta, with the biased variance
    (mean of squared deviations).
    """
    x = np.asarray(x, dtype=np.float64)
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    return (x - mean) / np.sqrt(var + eps) * gamma + beta


# ------------------------------------------------------------------ GEMM
def linear(x, w, b=None):
    """Dense projection with bias ("视觉算子": GEMM + bias).

    ``w`` is [out, in] (one row per output feature); y = x @ w^T + b.
    """
    y = np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T
    if b is not None:
        y = y + b
    return y


def gelu_tanh(u):
    """GELU, tanh form: 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3)))."""
    u = np.asarray(u, dtype=np.float64)
    return 0.5 * u * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (u + 0.044715 * u ** 3)))


# ------------------------------------------------------------------ 2D RoPE
def rope2d_frequencies(head_dim, theta=10000.0):
    """Per-axis rotation frequencies w_j = theta^(-2j/h), h = head_dim/2,
    j = 0 .. h/2-1 (reading 4 above; intro bullet "2D RoPE")."""
    if head_dim % 4:
        raise ValueError("2D RoPE needs head_dim divisible by 4")
    h = head_dim // 2
    j = np.arange(h // 2, dtype=np.float64)
    return theta ** (-2.0 * j / h)


def rope2d(x, pos_rc, theta=10000.0):
    """Rotate every head of ``x`` [T, H, d] by the token positions
    ``pos_rc`` [T, 2] = (row, col) (intro bullet "2D RoPE"; "视觉算子").

    Dims [0, h) use the row, dims [h, d) the column; inside a half, dim j is
    paired with dim j + h/2.
    """
    x = np.asarray(x, dtype=np.float64)
    T, H, d = x.shape
    h = d // 2
    q = h // 2
    w = rope2d_frequencies(d, theta)                       # [q]
    out = x.copy()
    for axis in (0, 1):                                    # 0: row, 1: col
        p = np.asarray(pos_rc, dtype=np.float64)[:, axis]  # [T]
        ang = p[:, None] * w[None, :]                      # [T, q]
        c = np.cos(ang)[:, None, :]
        s = np.sin(ang)[:, None, :]
        lo = axis * h
        a = x[:, :, lo:lo + q]
        b = x[:, :, lo + q:lo + h]
        out[:, :, lo:lo + q] = a * c - b * s
        out[:, :, lo + q:lo + h] = b * c + a * s
    return out


# ------------------------------------------------------------------ attention
def attention_segment(q, k, v, scale):
    """Bidirectional attention of one segment and one head
    ("视觉算子": two batched GEMMs around a softmax, no causal mask).

    q [n, d], k [m, d], v [m, d]; returns softmax(q k^T * scale) v.
    """
    s = (q @ k.T) * scale
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ v


def split_qkv(qkv, heads, head_dim):
    """[T, 3*H*d] -> q, k, v each [T, H, d]; the projection's output features
    are ordered Q (head-major), then K, then V."""
    T = qkv.shape[0]
    t = np.asarray(qkv, dtype=np.float64).reshape(T, 3, heads, head_dim)
    return t[:, 0], t[:, 1], t[:, 2]


def attention(q, k, v, cu_seqlens, pos_rc=None, prefix_kv=None, scale=None,
              theta=10000.0):
    """Varlen bidirectional multi-head attention.

    q, k, v: [T, H, d]; tokens of sequence s are rows cu_seqlens[s] ..
    cu_seqlens[s+1]-1 and attend only to keys of the same sequence
    (block-diagonal mask).  ``pos_rc`` [T, 2] rotates q and k first (2D RoPE).
    ``prefix_kv`` [S, 2, P, Hkv, d] puts P extra keys/values, used as given,
    in front of each sequence's own keys; query head h reads prefix head
    h // (H / Hkv).  Returns o [T, H, d].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    T, H, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if pos_rc is not None:
        q = rope2d(q, pos_rc, theta)
        k = rope2d(k, pos_rc, theta)
    o = np.zeros_like(q)
    cu = [int(c) for c in cu_seqlens]
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if b == a:
            continue
        for h in range(H):
            ks, vs = k[a:b, h], v[a:b, h]
            if prefix_kv is not None:
                pkv = np.asarray(prefix_kv[s], dtype=np.float64)   # [2, P, Hkv, d]
                g = H // pkv.shape[2]
                ks = np.concatenate([pkv[0, :, h // g], ks], axis=0)
                vs = np.concatenate([pkv[1, :, h // g], vs], axis=0)
            o[a:b, h] = attention_segment(q[a:b, h], ks, vs, scale)
    return o


# ------------------------------------------------------------------ layer
def layer_forward(x, w, cu_seqlens, pos_rc, heads, head_dim, eps=1e-6,
                  theta=10000.0, prefix_kv=None, attn_only=False, scale=None):
    """One pre-LN encoder layer (reading 1).  ``w`` maps the names ln1_g,
    ln1_b, w_qkv, b_qkv, w_o, b_o, ln2_g, ln2_b, w_fc1, b_fc1, w_fc2, b_fc2 to
    fp64 arrays.  ``pos_rc`` None disables RoPE.  ``attn_only`` stops after
    the attention residual (DiT-style attention half-layer)."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    hN = layernorm(x, w["ln1_g"], w["ln1_b"], eps)
    qkv = linear(hN, w["w_qkv"], w["b_qkv"])
    q, k, v = split_qkv(qkv, heads, head_dim)
    o = attention(q, k, v, cu_seqlens, pos_rc, prefix_kv, scale, theta)
    x1 = x + linear(o.reshape(T, heads * head_dim), w["w_o"], w["b_o"])
    if attn_only:
        return x1
    h2 = layernorm(x1, w["ln2_g"], w["ln2_b"], eps)
    g = gelu_tanh(linear(h2, w["w_fc1"], w["b_fc1"]))
    return x1 + linear(g, w["w_fc2"], w["b_fc2"])


def encoder_forward(x, layer_weights, cu_seqlens, pos_rc, heads, head_dim,
                    eps=1e-6, theta=10000.0, prefix_kv=None, attn_only=False):
    """The layer stack: each layer's output feeds the next (intro bullet:
    27 layers).  ``layer_weights`` is a sequence of per-layer dicts; anything
    with ``len()`` and indexing will do, so a caller can widen each layer's
    parameters only when the stack reaches it."""
    y = np.asarray(x, dtype=np.float64)
    for i in range(len(layer_weights)):
        y = layer_forward(y, layer_weights[i], cu_seqlens, pos_rc, heads, head_dim, eps,
                          theta, prefix_kv, attn_only)
    return y


# ------------------------------------------------------------------ projector
def projector(x, w, eps=1e-6):
    """The projector that may follow the 2x2 merge, as a composition of the
    steps above with caller-chosen widths (the intro bullet names the
    projector only as the 2x2 spatial merge; a LayerNorm and a two-layer
    GELU MLP after it is the reading taken for models that add one):
    y = GELU_tanh(LN(x) W1^T + b1) W2^T + b2.  ``w`` maps ln_g, ln_b, w1,
    b1, w2, b2 to fp64 arrays."""
    h = layernorm(x, w["ln_g"], w["ln_b"], eps)
    return linear(gelu_tanh(linear(h, w["w1"], w["b1"])), w["w2"], w["b2"])


# ------------------------------------------------------------------ merge
def spatial_merge_2x2(x, grids):
    """2x2 spatial merge (intro bullet: "Projector（2×2 spatial merge）";
    "视觉算子").  Per image with an (H, W) grid of row-major tokens, merged
    token (R, Q) is the concatenation of tokens (2R, 2Q), (2R, 2Q+1),
    (2R+1, 2Q), (2R+1, 2Q+1).  Returns [sum(H*W)/4, 4C]."""
    x = np.asarray(x)
    C = x.shape[1]
    outs = []
    base = 0
    for (H, W) in grids:
        if H % 2 or W % 2:
            raise ValueError("2x2 merge needs even grid sides")
        img = x[base:base + H * W]
        rows = []
        for R in range(H // 2):
            for Q in range(W // 2):
                parts = [img[(2 * R + dr) * W + (2 * Q + dc)]
                         for dr in (0, 1) for dc in (0, 1)]
                rows.append(np.concatenate(parts))
        outs.append(np.stack(rows) if rows else np.zeros((0, 4 * C), x.dtype))
        base += H * W
    return np.concatenate(outs, axis=0) if outs else np.zeros((0, 4 * C), x.dtype)


def positions_from_grids(grids):
    """Sequence offsets and per-token (row, col) for packed images
    (reading 5).  Returns cu_seqlens [S+1] and pos_rc [T, 2], both int32."""
    cu = [0]
    pos = []
    for (H, W) in grids:
        for r in range(H):
            for c in range(W):
                pos.append((r, c))
        cu.append(cu[-1] + H * W)
    return (np.asarray(cu, dtype=np.int32),
            np.asarray(pos, dtype=np.int32).reshape(-1, 2))
