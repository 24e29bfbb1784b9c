"""fp64 CPU oracle of an MXFP8 block-scaled linear layer.  TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import or run this module; the CUDA library never calls it
and shares no code with it.

The pages point at 8-bit arithmetic without defining a format: the NEO++
launcher page lists fp8 variants of its dense checkpoints next to the bf16
ones, and the KLiteInfer README, section "已知限制与后续", puts FP16 / INT8
after CUDA Graph and operator fusion.  The readings taken here (listed in the
design notes):

12. Format: the OCP Microscaling (MX) v1.0 definition of MXFP8 with E4M3
    elements.  Blocks of 32 consecutive elements along the contraction
    dimension K share one E8M0 scale 2^X (the byte X + 127).  An E4M3 byte
    is sign | 4 exponent bits (bias 7) | 3 mantissa bits; exponent field 0
    holds the subnormals m·2^-9; the all-ones pattern S.1111.111 is NaN;
    there is no infinity; the largest normal is 1.75·2^8 = 448.
13. A block's shared exponent is X = floor(log2(amax)) - 8, where 8 is the
    exponent of E4M3's largest normal, clamped to [-127, 127]; an all-zero
    block takes X = -127.  Each element becomes x / 2^X rounded to nearest
    (ties to even) in E4M3, with magnitudes above 448 clamped to 448 (the
    scaled block maximum lies in [256, 512), so the clamp can only touch
    elements above 448·2^X).
14. When K is not a multiple of 32 the last block holds the remaining
    elements only.
15. The layer is y = deq(A) · deq(W)^T + b, followed by the epilogue of the
    bf16 path it stands in for (none, GELU-tanh, or + residual), in fp64.
    A is [M, K] (activations, blocks along each row); W is [N, K] (a
    PyTorch Linear weight, blocks along each row, i.e. per output column
    of y).
16. An FP8 encoder layer runs the four projections (QKV, output, fc1, fc2)
    in MXFP8: each projection's input activation and weight are quantised
    along K, then multiplied as in 15.  LayerNorm, RoPE, attention, GELU
    and the residual adds are those of the bf16 layer (vit_ref).

Parity status: pinned by tests/test_oracle.py -- the E4M3 table and the
rounding against PyTorch's float8_e4m3fn conversion, round trips of every
code, the block exponent's closed form, exactness on representable blocks,
the error bound of round-to-nearest, the linear layer against an integer
matmul and under power-of-two rescaling, and the FP8 encoder layer against
the fp64 layer (equal with the projections unquantised; every projection
routed through the quantised product; bounded error when quantised).
"""
from __future__ import annotations

import numpy as np

from . import vit_ref as R

__all__ = ["E4M3_MAX", "BLOCK", "e4m3_decode", "e4m3_encode", "mx_block_exponents",
           "mx_quantize", "mx_dequantize", "mx_linear", "mx_project", "layer_forward_mx8"]

E4M3_MAX = 448.0
BLOCK = 32
_EMAX = 8          # exponent of the largest E4M3 normal (reading 13)
_EMIN = -6         # exponent of the smallest E4M3 normal
_MBITS = 3


def e4m3_decode(codes):
    """E4M3 bytes -> fp64 values, from the bit fields (reading 12)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    sub = m * 2.0 ** -9
    v = s * np.where(e == 0, sub, normal)
    return np.where((e == 15) & (m == 7), np.nan, v)


def e4m3_encode(x):
    """fp64 values -> E4M3 bytes: round to nearest, ties to even, magnitudes
    above 448 clamped to 448, NaN to 0x7F (reading 13)."""
    x = np.asarray(x, dtype=np.float64)
    nan = np.isnan(x)
    a = np.minimum(np.abs(np.where(nan, 0.0, x)), E4M3_MAX)
    _, fe = np.frexp(a)                              # a = f·2^fe, f in [0.5, 1)
    e = np.maximum(fe - 1, _EMIN)                    # binade of a (subnormals share the lowest)
    q = np.exp2((e - _MBITS).astype(np.float64))     # spacing of E4M3 values in that binade
    r = np.rint(a / q)                               # a/q is exact; rint rounds ties to even
    up = r >= 2 ** (_MBITS + 1)                      # rounded up into the next binade
    e = np.where(up, e + 1, e)
    r = np.where(up, r / 2, r).astype(np.int64)
    subnormal = (e == _EMIN) & (r < 2 ** _MBITS)
    field_e = np.where(subnormal, 0, e + 7)
    field_m = np.where(subnormal, r, r - 2 ** _MBITS)
    code = (field_e << _MBITS) | field_m
    code = np.where(a == 0, 0, code)
    code = code | np.where(np.signbit(x), 0x80, 0)
    return np.where(nan, 0x7F, code).astype(np.uint8)


def _blocks(k):
    """[start, stop) of each 32-element block of a K-long row (reading 14)."""
    return [(s, min(s + BLOCK, k)) for s in range(0, k, BLOCK)]


def mx_block_exponents(x):
    """[R, K] -> shared exponents X [R, ceil(K/32)] (reading 13)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty((x.shape[0], len(_blocks(x.shape[1]))), dtype=np.int64)
    for j, (s, t) in enumerate(_blocks(x.shape[1])):
        amax = np.max(np.abs(x[:, s:t]), axis=1)
        _, fe = np.frexp(amax)
        out[:, j] = np.where(amax > 0, fe - 1 - _EMAX, -127)
    return np.clip(out, -127, 127)


def mx_quantize(x):
    """[R, K] -> (E4M3 codes [R, K], E8M0 scale bytes [R, ceil(K/32)])."""
    x = np.asarray(x, dtype=np.float64)
    X = mx_block_exponents(x)
    codes = np.empty(x.shape, dtype=np.uint8)
    for j, (s, t) in enumerate(_blocks(x.shape[1])):
        codes[:, s:t] = e4m3_encode(x[:, s:t] / np.exp2(X[:, j:j + 1].astype(np.float64)))
    return codes, (X + 127).astype(np.uint8)


def mx_dequantize(codes, scales):
    """(codes [R, K], scale bytes [R, nb]) -> fp64 [R, K]."""
    v = e4m3_decode(codes)
    sc = np.asarray(scales, dtype=np.int64) - 127
    out = np.empty(v.shape)
    for j, (s, t) in enumerate(_blocks(v.shape[1])):
        out[:, s:t] = v[:, s:t] * np.exp2(sc[:, j:j + 1].astype(np.float64))
    return out


def mx_linear(a_codes, a_scales, w_codes, w_scales, bias=None, epilogue="none", residual=None):
    """y = deq(A)·deq(W)^T + b, then the epilogue (reading 15)."""
    y = mx_dequantize(a_codes, a_scales) @ mx_dequantize(w_codes, w_scales).T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)
    if epilogue == "gelu":
        y = 0.5 * y * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (y + 0.044715 * y ** 3)))
    elif epilogue == "residual":
        y = y + np.asarray(residual, dtype=np.float64)
    elif epilogue != "none":
        raise ValueError(epilogue)
    return y


def mx_project(x, w, b=None):
    """One projection of the FP8 layer: x [M, K] and w [N, K] each quantised
    along K, then deq(x)·deq(w)^T + b (readings 13, 15, 16)."""
    qa, sa = mx_quantize(x)
    qw, sw = mx_quantize(w)
    return mx_linear(qa, sa, qw, sw, b)


def layer_forward_mx8(x, w, cu_seqlens, pos_rc, heads, head_dim, eps=1e-6, theta=10000.0,
                      prefix_kv=None, attn_only=False, project=mx_project):
    """The pre-LN encoder layer of vit_ref.layer_forward with its four
    projections computed by ``project`` (MXFP8 by default, reading 16)."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    h = R.layernorm(x, w["ln1_g"], w["ln1_b"], eps)
    q, k, v = R.split_qkv(project(h, w["w_qkv"], w["b_qkv"]), heads, head_dim)
    o = R.attention(q, k, v, cu_seqlens, pos_rc, prefix_kv, None, theta)
    x1 = x + project(o.reshape(T, heads * head_dim), w["w_o"], w["b_o"])
    if attn_only:
        return x1
    h2 = R.layernorm(x1, w["ln2_g"], w["ln2_b"], eps)
    g = R.gelu_tanh(project(h2, w["w_fc1"], w["b_fc1"]))
    return x1 + project(g, w["w_fc2"], w["b_fc2"])
