"""fp64 CPU oracle of the steps before the encoder: patch embedding and the
bilinear interpolation of the position-embedding table.  TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import or run this module; the CUDA library never calls it
and shares no code with it.

KLiteInfer README:
* section "精度与性能": patch embedding is the first of the eight stages the
  implementation is compared on;
* section "架构", paragraph "视觉算子": a bilinear position-embedding
  interpolation is one of the vision operators.

The pages give neither the patch size nor the table size, nor the layout or
interpolation convention.  The readings taken here (listed in the design
notes):

9.  An image is [3, rows*p, cols*p], channels first.  Its tokens are its
    rows x cols patches in row-major order (the token order of the encoder).
    A token is a stride-p convolution of its patch: y = w_pe · vec(patch) +
    b_pe.  Here w_pe is [C, 3*p*p], a Conv2d weight [C, 3, p, p] flattened,
    and vec() flattens the patch in (channel, y, x) order.
10. A learned table [gh, gw, C] is resized to each image's (rows, cols) by
    bilinear interpolation with half-pixel centres, as PyTorch's default
    (align_corners=False, no antialiasing).  Source coordinate
    s = (i + 0.5)·g/n − 0.5, clamped below at 0; neighbours floor(s) and
    min(floor(s) + 1, g − 1).  The resized table is added to the patch
    embeddings.
11. Images are embedded independently and packed in order.

Parity status: pinned by tests/test_oracle.py (fp64 conv2d and interpolate
library routines, an exact closed form for affine tables, identity and
constant cases).
"""
from __future__ import annotations

import numpy as np

__all__ = ["patchify", "patch_embed", "bilinear_source", "bilinear_resize", "embed_images"]


def patchify(image, p):
    """[3, rows*p, cols*p] -> [rows*cols, 3*p*p]: patch (r, c) flattened in
    (channel, y, x) order, patches row-major (reading 9)."""
    image = np.asarray(image, dtype=np.float64)
    ch, h, w = image.shape
    rows, cols = h // p, w // p
    out = np.empty((rows * cols, ch * p * p))
    for r in range(rows):
        for c in range(cols):
            out[r * cols + c] = image[:, r * p:(r + 1) * p, c * p:(c + 1) * p].reshape(-1)
    return out


def patch_embed(image, w_pe, b_pe, p):
    """Stride-p convolution of one image as tokens [rows*cols, C] (reading 9)."""
    return patchify(image, p) @ np.asarray(w_pe, np.float64).T + np.asarray(b_pe, np.float64)


def bilinear_source(i, n_out, n_in):
    """Half-pixel source coordinate of output index i (reading 10): the two
    neighbours and the weight of the second."""
    s = max((i + 0.5) * n_in / n_out - 0.5, 0.0)
    i0 = int(np.floor(s))
    i1 = min(i0 + 1, n_in - 1)
    return i0, i1, s - i0


def bilinear_resize(table, out_h, out_w):
    """[gh, gw, C] -> [out_h, out_w, C] by bilinear interpolation (reading 10)."""
    table = np.asarray(table, dtype=np.float64)
    gh, gw, ch = table.shape
    out = np.empty((out_h, out_w, ch))
    for i in range(out_h):
        y0, y1, wy = bilinear_source(i, out_h, gh)
        for j in range(out_w):
            x0, x1, wx = bilinear_source(j, out_w, gw)
            top = (1.0 - wx) * table[y0, x0] + wx * table[y0, x1]
            bot = (1.0 - wx) * table[y1, x0] + wx * table[y1, x1]
            out[i, j] = (1.0 - wy) * top + wy * bot
    return out


def embed_images(images, grids, p, w_pe, b_pe, table):
    """Tokens [T, C] of the packed images: patch embedding plus the table
    resized to each image's grid (readings 9-11)."""
    out = []
    for img, (rows, cols) in zip(images, grids):
        emb = patch_embed(img, w_pe, b_pe, p)
        pos = bilinear_resize(table, rows, cols).reshape(rows * cols, -1)
        out.append(emb + pos)
    return np.concatenate(out, axis=0)
