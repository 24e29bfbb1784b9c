"""Python binding of libvit (include/vit.h): a B200 (sm_100a) implementation
of the vision-transformer encoder hot path -- pre-LN layers of LayerNorm,
QKV GEMM + bias, 2D RoPE, bidirectional varlen attention (optional prefix
K/V), output projection + residual and a GELU-tanh MLP, then the 2x2 spatial
merge.

This module only marshals arguments: every step runs in the CUDA kernels of
``libvit.so``.  There is no fallback; importing fails loudly when the library
has not been built (``python vision_transformer_encoder_layernorm_b200/build.py``).
Tensors are PyTorch tensors (device memory and streams only).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

__all__ = [
    "lib", "LIB_PATH", "VitError", "VitConfig", "VitLayerWeights", "VitProjectorWeights",
    "VitSeqs", "Context",
    "F32", "BF16", "FLAG_NO_ROPE", "FLAG_NO_MLP", "EPI_BIAS", "EPI_BIAS_GELU",
    "EPI_BIAS_RESIDUAL", "STATUS", "ABI_FUNCTIONS", "KERNEL_KINDS", "Graph",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvit.so")

F32, BF16 = 0, 1
FLAG_NO_ROPE, FLAG_NO_MLP = 0x1, 0x2
EPI_BIAS, EPI_BIAS_GELU, EPI_BIAS_RESIDUAL = 0, 1, 2
KERNEL_KINDS = ("layernorm", "gemm_qkv", "rope", "attention", "gemm_out", "gemm_fc1",
                "gemm_fc2", "merge", "positions", "gemm", "embed", "mx8_quantize", "gemm_mx8",
                "rowstats", "fold")
STATUS = {0: "VIT_OK", 1: "VIT_ERR_INVALID_ARG", 2: "VIT_ERR_SHAPE", 3: "VIT_ERR_UNSUPPORTED",
          4: "VIT_ERR_WORKSPACE", 5: "VIT_ERR_CUDA", 6: "VIT_ERR_TIMEOUT",
          7: "VIT_ERR_DEVICE_BOUNDS"}


class VitError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} -> {STATUS.get(code, code)}")
        self.code = code


class VitConfig(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("mlp", ctypes.c_int), ("ln_eps", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("dtype", ctypes.c_int), ("flags", ctypes.c_uint)]


_WKEYS = ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o",
          "ln2_g", "ln2_b", "w_fc1", "b_fc1", "w_fc2", "b_fc2", "qkv_fold", "fc1_fold")


class VitLayerWeights(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in _WKEYS]


class VitProjectorWeights(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in ("ln_g", "ln_b", "w1", "b1", "w2", "b2")]


_MX8KEYS = ("ln1_g", "ln1_b", "b_qkv", "b_o", "ln2_g", "ln2_b", "b_fc1", "b_fc2",
            "w_qkv_codes", "w_qkv_scales", "w_o_codes", "w_o_scales",
            "w_fc1_codes", "w_fc1_scales", "w_fc2_codes", "w_fc2_scales")


class VitLayerWeightsMx8(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in _MX8KEYS]


class VitSeqs(ctypes.Structure):
    _fields_ = [("total_tokens", ctypes.c_int), ("n_seqs", ctypes.c_int),
                ("max_seqlen", ctypes.c_int), ("cu_seqlens", ctypes.c_void_p),
                ("pos_rc", ctypes.c_void_p), ("prefix_kv", ctypes.c_void_p),
                ("prefix_len", ctypes.c_int), ("kv_heads", ctypes.c_int)]


_P = ctypes.c_void_p
_I = ctypes.c_int
# name -> (restype, argtypes); the exported C ABI of include/vit.h
ABI_FUNCTIONS = {
    "vit_init": (_I, [ctypes.POINTER(VitConfig), _I, ctypes.POINTER(_P)]),
    "vit_destroy": (None, [_P]),
    "vit_workspace_bytes": (ctypes.c_size_t, [_P, _I]),
    "vit_fold_layernorm": (_I, [_P, ctypes.POINTER(VitLayerWeights), _P, _P, _P, _P, _P]),
    "vit_layer_forward": (_I, [_P, ctypes.POINTER(VitLayerWeights), _P, _P,
                               ctypes.POINTER(VitSeqs), _P, ctypes.c_size_t, _P]),
    "vit_layer_forward_noalloc": (_I, [_P, ctypes.POINTER(VitLayerWeights), _P, _P,
                                       ctypes.POINTER(VitSeqs), _P]),
    "vit_encoder_forward": (_I, [_P, ctypes.POINTER(VitLayerWeights), _I, _P, _P,
                                 ctypes.POINTER(VitSeqs), _P, ctypes.c_size_t, _P]),
    "vit_attention": (_I, [_P, _P, _P, ctypes.POINTER(VitSeqs), ctypes.c_float, _P]),
    "vit_spatial_merge_2x2": (_I, [_P, _P, _P, ctypes.POINTER(ctypes.c_int32), _I, _I, _P]),
    "vit_positions_from_grids": (_I, [_P, ctypes.POINTER(ctypes.c_int32), _I, _P, _P, _P]),
    "vit_layernorm": (_I, [_P, _P, _P, _P, _P, _I, _I, ctypes.c_float, _P]),
    "vit_linear": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "vit_rope2d": (_I, [_P, _P, _P, _I, _P]),
    "vit_profile_enable": (_I, [_P, _I]),
    "vit_profile_read": (_I, [_P, _I, ctypes.POINTER(ctypes.c_longlong),
                              ctypes.POINTER(ctypes.c_double), _I]),
    "vit_embed_workspace_bytes": (ctypes.c_size_t, [_P, _I, _I]),
    "vit_projector_workspace_bytes": (ctypes.c_size_t, [_P, _I, _I, _I]),
    "vit_workspace_bytes_mx8": (ctypes.c_size_t, [_P, _I]),
    "vit_encoder_forward_mx8": (_I, [_P, ctypes.POINTER(VitLayerWeightsMx8), _I, _P, _P,
                                     ctypes.POINTER(VitSeqs), _P, ctypes.c_size_t, _P]),
    "vit_projector": (_I, [_P, ctypes.POINTER(VitProjectorWeights), _P, _P, _I, _I, _I, _I, _P,
                           ctypes.c_size_t, _P]),
    "vit_patch_embed": (_I, [_P, _P, ctypes.POINTER(ctypes.c_int32), _I, _I, _P, _P, _P, _I, _I,
                             _P, _P, ctypes.c_size_t, _P]),
    "vit_patch_embed_padded": (_I, [_P, _P, ctypes.POINTER(ctypes.c_int32), _I, _I, _P, _P, _P, _I,
                                    _I, _P, _P, ctypes.c_size_t, _P]),
    "vit_patch_kp": (_I, [_I]),
    "vit_pad_patch_weight": (_I, [_P, _P, _I, _P, _P]),
    "vit_pos_interp": (_I, [_P, _P, _I, _I, ctypes.POINTER(ctypes.c_int32), _I, _P, _P]),
    "vit_graph_begin": (_I, [_P, ctypes.POINTER(_P)]),
    "vit_graph_end": (_I, [_P, ctypes.POINTER(_P)]),
    "vit_graph_launch": (_I, [_P, _P]),
    "vit_graph_kernels": (ctypes.c_longlong, [_P]),
    "vit_graph_destroy": (None, [_P]),
    "vit_mx8_row_bytes": (ctypes.c_size_t, [_I]),
    "vit_mx8_scale_bytes": (ctypes.c_size_t, [_I, _I]),
    "vit_mx8_quantize": (_I, [_P, _P, _I, _I, _P, _P, _P]),
    "vit_layernorm_mx8": (_I, [_P, _P, _P, _P, _I, _I, ctypes.c_float, _P, _P, _P]),
    "vit_linear_mx8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "vit_get_last_device_status": (_I, [_P]),
    "vit_debug_lost_tx": (_I, [_P, ctypes.c_uint]),
    "vit_status_string": (ctypes.c_char_p, [_I]),
    "vit_version": (ctypes.c_char_p, []),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python vision_transformer_encoder_layernorm_b200/build.py` (nvcc, sm_100a)")
    h = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in ABI_FUNCTIONS.items():
        fn = getattr(h, name)
        fn.restype = res
        fn.argtypes = args
    return h


lib = _load()


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _check(fn: str, code: int):
    if code != 0:
        raise VitError(fn, code)


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def mx8_row_bytes(K: int) -> int:
    """Bytes per row of an MXFP8 code matrix with K columns."""
    return int(lib.vit_mx8_row_bytes(K))


def mx8_scale_bytes(rows: int, K: int) -> int:
    """Bytes of the E8M0 scale blocks of a [rows, K] MXFP8 matrix."""
    return int(lib.vit_mx8_scale_bytes(rows, K))


def _grids_arr(grids: Sequence[Sequence[int]]):
    flat = [int(v) for g in grids for v in g]
    return (ctypes.c_int32 * len(flat))(*flat), len(grids)


def layer_weights(d) -> VitLayerWeights:
    """A VitLayerWeights from a mapping of the parameter names (the 12 of a
    layer, plus qkv_fold / fc1_fold of folded LayerNorms) to tensors (missing
    or None entries become NULL).  The struct keeps the tensors alive: it
    holds raw device pointers."""
    lw = VitLayerWeights(*[_ptr(d.get(k)) for k in _WKEYS])
    lw._tensors = dict(d)
    return lw


def seqs(total_tokens: int, n_seqs: int, max_seqlen: int, cu_seqlens, pos_rc=None,
         prefix_kv=None, prefix_len: int = 0, kv_heads: int = 0) -> VitSeqs:
    """A VitSeqs for packed sequences.  The struct keeps the cu_seqlens,
    pos_rc and prefix_kv tensors alive (it holds their raw device pointers),
    so temporaries passed here cannot be freed and reused while it lives."""
    s = VitSeqs(total_tokens, n_seqs, max_seqlen, _ptr(cu_seqlens), _ptr(pos_rc),
                _ptr(prefix_kv), prefix_len if prefix_kv is not None else 0, kv_heads)
    s._tensors = (cu_seqlens, pos_rc, prefix_kv)
    return s


class Graph:
    """A captured sequence of library calls (see vit_graph_begin in vit.h).
    Every pointer used while capturing is baked in: keep those tensors alive."""

    def __init__(self, handle: int):
        self._h = handle
        self.kernels = int(lib.vit_graph_kernels(handle))

    def launch(self, stream=None):
        _check("vit_graph_launch", lib.vit_graph_launch(self._h, _stream(stream)))

    def close(self):
        if self._h:
            lib.vit_graph_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Context:
    """Owns one ``vit_ctx``; each method is the C entry point of the same name
    (without the ``vit_`` prefix) with tensors in place of pointers."""

    def __init__(self, hidden, heads, head_dim, mlp, dtype=BF16, ln_eps=1e-6,
                 rope_theta=10000.0, flags=0, device=0):
        self.cfg = VitConfig(hidden, heads, head_dim, mlp, ln_eps, rope_theta, dtype, flags)
        h = ctypes.c_void_p()
        _check("vit_init", lib.vit_init(ctypes.byref(self.cfg), device, ctypes.byref(h)))
        self._h = h

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None):
            lib.vit_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace_bytes(self, total_tokens: int) -> int:
        return lib.vit_workspace_bytes(self._h, total_tokens)

    def fold_layernorm(self, weights, in_place: bool = False, stream=None):
        """vit_fold_layernorm: returns a copy of the layer's weight mapping
        whose w_qkv / w_fc1 are the LayerNorm-folded weights, with the
        qkv_fold / fc1_fold vectors (new tensors; with in_place the folded
        weights overwrite w_qkv / w_fc1 of ``weights``)."""
        import torch
        w_qkv, w_fc1 = weights["w_qkv"], weights.get("w_fc1")
        mlp = w_fc1 is not None and not (self.cfg.flags & FLAG_NO_MLP)
        out = dict(weights)
        out["w_qkv"] = w_qkv if in_place else torch.empty_like(w_qkv)
        out["qkv_fold"] = torch.empty((2, w_qkv.shape[0]), dtype=torch.float32,
                                      device=w_qkv.device)
        if mlp:
            out["w_fc1"] = w_fc1 if in_place else torch.empty_like(w_fc1)
            out["fc1_fold"] = torch.empty((2, w_fc1.shape[0]), dtype=torch.float32,
                                          device=w_fc1.device)
        lw = layer_weights(weights)
        _check("vit_fold_layernorm", lib.vit_fold_layernorm(
            self._h, ctypes.byref(lw), _ptr(out["w_qkv"]), _ptr(out["qkv_fold"]),
            _ptr(out.get("w_fc1") if mlp else None), _ptr(out.get("fc1_fold")),
            _stream(stream)))
        for k in ("ln1_g", "ln1_b", "b_qkv") + (("ln2_g", "ln2_b", "b_fc1") if mlp else ()):
            out[k] = None  # not read by a folded layer
        return out

    def quantize_layer_mx8(self, weights, stream=None):
        """The layer's four projection weights quantised once to MXFP8 (new
        tensors); returns the mapping vit_encoder_forward_mx8 takes (the
        LayerNorm vectors and biases are passed through)."""
        import torch
        out = {k: weights.get(k) for k in ("ln1_g", "ln1_b", "b_qkv", "b_o", "ln2_g", "ln2_b",
                                           "b_fc1", "b_fc2")}
        for name in ("w_qkv", "w_o", "w_fc1", "w_fc2"):
            w = weights.get(name)
            if w is None:
                continue
            n, k = w.shape
            codes = torch.empty((n, mx8_row_bytes(k)), dtype=torch.uint8, device=w.device)
            scales = torch.empty(mx8_scale_bytes(n, k), dtype=torch.uint8, device=w.device)
            self.mx8_quantize(w, codes, scales, stream)
            out[name + "_codes"], out[name + "_scales"] = codes, scales
        return out

    def workspace_bytes_mx8(self, total_tokens: int) -> int:
        return int(lib.vit_workspace_bytes_mx8(self._h, total_tokens))

    def encoder_forward_mx8(self, layers, x, y, sq: VitSeqs, workspace, stream=None):
        """vit_encoder_forward_mx8; ``layers`` are mappings from
        quantize_layer_mx8."""
        arr = (VitLayerWeightsMx8 * len(layers))(
            *[VitLayerWeightsMx8(*[_ptr(l.get(k)) for k in _MX8KEYS]) for l in layers])
        _check("vit_encoder_forward_mx8", lib.vit_encoder_forward_mx8(
            self._h, arr, len(layers), _ptr(x), _ptr(y), ctypes.byref(sq), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream)))

    def layer_forward(self, weights, x, y, sq: VitSeqs, workspace, stream=None):
        lw = layer_weights(weights) if not isinstance(weights, VitLayerWeights) else weights
        _check("vit_layer_forward", lib.vit_layer_forward(
            self._h, ctypes.byref(lw), _ptr(x), _ptr(y), ctypes.byref(sq), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream)))

    def layer_forward_noalloc(self, weights, x, y, sq: VitSeqs, stream=None):
        """vit_layer_forward_noalloc: the layer with the library's fixed
        32 MiB scratch instead of a workspace (allocates nothing)."""
        lw = layer_weights(weights) if not isinstance(weights, VitLayerWeights) else weights
        _check("vit_layer_forward_noalloc", lib.vit_layer_forward_noalloc(
            self._h, ctypes.byref(lw), _ptr(x), _ptr(y), ctypes.byref(sq), _stream(stream)))

    def encoder_forward(self, layers, x, y, sq: VitSeqs, workspace, stream=None):
        arr = (VitLayerWeights * len(layers))(
            *[l if isinstance(l, VitLayerWeights) else layer_weights(l) for l in layers])
        _check("vit_encoder_forward", lib.vit_encoder_forward(
            self._h, arr, len(layers), _ptr(x), _ptr(y), ctypes.byref(sq), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream)))

    def attention(self, qkv, o, sq: VitSeqs, scale: float = 0.0, stream=None):
        _check("vit_attention", lib.vit_attention(self._h, _ptr(qkv), _ptr(o), ctypes.byref(sq),
                                                  scale, _stream(stream)))

    def spatial_merge_2x2(self, x, y, grids, channels: int, stream=None):
        arr, n = _grids_arr(grids)
        _check("vit_spatial_merge_2x2", lib.vit_spatial_merge_2x2(
            self._h, _ptr(x), _ptr(y), arr, n, channels, _stream(stream)))

    def positions_from_grids(self, grids, cu_seqlens, pos_rc, stream=None):
        arr, n = _grids_arr(grids)
        _check("vit_positions_from_grids", lib.vit_positions_from_grids(
            self._h, arr, n, _ptr(cu_seqlens), _ptr(pos_rc), _stream(stream)))

    def layernorm(self, x, y, gamma, beta, eps: float = 1e-6, stream=None):
        rows, cols = x.shape
        _check("vit_layernorm", lib.vit_layernorm(self._h, _ptr(x), _ptr(y), _ptr(gamma),
                                                  _ptr(beta), rows, cols, eps, _stream(stream)))

    def linear(self, x, w, bias, y, epi=EPI_BIAS, residual=None, stream=None):
        M, K = x.shape
        N = w.shape[0]
        _check("vit_linear", lib.vit_linear(self._h, _ptr(x), _ptr(w), _ptr(bias), _ptr(residual),
                                            _ptr(y), M, N, K, epi, _stream(stream)))

    def mx8_quantize(self, x, codes, scales, stream=None):
        """bf16 x [rows, K] -> MXFP8 codes [rows, mx8_row_bytes(K)] (uint8) and
        scales [mx8_scale_bytes(rows, K)] (uint8), see vit_mx8_quantize."""
        rows, K = x.shape
        _check("vit_mx8_quantize", lib.vit_mx8_quantize(self._h, _ptr(x), rows, K, _ptr(codes),
                                                        _ptr(scales), _stream(stream)))

    def layernorm_mx8(self, x, gamma, beta, codes, scales, eps=None, stream=None):
        """vit_layernorm_mx8: LayerNorm of bf16 x [rows, cols] straight to MXFP8
        codes / scales (the layout of mx8_quantize)."""
        rows, cols = x.shape
        e = self.cfg.ln_eps if eps is None else eps
        _check("vit_layernorm_mx8", lib.vit_layernorm_mx8(self._h, _ptr(x), _ptr(gamma), _ptr(beta),
                                                          rows, cols, e, _ptr(codes), _ptr(scales),
                                                          _stream(stream)))

    def linear_mx8(self, a, w, bias, y, K, epi=EPI_BIAS, residual=None, stream=None):
        """y = epi(deq(A) deq(W)^T + bias) with a = (codes, scales) [M, K] and
        w = (codes, scales) [N, K] from mx8_quantize."""
        M, N = y.shape
        _check("vit_linear_mx8", lib.vit_linear_mx8(self._h, _ptr(a[0]), _ptr(a[1]), _ptr(w[0]),
                                                    _ptr(w[1]), _ptr(bias), _ptr(residual), _ptr(y),
                                                    M, N, K, epi, _stream(stream)))

    def rope2d(self, qkv, pos_rc, stream=None):
        _check("vit_rope2d", lib.vit_rope2d(self._h, _ptr(qkv), _ptr(pos_rc), qkv.shape[0],
                                            _stream(stream)))

    def debug_lost_tx(self, nbytes: int):
        """Fault injection for the watchdog tests (vit_debug_lost_tx)."""
        _check("vit_debug_lost_tx", lib.vit_debug_lost_tx(self._h, nbytes))

    def device_status(self) -> int:
        return lib.vit_get_last_device_status(self._h)

    def profile_enable(self, enable: bool = True):
        _check("vit_profile_enable", lib.vit_profile_enable(self._h, int(bool(enable))))

    def projector_workspace_bytes(self, M: int, d_in: int, d_hidden: int) -> int:
        return int(lib.vit_projector_workspace_bytes(self._h, M, d_in, d_hidden))

    def projector(self, weights, x, y, workspace, stream=None):
        """vit_projector: y = GELU(LN(x) W1^T + b1) W2^T + b2; ``weights``
        maps ln_g, ln_b, w1, b1, w2, b2 to tensors."""
        M, d_in = x.shape
        d_hidden, d_out = weights["w1"].shape[0], weights["w2"].shape[0]
        pw = VitProjectorWeights(*[_ptr(weights.get(k)) for k in
                                   ("ln_g", "ln_b", "w1", "b1", "w2", "b2")])
        _check("vit_projector", lib.vit_projector(
            self._h, ctypes.byref(pw), _ptr(x), _ptr(y), M, d_in, d_hidden, d_out,
            _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))

    def embed_workspace_bytes(self, total_tokens: int, patch: int) -> int:
        return int(lib.vit_embed_workspace_bytes(self._h, total_tokens, patch))

    def patch_embed(self, pixels, grids, patch: int, w_pe, b_pe, pos_table, y, workspace,
                    stream=None):
        """Tokens y [T, C] of packed images (pixels: all images' [3, rows*patch,
        cols*patch] back to back); pos_table [table_h, table_w, C]."""
        arr, n = _grids_arr(grids)
        th, tw = int(pos_table.shape[0]), int(pos_table.shape[1])
        _check("vit_patch_embed", lib.vit_patch_embed(
            self._h, _ptr(pixels), arr, n, patch, _ptr(w_pe), _ptr(b_pe), _ptr(pos_table), th, tw,
            _ptr(y), _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(stream)))

    def pad_patch_weight(self, w_pe, patch: int, stream=None):
        """vit_pad_patch_weight: w_pe [C, 3*patch*patch] (or [C, 3, patch,
        patch]) -> a new [C, vit_patch_kp(patch)] tensor in the GEMM's layout."""
        import torch
        kp = int(lib.vit_patch_kp(patch))
        if kp <= 0:
            raise VitError(STATUS["VIT_ERR_INVALID_ARG"], "vit_patch_kp")
        w_pad = torch.empty((w_pe.shape[0], kp), dtype=w_pe.dtype, device=w_pe.device)
        _check("vit_pad_patch_weight", lib.vit_pad_patch_weight(self._h, _ptr(w_pe), patch,
                                                                _ptr(w_pad), _stream(stream)))
        return w_pad

    def patch_embed_padded(self, pixels, grids, patch: int, w_pad, b_pe, pos_table, y, workspace,
                           stream=None):
        """patch_embed with the weight from pad_patch_weight (one launch fewer)."""
        arr, n = _grids_arr(grids)
        th, tw = int(pos_table.shape[0]), int(pos_table.shape[1])
        _check("vit_patch_embed_padded", lib.vit_patch_embed_padded(
            self._h, _ptr(pixels), arr, n, patch, _ptr(w_pad), _ptr(b_pe), _ptr(pos_table), th, tw,
            _ptr(y), _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(stream)))

    def pos_interp(self, pos_table, grids, y, stream=None):
        arr, n = _grids_arr(grids)
        _check("vit_pos_interp", lib.vit_pos_interp(
            self._h, _ptr(pos_table), int(pos_table.shape[0]), int(pos_table.shape[1]), arr, n,
            _ptr(y), _stream(stream)))

    def graph_begin(self) -> int:
        """Starts capturing this context's calls; returns the capture stream
        (pass it as `stream=` to the calls to record)."""
        h = _P()
        _check("vit_graph_begin", lib.vit_graph_begin(self._h, ctypes.byref(h)))
        return h.value

    def graph_end(self) -> "Graph":
        """Ends the capture started by graph_begin and returns the graph."""
        h = _P()
        _check("vit_graph_end", lib.vit_graph_end(self._h, ctypes.byref(h)))
        return Graph(h.value)

    def profile_read(self, reset: bool = False):
        """{kind name: (launches, total device ms)} for every kernel kind."""
        out = {}
        for k, name in enumerate(KERNEL_KINDS):
            n, ms = ctypes.c_longlong(), ctypes.c_double()
            _check("vit_profile_read", lib.vit_profile_read(self._h, k, ctypes.byref(n),
                                                            ctypes.byref(ms), 0))
            out[name] = (n.value, ms.value)
        if reset:
            n, ms = ctypes.c_longlong(), ctypes.c_double()
            _check("vit_profile_read", lib.vit_profile_read(self._h, 0, ctypes.byref(n),
                                                            ctypes.byref(ms), 1))
        return out
