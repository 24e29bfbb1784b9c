"""Host-only checks of the C ABI library: it loads, exports every entry point
declared in include/vit.h, and rejects bad arguments without touching a GPU.
No compute call is made here."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vit.h")


def header_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"VIT_API\s+[\w\s\*]+?\b(vit_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    fns = header_functions()
    for name in ("vit_init", "vit_destroy", "vit_workspace_bytes", "vit_layer_forward",
                 "vit_encoder_forward", "vit_attention", "vit_spatial_merge_2x2",
                 "vit_positions_from_grids", "vit_get_last_device_status", "vit_status_string"):
        assert name in fns


def test_library_exports_every_declared_symbol():
    import vision_transformer_encoder_layernorm_b200 as vit
    out = subprocess.run(["nm", "-D", "--defined-only", vit.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (vit_\w+)", out))
    declared = set(header_functions())
    assert declared <= exported, declared - exported
    assert set(vit.ABI_FUNCTIONS) == declared


def test_status_strings_and_version():
    import vision_transformer_encoder_layernorm_b200 as vit
    for code, name in vit.STATUS.items():
        assert vit.lib.vit_status_string(code).decode() == name
    assert vit.lib.vit_status_string(99).decode() == "VIT_ERR_UNKNOWN"
    assert b"sm_100a" in vit.lib.vit_version()


def test_null_arguments_rejected_without_gpu():
    import vision_transformer_encoder_layernorm_b200 as vit
    L = vit.lib
    assert L.vit_init(None, 0, None) == 1
    h = ctypes.c_void_p()
    assert L.vit_init(None, 0, ctypes.byref(h)) == 1 and not h.value
    bad = vit.VitConfig(100, 3, 72, 512, 1e-6, 1e4, vit.BF16, 0)    # 3*72 != 100
    assert L.vit_init(ctypes.byref(bad), 0, ctypes.byref(h)) == 2
    bad = vit.VitConfig(256, 4, 64, 1024, 1e-6, 1e4, vit.BF16, 0)   # d=64 is fp32-only
    assert L.vit_init(ctypes.byref(bad), 0, ctypes.byref(h)) == 3
    bad = vit.VitConfig(1152, 16, 72, 4304, 1e-6, 1e4, 7, 0)        # bad dtype
    assert L.vit_init(ctypes.byref(bad), 0, ctypes.byref(h)) == 1
    L.vit_destroy(None)
    assert L.vit_workspace_bytes(None, 10) == 0
    assert L.vit_layer_forward(None, None, None, None, None, None, 0, None) == 1
    assert L.vit_encoder_forward(None, None, 1, None, None, None, None, 0, None) == 1
    assert L.vit_attention(None, None, None, None, 0.0, None) == 1
    assert L.vit_spatial_merge_2x2(None, None, None, None, 0, 0, None) == 1
    assert L.vit_positions_from_grids(None, None, 0, None, None, None) == 1
    assert L.vit_layernorm(None, None, None, None, None, 0, 0, 0.0, None) == 1
    assert L.vit_linear(None, None, None, None, None, None, 0, 0, 0, 0, None) == 1
    assert L.vit_rope2d(None, None, None, 0, None) == 1
    assert L.vit_get_last_device_status(None) == 1


def test_init_without_device_reports_cuda_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    import vision_transformer_encoder_layernorm_b200 as vit
    cfg = vit.VitConfig(1152, 16, 72, 4304, 1e-6, 1e4, vit.BF16, 0)
    h = ctypes.c_void_p()
    assert vit.lib.vit_init(ctypes.byref(cfg), 0, ctypes.byref(h)) == 5
    assert not h.value


def test_structs_keep_their_tensors_alive():
    # VitSeqs / VitLayerWeights hold raw device pointers: the binding must keep
    # the tensors they point to alive, or a temporary passed to seqs() could be
    # freed and its memory handed to the next allocation
    import gc
    import weakref

    import torch

    import vision_transformer_encoder_layernorm_b200 as vit
    t = torch.zeros(4, dtype=torch.int32)
    ref = weakref.ref(t)
    s = vit.seqs(3, 1, 3, t)
    del t
    gc.collect()
    assert ref() is not None and s.cu_seqlens == ref().data_ptr()
    del s
    gc.collect()
    assert ref() is None
    w = torch.zeros(8)
    wref = weakref.ref(w)
    lw = vit.layer_weights({"w_qkv": w})
    del w
    gc.collect()
    assert wref() is not None and lw.w_qkv == wref().data_ptr() and lw.w_o is None


def test_mx8_sizes_and_null_arguments_without_gpu():
    # MXFP8 buffer sizes: rows of ceil(K/16)*16 code bytes; one 512-byte scale
    # block per (128 rows, 128 columns), each holding 128 rows x 4 groups of 32
    import vision_transformer_encoder_layernorm_b200 as vit
    L = vit.lib
    for K, rb in [(1, 16), (16, 16), (17, 32), (1152, 1152), (4304, 4304), (4305, 4320)]:
        assert vit.mx8_row_bytes(K) == rb
    for rows, K in [(1, 1), (128, 128), (129, 128), (3900, 1152), (4304, 4304), (0, 64)]:
        assert vit.mx8_scale_bytes(rows, K) == -(-rows // 128) * -(-K // 128) * 512
    assert L.vit_mx8_row_bytes(-1) == 0 and L.vit_mx8_scale_bytes(-1, 8) == 0
    assert L.vit_mx8_quantize(None, None, 0, 0, None, None, None) == 1
    assert L.vit_linear_mx8(None, None, None, None, None, None, None, None, 0, 0, 0, 0, None) == 1


def test_mx8_scale_layout_is_a_bijection():
    # the documented block layout (include/vit.h, vit_mx8_quantize) gives every
    # (row, 32-column group) its own byte inside the buffer; what is left over
    # is the padding of the last row block and column block
    import vision_transformer_encoder_layernorm_b200 as vit
    import numpy as np
    for rows, K in [(300, 1152), (130, 4304), (5, 48), (257, 200)]:
        nkb = -(-K // 128)
        r = np.arange(rows)[:, None]
        j = np.arange(-(-K // 32))[None, :]
        off = ((r // 128) * nkb + j // 4) * 512 + (r % 32) * 16 + (r % 128 // 32) * 4 + j % 4
        assert off.min() >= 0 and off.max() < vit.mx8_scale_bytes(rows, K)
        assert np.unique(off).size == off.size
        # a full 128-row x 128-column block uses each of its 512 bytes once
        if rows >= 128 and K >= 128:
            assert np.array_equal(np.sort(off[:128, :4].ravel()), np.arange(512))
