"""Patch embedding and bilinear position-table interpolation on the GPU
against the fp64 oracle (oracle/embed_ref.py), through the C ABI."""
import numpy as np
import pytest
import torch

import synth
from oracle import embed_ref as E
from tests.gpu_util import assert_close, context_for, from_dev, to_dev

pytestmark = pytest.mark.gpu

vit = pytest.importorskip("vision_transformer_encoder_layernorm_b200")

# bf16: tokens are rounded once (2^-9 relative); the GEMM's bar as elsewhere
TOL = {"bf16": (1e-2, 0.99999), "f32": (1e-5, None)}
TOL_INTERP = {"bf16": (4e-3, 0.99999), "f32": (1e-6, None)}


def _pixels(inp, dt):
    return to_dev(np.concatenate([im.reshape(-1) for im in inp.images]), dt)


@pytest.mark.parametrize("name,grids,table", [
    ("c1", [(50, 78)], (27, 27)), ("c1", [(4, 6), (6, 4), (1, 1)], (27, 27)),
    ("c1", [(30, 32), (27, 27)], (16, 20)), ("c0", [(16, 16), (3, 5)], (7, 9))])
def test_pos_interp(name, grids, table):
    wl = synth.get(name).with_(grids=grids)
    inp = synth.make_embed_inputs(wl, patch=2, table_hw=table)
    ctx = context_for(wl)
    T = sum(r * c for r, c in grids)
    y = torch.full((T, wl.hidden), 7.0, device="cuda").to(torch.bfloat16 if wl.dtype == "bf16" else torch.float32)
    ctx.pos_interp(to_dev(inp.table, wl.dtype), grids, y)
    torch.cuda.synchronize()
    t64 = synth.to_f64(inp.table, wl.dtype)
    ref = np.concatenate([E.bilinear_resize(t64, r, c).reshape(r * c, -1) for r, c in grids])
    assert_close(from_dev(y), ref, *TOL_INTERP[wl.dtype], f"interp {name} {grids}")
    ctx.close()


@pytest.mark.parametrize("name,grids,patch", [
    ("c1", [(4, 6), (6, 4), (2, 2)], 14), ("c1", [(50, 78)], 14), ("c1", [(3, 5)], 16),
    ("c0", [(4, 4), (2, 6)], 4), ("c0", [(5, 3)], 7)])
def test_patch_embed(name, grids, patch):
    wl = synth.get(name).with_(grids=grids)
    inp = synth.make_embed_inputs(wl, patch=patch)
    ctx = context_for(wl)
    T = sum(r * c for r, c in grids)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    y = torch.empty((T, wl.hidden), dtype=dt, device="cuda")
    ws = torch.empty(ctx.embed_workspace_bytes(T, patch), dtype=torch.uint8, device="cuda")
    ctx.patch_embed(_pixels(inp, wl.dtype), grids, patch, to_dev(inp.w_pe, wl.dtype),
                    to_dev(inp.b_pe, wl.dtype), to_dev(inp.table, wl.dtype), y, ws)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    f = lambda a: synth.to_f64(a, wl.dtype)
    ref = E.embed_images([f(im) for im in inp.images], grids, patch, f(inp.w_pe), f(inp.b_pe),
                         f(inp.table))
    assert_close(from_dev(y), ref, *TOL[wl.dtype], f"embed {name} {grids} p{patch}")
    ctx.close()


def test_patch_embed_errors_leave_output_untouched():
    wl = synth.get("c1").with_(grids=[(2, 2)])
    inp = synth.make_embed_inputs(wl, patch=14)
    ctx = context_for(wl)
    px = _pixels(inp, "bf16")
    w, b, t = (to_dev(a, "bf16") for a in (inp.w_pe, inp.b_pe, inp.table))
    y = torch.full((4, wl.hidden), 3.0, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(ctx.embed_workspace_bytes(4, 14), dtype=torch.uint8, device="cuda")
    cases = [(dict(patch=0), 1), (dict(grids=[(2, 0)]), 2), (dict(ws=ws[:64]), 4),
             (dict(grids=[]), 1), (dict(patch=33), 1)]
    for kw, code in cases:
        a = dict(pixels=px, grids=[(2, 2)], patch=14, w_pe=w, b_pe=b, pos_table=t, y=y, workspace=ws)
        if "ws" in kw:
            a["workspace"] = kw.pop("ws")
        a.update(kw)
        with pytest.raises(vit.VitError) as ei:
            ctx.patch_embed(**a)
        assert ei.value.code == code, kw
    torch.cuda.synchronize()
    assert bool((y == 3.0).all())
    ctx.close()


@pytest.mark.parametrize("name,grids,patch,px_offset", [
    ("c1", [(50, 78)], 14, 0), ("c1", [(4, 6), (6, 4), (2, 2)], 14, 1), ("c1", [(3, 5)], 16, 0),
    ("c0", [(5, 3)], 7, 0), ("c0", [(4, 4), (2, 6)], 4, 0)])
def test_patch_embed_padded_weight(name, grids, patch, px_offset):
    """The weight padded once (vit_pad_patch_weight) and the padded entry give
    the same tokens as vit_patch_embed, bit for bit, and match the oracle;
    px_offset = 1 starts the pixels off a four-byte boundary (element path)."""
    wl = synth.get(name).with_(grids=grids)
    inp = synth.make_embed_inputs(wl, patch=patch)
    ctx = context_for(wl)
    T = sum(r * c for r, c in grids)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    flat = _pixels(inp, wl.dtype)
    px = torch.empty(flat.numel() + px_offset, dtype=flat.dtype, device="cuda")[px_offset:]
    px.copy_(flat)
    w = to_dev(inp.w_pe, wl.dtype)
    b, t = to_dev(inp.b_pe, wl.dtype), to_dev(inp.table, wl.dtype)
    w_pad = ctx.pad_patch_weight(w, patch)
    kp = vit.lib.vit_patch_kp(patch)
    assert w_pad.shape == (wl.hidden, kp) and kp % 8 == 0 and kp >= 3 * patch * patch
    assert torch.equal(w_pad[:, :3 * patch * patch], w) and not w_pad[:, 3 * patch * patch:].any()
    ws = torch.empty(ctx.embed_workspace_bytes(T, patch), dtype=torch.uint8, device="cuda")
    y0 = torch.empty((T, wl.hidden), dtype=dt, device="cuda")
    y1 = torch.empty_like(y0)
    ctx.patch_embed(px, grids, patch, w, b, t, y0, ws)
    ctx.patch_embed_padded(px, grids, patch, w_pad, b, t, y1, ws)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    assert torch.equal(y0, y1)
    f = lambda a: synth.to_f64(a, wl.dtype)
    ref = E.embed_images([f(im) for im in inp.images], grids, patch, f(inp.w_pe), f(inp.b_pe),
                         f(inp.table))
    assert_close(from_dev(y1), ref, *TOL[wl.dtype], f"embed padded {name} {grids} p{patch}")
    ctx.close()
