"""CUDA-graph capture of library calls (vit_graph_begin/end/launch): a
replayed stack + merge equals the direct calls bit for bit, sees refilled
inputs, and capture misuse is rejected."""
import numpy as np
import pytest
import torch

import synth
from tests.gpu_util import context_for, layer_dev, to_dev

pytestmark = pytest.mark.gpu

vit = pytest.importorskip("vision_transformer_encoder_layernorm_b200")


def _setup(n_layers=3):
    wl = synth.get("c1")
    inp = synth.make_inputs(wl)
    ctx = context_for(wl)
    T, C = wl.tokens, wl.hidden
    cu = torch.empty(len(wl.grids) + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, 2), dtype=torch.int32, device="cuda")
    ctx.positions_from_grids(wl.grids, cu, pos)
    sq = vit.seqs(T, len(wl.grids), int(max(h * w for h, w in wl.grids)), cu, pos)
    layers = [layer_dev(inp, 0) for _ in range(n_layers)]
    x = to_dev(inp.x, wl.dtype)
    ws = torch.empty(ctx.workspace_bytes(T), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(x)
    out = torch.empty((T // 4, 4 * C), dtype=x.dtype, device="cuda")
    return wl, ctx, sq, layers, x, ws, y, out


def test_graph_replay_equals_direct_calls():
    wl, ctx, sq, layers, x, ws, y, out = _setup()
    T, C = wl.tokens, wl.hidden
    ctx.profile_read(reset=True)  # count only the launches below
    ctx.encoder_forward(layers, x, y, sq, ws)
    ctx.spatial_merge_2x2(y, out, wl.grids, C)
    torch.cuda.synchronize()
    direct = out.clone()
    before = sum(n for n, _ in ctx.profile_read(reset=True).values())
    assert before > 0

    cs = ctx.graph_begin()
    ctx.encoder_forward(layers, x, y, sq, ws, stream=cs)
    ctx.spatial_merge_2x2(y, out, wl.grids, C, stream=cs)
    g = ctx.graph_end()
    assert g.kernels == before  # the same launches, recorded once
    out.zero_()
    y.zero_()
    g.launch()
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    assert torch.equal(out, direct)

    # refilled input: the replay reads the same buffer
    x2 = torch.randn_like(x.float()).to(x.dtype)
    x.copy_(x2)
    g.launch()
    torch.cuda.synchronize()
    replay2 = out.clone()
    ctx.encoder_forward(layers, x, y, sq, ws)
    ctx.spatial_merge_2x2(y, out, wl.grids, C)
    torch.cuda.synchronize()
    assert torch.equal(replay2, out)
    assert not torch.equal(replay2, direct)
    g.close()
    ctx.close()


def test_graph_capture_misuse():
    wl, ctx, sq, layers, x, ws, y, out = _setup(1)
    with pytest.raises(vit.VitError):
        ctx.graph_end()  # no capture in progress
    cs = ctx.graph_begin()
    with pytest.raises(vit.VitError):
        ctx.graph_begin()  # one capture at a time
    # an invalid call inside the capture is rejected before any launch and
    # leaves the capture usable
    with pytest.raises(vit.VitError):
        ctx.encoder_forward(layers, x, y, sq, ws[:16], stream=cs)
    ctx.encoder_forward(layers, x, y, sq, ws, stream=cs)
    g = ctx.graph_end()
    assert g.kernels > 0
    g.launch()
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    g.close()
    ctx.close()
