"""The LayerNorm folded into the projection after it (vit_fold_layernorm and
the layer path that uses it), on a GPU, through the C ABI.

* The fold's outputs against their definitions, computed here in fp64 from
  the same bf16 inputs: W' = W diag(gamma) rounded once to bf16 (bit for
  bit: a product of two bf16 values is exact in fp32), s = row sums of W',
  c = b + W beta.
* Folded layers and stacks against the fp64 oracle (which runs the
  LayerNorm, then the projection) at the same bars as the plain path:
  per layer max-rel <= 2e-2 and cosine >= 0.9999; small ragged stacks at the
  bars of their plain counterparts.
* Mixed stacks (only the first LayerNorm folded, only the second, neither)
  so every hand-over of row statistics between layers is exercised.
* A graph replay of a folded stack equals its direct calls bit for bit."""
import numpy as np
import pytest
import torch

import synth
from oracle import run as orun
from oracle import vit_ref as R
from tests.gpu_util import assert_close, context_for, from_dev, int_dev, layer_dev, to_dev

pytestmark = pytest.mark.gpu

vit = pytest.importorskip("vision_transformer_encoder_layernorm_b200")


def _seqs(ctx, wl):
    T = wl.tokens
    cu = torch.empty(len(wl.grids) + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, 2), dtype=torch.int32, device="cuda")
    ctx.positions_from_grids(wl.grids, cu, pos)
    return vit.seqs(T, len(wl.grids), int(max(h * w for h, w in wl.grids)), cu,
                    pos if wl.rope else None)


def test_fold_outputs_match_their_definition():
    wl = synth.get("c1")
    inp = synth.make_inputs(wl)
    ctx = context_for(wl)
    lw = layer_dev(inp, 0)
    f = ctx.fold_layernorm(lw)
    torch.cuda.synchronize()
    for w, g, be, b, wf, sc in [("w_qkv", "ln1_g", "ln1_b", "b_qkv", "w_qkv", "qkv_fold"),
                                ("w_fc1", "ln2_g", "ln2_b", "b_fc1", "w_fc1", "fc1_fold")]:
        W = lw[w].float()
        want = (W * lw[g].float()[None, :]).to(torch.bfloat16)
        assert torch.equal(f[wf], want), f"{wf}: folded weight differs"
        s_ref = want.double().sum(dim=1)
        c_ref = lw[b].double() + lw[w].double() @ lw[be].double()
        got = f[sc].double()
        assert got.shape == (2, W.shape[0])
        assert float((got[0] - s_ref).abs().max()) <= 1e-5 * float(s_ref.abs().max()) + 1e-6
        assert float((got[1] - c_ref).abs().max()) <= 1e-5 * float(c_ref.abs().max()) + 1e-6
    # in place: the same values, written over the given weights
    lw2 = {k: (v.clone() if v is not None else None) for k, v in lw.items()}
    f2 = ctx.fold_layernorm(lw2, in_place=True)
    torch.cuda.synchronize()
    assert f2["w_qkv"].data_ptr() == lw2["w_qkv"].data_ptr()
    assert torch.equal(f2["w_qkv"], f["w_qkv"]) and torch.equal(f2["w_fc1"], f["w_fc1"])
    assert torch.equal(f2["qkv_fold"], f["qkv_fold"]) and torch.equal(f2["fc1_fold"], f["fc1_fold"])
    ctx.close()


def _run(wl, inp, fold_pattern, n_layers=None):
    """Stack on the GPU with layer i's LayerNorms folded per fold_pattern[i]
    = (qkv, fc1); returns fp64 numpy."""
    ctx = context_for(wl)
    T = wl.tokens
    sq = _seqs(ctx, wl)
    n = len(inp.layers) if n_layers is None else n_layers
    layers = []
    for i in range(n):
        lw = layer_dev(inp, i)
        fq, f1 = fold_pattern[i % len(fold_pattern)]
        if fq or f1:
            full = ctx.fold_layernorm(lw)
            if fq:
                for k in ("w_qkv", "qkv_fold", "ln1_g", "ln1_b", "b_qkv"):
                    lw[k] = full[k]
            if f1 and not wl.attn_only:
                for k in ("w_fc1", "fc1_fold", "ln2_g", "ln2_b", "b_fc1"):
                    lw[k] = full[k]
        layers.append(lw)
    x = to_dev(inp.x, wl.dtype)
    pkv = None if inp.prefix_kv is None else to_dev(inp.prefix_kv, wl.dtype)
    if pkv is not None:
        sq = vit.seqs(T, len(wl.grids), int(max(h * w for h, w in wl.grids)), sq._tensors[0],
                      sq._tensors[1], pkv, wl.prefix_len, wl.prefix_heads)
    ws = torch.empty(ctx.workspace_bytes(T), dtype=torch.uint8, device="cuda")
    y = torch.full_like(x, float("nan"))
    ctx.encoder_forward(layers, x, y, sq, ws)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    out = from_dev(y)
    ctx.close()
    return out


def test_c1_folded_layer_vs_oracle():
    wl = synth.get("c1")
    inp = synth.make_inputs(wl)
    got = _run(wl, inp, [(True, True)])
    assert_close(got, orun.run_layers(inp), 2e-2, 0.9999, "c1 folded layer")


@pytest.mark.parametrize("grid", [(50, 78)])
def test_c2_folded_layer_vs_oracle(grid):
    wl = synth.get("c2").with_(layers=1, grids=[grid], merge=False)
    inp = synth.make_inputs(wl, layers=1)
    got = _run(wl, inp, [(True, True)])
    assert_close(got, orun.run_layers(inp), 2e-2, 0.9999, "3900-token folded layer")


@pytest.mark.parametrize("pattern", [
    [(True, True)],                                              # every LayerNorm folded
    [(True, True), (True, False), (False, True), (False, False)],  # every hand-over
])
def test_small_folded_stack_vs_oracle(pattern):
    # 4 layers, two images with ragged tiles, hidden 288 (4 x 72)
    wl = synth.Workload("t", 7, "bf16", 288, 4, 72, 640, 4, ((13, 11), (6, 30)))
    inp = synth.make_inputs(wl)
    got = _run(wl, inp, pattern)
    assert_close(got, orun.run_layers(inp), 5e-2, 0.999, f"small folded stack {pattern}")


def test_small_folded_attention_only_stack_vs_oracle():
    wl = synth.Workload("t", 8, "bf16", 256, 2, 128, 0, 2, ((10, 20), (7, 9)),
                        prefix_len=150, kv_heads=1, attn_only=True)
    inp = synth.make_inputs(wl)
    got = _run(wl, inp, [(True, False)])
    assert_close(got, orun.run_layers(inp), 5e-2, 0.999, "folded attention-only stack")


def test_folded_stack_graph_replay_equals_direct_calls():
    wl = synth.Workload("t", 9, "bf16", 288, 4, 72, 640, 3, ((13, 11), (6, 30)))
    inp = synth.make_inputs(wl)
    ctx = context_for(wl)
    T = wl.tokens
    sq = _seqs(ctx, wl)
    layers = [ctx.fold_layernorm(layer_dev(inp, i)) for i in range(wl.layers)]
    x = to_dev(inp.x, wl.dtype)
    ws = torch.empty(ctx.workspace_bytes(T), dtype=torch.uint8, device="cuda")
    y1, y2 = torch.empty_like(x), torch.empty_like(x)
    ctx.encoder_forward(layers, x, y1, sq, ws)
    cs = ctx.graph_begin()
    ctx.encoder_forward(layers, x, y2, sq, ws, stream=cs)
    g = ctx.graph_end()
    g.launch()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    g.close()
    ctx.close()


def test_fold_argument_errors():
    wl = synth.get("c1")
    ctx = context_for(wl)
    lw = layer_dev(synth.make_inputs(wl), 0)
    lws = vit.layer_weights(lw)
    import ctypes
    L = vit.lib
    out = torch.empty_like(lw["w_qkv"])
    sc = torch.empty((2, lw["w_qkv"].shape[0]), dtype=torch.float32, device="cuda")
    # a weight without its vectors, or vectors without a weight
    assert L.vit_fold_layernorm(ctx.handle, ctypes.byref(lws), out.data_ptr(), None, None, None,
                                None) == 1
    assert L.vit_fold_layernorm(ctx.handle, ctypes.byref(lws), None, sc.data_ptr(), None, None,
                                None) == 1
    # nothing asked: a no-op
    assert L.vit_fold_layernorm(ctx.handle, ctypes.byref(lws), None, None, None, None, None) == 0
    ctx.close()
    # fp32 contexts have no folded path
    c32 = vit.Context(256, 4, 64, 1024, vit.F32)
    w32 = {k: torch.zeros(4, dtype=torch.float32, device="cuda") for k in ("ln1_g", "ln1_b", "b_qkv")}
    w32["w_qkv"] = torch.zeros((768, 256), dtype=torch.float32, device="cuda")
    assert L.vit_fold_layernorm(c32.handle, ctypes.byref(vit.layer_weights(w32)),
                                out.data_ptr(), sc.data_ptr(), None, None, None) == 3
    c32.close()
