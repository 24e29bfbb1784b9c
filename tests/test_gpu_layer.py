"""Layer- and stack-level parity of the CUDA path against the fp64 oracle on
the seeded workloads, through the C ABI, plus boundary behaviour on a GPU
(errors before any launch, outputs untouched)."""
import numpy as np
import pytest
import torch

import synth
from oracle import run as orun
from oracle import vit_ref as R
from tests.gpu_util import assert_close, context_for, from_dev, int_dev, layer_dev, to_dev

pytestmark = pytest.mark.gpu

vit = pytest.importorskip("vision_transformer_encoder_layernorm_b200")


def _device_run(wl, inputs, n_layers=None, merge=None, fold=False):
    """Runs the workload's stack (and merge) on the GPU; returns fp64 numpy.
    fold: every layer's LayerNorms folded into the projections after them
    (vit_fold_layernorm), the path the benchmark times."""
    ctx = context_for(wl)
    T, C = wl.tokens, wl.hidden
    cu_r, pos_r = R.positions_from_grids(wl.grids)
    cu = torch.empty(len(wl.grids) + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, 2), dtype=torch.int32, device="cuda")
    ctx.positions_from_grids(wl.grids, cu, pos)
    x = to_dev(inputs.x, wl.dtype)
    pkv = None if inputs.prefix_kv is None else to_dev(inputs.prefix_kv, wl.dtype)
    sq = vit.seqs(T, len(wl.grids), int(max(h * w for h, w in wl.grids)), cu,
                  pos if wl.rope else None, pkv, wl.prefix_len, wl.prefix_heads)
    n = len(inputs.layers) if n_layers is None else n_layers
    layers = [layer_dev(inputs, i) for i in range(n)]
    if fold:
        layers = [ctx.fold_layernorm(lw) for lw in layers]
    ws = torch.empty(ctx.workspace_bytes(T), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(x)
    ctx.encoder_forward(layers, x, y, sq, ws)
    out = y
    if merge if merge is not None else wl.merge:
        out = torch.empty((T // 4, 4 * C), dtype=x.dtype, device="cuda")
        ctx.spatial_merge_2x2(y, out, wl.grids, C)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    res = from_dev(out)
    ctx.close()
    return res


_ORACLE = {}  # workload name -> (inputs, oracle output): each stack oracle runs once


def _stack_case(name):
    if name not in _ORACLE:
        wl = synth.get(name)
        inp = synth.make_inputs(wl)
        _ORACLE[name] = (wl, inp, orun.run_workload(inp))
    return _ORACLE[name]


def test_c0_fp32_layer_and_merge():
    wl = synth.get("c0")
    inp = synth.make_inputs(wl)
    got = _device_run(wl, inp)
    ref = orun.run_workload(inp)
    assert got.shape == (64, 1024)
    assert_close(got, ref, 1e-4, None, "c0 fp32")


def test_c1_bf16_layer():
    wl = synth.get("c1")
    inp = synth.make_inputs(wl)
    got = _device_run(wl, inp)
    ref = orun.run_workload(inp)
    assert_close(got, ref, 2e-2, 0.9999, "c1 layer")


def test_small_stack_bf16():
    # 4 layers, two images with ragged tiles, hidden 288 (4 x 72)
    wl = synth.Workload("t", 7, "bf16", 288, 4, 72, 640, 4, ((13, 11), (6, 30)))
    inp = synth.make_inputs(wl)
    got = _device_run(wl, inp)
    ref = orun.run_workload(inp)
    assert_close(got, ref, 5e-2, 0.999, "small stack")


def test_small_stack_d128_prefix_no_mlp():
    wl = synth.Workload("t", 8, "bf16", 256, 2, 128, 0, 2, ((10, 20), (7, 9)),
                        prefix_len=150, kv_heads=1, attn_only=True)
    inp = synth.make_inputs(wl)
    got = _device_run(wl, inp)
    ref = orun.run_workload(inp)
    assert_close(got, ref, 5e-2, 0.999, "attention-only stack")


def test_encoder_one_layer_equals_layer_forward():
    wl = synth.get("c1")
    inp = synth.make_inputs(wl)
    ctx = context_for(wl)
    T = wl.tokens
    cu = int_dev(R.positions_from_grids(wl.grids)[0])
    pos = int_dev(R.positions_from_grids(wl.grids)[1])
    sq = vit.seqs(T, 1, T, cu, pos)
    x = to_dev(inp.x, wl.dtype)
    ws = torch.empty(ctx.workspace_bytes(T), dtype=torch.uint8, device="cuda")
    y1, y2 = torch.empty_like(x), torch.empty_like(x)
    lw = layer_dev(inp, 0)
    ctx.layer_forward(lw, x, y1, sq, ws)
    ctx.encoder_forward([lw], x, y2, sq, ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    ctx.close()


@pytest.mark.slow
@pytest.mark.parametrize("fold", [False, True], ids=["plain", "folded_ln"])
def test_c4_attention_half_layer(fold):
    wl, inp, ref = _stack_case("c4")
    got = _device_run(wl, inp, fold=fold)
    assert_close(got, ref, 2e-2, 0.9999, f"c4 attention half-layer (fold {fold})")


@pytest.mark.slow
def test_c3_first_layer_full_size():
    wl = synth.get("c3")
    inp = synth.make_inputs(wl, layers=1)
    got = _device_run(wl, inp, n_layers=1)
    ref = orun.run_layers(inp, n_layers=1)
    assert_close(got, ref, 2e-2, 0.9999, "c3 layer 0")


# Stack bar (27 layers, each side chaining from the same input): cosine >=
# 0.999, and max|y - r| / max|r| <= STACK_REL.  A cosine of 0.999 bounds the
# relative rms error at sqrt(2 (1 - 0.999)) ~= 0.045; after 27 layers the
# error is spread over every element, so the largest error relative to the
# largest value follows that rms ratio, and the bar allows twice it.
STACK_REL = 0.1


@pytest.mark.slow
@pytest.mark.parametrize("fold", [False, True], ids=["plain", "folded_ln"])
def test_c2_full_stack_and_merge(fold):
    # the headline workload: 27 layers over 3900 tokens, then the 2x2 merge;
    # plain layers, and layers with folded LayerNorms (the benchmark's path)
    wl, inp, ref = _stack_case("c2")
    got = _device_run(wl, inp, fold=fold)
    assert got.shape == (975, 4608)
    rel, cos = assert_close(got, ref, STACK_REL, 0.999, f"c2 27-layer stack + merge (fold {fold})")
    print(f"c2 27-layer stack + merge, fold {fold}: rel {rel:.4e} cos {cos:.7f}")


@pytest.mark.slow
@pytest.mark.parametrize("fold", [False, True], ids=["plain", "folded_ln"])
def test_c3_full_packed_stack(fold):
    # 27 layers over 5 packed images (780 + 888 + 960 + 3900 + 4408 tokens):
    # block-diagonal attention through cu_seqlens, per-image RoPE positions
    # and 27 layers of error growth together
    wl, inp, ref = _stack_case("c3")
    got = _device_run(wl, inp, fold=fold)
    assert got.shape == (10936, 1152)
    rel, cos = assert_close(got, ref, STACK_REL, 0.999, f"c3 27-layer packed stack (fold {fold})")
    print(f"c3 27-layer packed stack, fold {fold}: rel {rel:.4e} cos {cos:.7f}")


@pytest.mark.parametrize("grid", [(50, 78), (60, 65)])
def test_c2_one_layer(grid):
    # one 3900-token layer (the headline's size) against the oracle, on both
    # grids of the workload (the merged image and the encoder-only one)
    wl = synth.get("c2").with_(layers=1, grids=[grid])
    inp = synth.make_inputs(wl, layers=1)
    got = _device_run(wl, inp, merge=False)
    ref = orun.run_layers(inp)
    assert_close(got, ref, 2e-2, 0.9999, f"c2 layer, grid {grid}")


def test_c2_one_layer_split_attention_schedule():
    # the opt-in split schedule (key tiles shared evenly by the SMs, items
    # split between CTAs combined by the last part): a child process, since
    # the switch is read once per process
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    out = subprocess.run([sys.executable, os.path.join(here, "split_attention_check.py")],
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    rel, cos, status, ws = out.stdout.split()[-4:]
    assert int(status) == 0
    assert int(ws) > 20 << 20  # the split's scratch is part of the workspace
    assert float(rel) <= 2e-2 and float(cos) >= 0.9999, (rel, cos)


# ------------------------------------------------------------------ boundary
def test_boundary_errors_launch_nothing():
    wl = synth.get("c1")
    ctx = context_for(wl)
    T, C = wl.tokens, wl.hidden
    cu = int_dev(np.array([0, T]))
    pos = int_dev(R.positions_from_grids(wl.grids)[1])
    x = torch.zeros((T, C), dtype=torch.bfloat16, device="cuda")
    y = torch.full((T, C), 5.0, dtype=torch.bfloat16, device="cuda")
    inp = synth.make_inputs(wl)
    lw = layer_dev(inp, 0)
    need = ctx.workspace_bytes(T)
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    sq = vit.seqs(T, 1, T, cu, pos)
    cases = [
        (lambda: ctx.layer_forward(lw, x, y, sq, small), 4),                      # workspace
        (lambda: ctx.layer_forward(lw, x, x, sq, ws), 1),                         # aliasing
        (lambda: ctx.layer_forward(lw, x, y, vit.seqs(T, 1, T + 1, cu, pos), ws), 2),
        (lambda: ctx.layer_forward(lw, x, y, vit.seqs(T, 1, T, cu, None), ws), 1),  # no pos
        (lambda: ctx.layer_forward(dict(lw, w_o=None), x, y, sq, ws), 1),
        (lambda: ctx.attention(x[:, :3 * 8], y, vit.seqs(T, 1, T, cu, None, x, 4, 3)), 2),
        (lambda: ctx.linear(x[:, :12], x[:12, :12], None, y), 3),               # K % 8
    ]
    for fn, code in cases:
        with pytest.raises(vit.VitError) as e:
            fn()
        assert e.value.code == code
    torch.cuda.synchronize()
    assert torch.all(y == 5.0)
    ctx.close()


def test_unsupported_configs_rejected():
    with pytest.raises(vit.VitError) as e:
        vit.Context(96 * 4, 4, 96, 512, vit.BF16)
    assert e.value.code == 3
    with pytest.raises(vit.VitError) as e:
        vit.Context(256, 4, 64, 1024, vit.BF16)
    assert e.value.code == 3


def test_empty_input_is_a_no_op():
    wl = synth.get("c1")
    ctx = context_for(wl)
    x = torch.zeros((0, wl.hidden), dtype=torch.bfloat16, device="cuda")
    cu = int_dev(np.array([0, 0]))
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    ctx.layer_forward(layer_dev(synth.make_inputs(wl), 0), x, torch.empty_like(x),
                      vit.seqs(0, 1, 0, cu, cu), ws)
    ctx.attention(torch.zeros((0, 3 * wl.hidden), dtype=torch.bfloat16, device="cuda"), x,
                  vit.seqs(0, 1, 0, cu))
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    ctx.close()
