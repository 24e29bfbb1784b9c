"""The FP8 encoder layer (vit_encoder_forward_mx8: the four projections in
MXFP8, the rest as the bf16 layer) against the fp64 oracle of the same
layer, oracle/mxfp8_ref.layer_forward_mx8, on a GPU through the C ABI.

Bars (stated in the design notes, reading on the FP8 layer's tolerance): the
GPU quantises its own bf16 intermediates (LayerNorm output, attention output,
GELU output), the oracle the exact fp64 values, so an element lying within
bf16 rounding (2^-9 relative) of an E4M3 rounding midpoint can land one E4M3
step (up to 2^-3 relative) apart; about 2^-5 of the activations can flip,
which bounds the layer's deviation from the MXFP8 oracle at max-rel <= 5e-2,
cosine >= 0.9995.  Against the unquantised fp64 layer the quantisation itself
is the error: cosine >= 0.995 (the MXFP8 GEMM bar)."""
import numpy as np
import pytest
import torch

import synth
from oracle import mxfp8_ref as MX
from oracle import run as orun
from oracle import vit_ref as R
from tests.gpu_util import assert_close, context_for, from_dev, layer_dev, to_dev

pytestmark = pytest.mark.gpu

vit = pytest.importorskip("vision_transformer_encoder_layernorm_b200")


def _gpu_mx8(wl, inp, n_layers=None):
    ctx = context_for(wl)
    T = wl.tokens
    n = len(inp.layers) if n_layers is None else n_layers
    layers = [ctx.quantize_layer_mx8(layer_dev(inp, i)) for i in range(n)]
    cu = torch.empty(len(wl.grids) + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, 2), dtype=torch.int32, device="cuda")
    ctx.positions_from_grids(wl.grids, cu, pos)
    sq = vit.seqs(T, len(wl.grids), int(max(h * w for h, w in wl.grids)), cu,
                  pos if wl.rope else None)
    x = to_dev(inp.x, wl.dtype)
    y = torch.full_like(x, float("nan"))
    ws = torch.empty(ctx.workspace_bytes_mx8(T), dtype=torch.uint8, device="cuda")
    ctx.encoder_forward_mx8(layers, x, y, sq, ws)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    out = from_dev(y)
    ctx.close()
    return out


def _oracle_mx8(wl, inp, n_layers=None):
    cu, pos = R.positions_from_grids(wl.grids)
    y = synth.to_f64(inp.x, wl.dtype)
    n = len(inp.layers) if n_layers is None else n_layers
    for i in range(n):
        y = MX.layer_forward_mx8(y, orun.layer_f64(inp, i), cu, pos if wl.rope else None,
                                 wl.heads, wl.head_dim, wl.ln_eps, wl.rope_theta)
    return y


def test_c1_fp8_layer_vs_mx8_oracle():
    wl = synth.get("c1")
    inp = synth.make_inputs(wl)
    got = _gpu_mx8(wl, inp)
    rel, cos = assert_close(got, _oracle_mx8(wl, inp), 5e-2, 0.9995, "c1 FP8 layer vs MXFP8 oracle")
    print(f"c1 FP8 layer vs MXFP8 oracle: rel {rel:.3e} cos {cos:.7f}")
    rel2, cos2 = assert_close(got, orun.run_layers(inp), 0.15, 0.995, "c1 FP8 layer vs fp64 layer")
    print(f"c1 FP8 layer vs fp64 layer: rel {rel2:.3e} cos {cos2:.7f}")


def test_small_fp8_stack_vs_mx8_oracle():
    # 3 layers, two images with ragged tiles, hidden 288 (4 x 72)
    wl = synth.Workload("t", 17, "bf16", 288, 4, 72, 640, 3, ((13, 11), (6, 30)))
    inp = synth.make_inputs(wl)
    got = _gpu_mx8(wl, inp)
    rel, cos = assert_close(got, _oracle_mx8(wl, inp), 5e-2, 0.9995, "small FP8 stack")
    print(f"small FP8 stack vs MXFP8 oracle: rel {rel:.3e} cos {cos:.7f}")


def test_c2_fp8_layer_vs_mx8_oracle():
    wl = synth.get("c2").with_(layers=1, merge=False)
    inp = synth.make_inputs(wl, layers=1)
    got = _gpu_mx8(wl, inp)
    rel, cos = assert_close(got, _oracle_mx8(wl, inp), 5e-2, 0.9995, "3900-token FP8 layer")
    print(f"3900-token FP8 layer vs MXFP8 oracle: rel {rel:.3e} cos {cos:.7f}")


def test_fp8_layer_errors():
    wl = synth.get("c1")
    ctx = context_for(wl)
    T, C = wl.tokens, wl.hidden
    lw = ctx.quantize_layer_mx8(layer_dev(synth.make_inputs(wl), 0))
    cu = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    pos = torch.zeros((T, 2), dtype=torch.int32, device="cuda")
    x = torch.zeros((T, C), dtype=torch.bfloat16, device="cuda")
    y = torch.full((T, C), 3.0, dtype=torch.bfloat16, device="cuda")
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(vit.VitError) as e:
        ctx.encoder_forward_mx8([lw], x, y, vit.seqs(T, 1, T, cu, pos), small)
    assert e.value.code == 4
    ws = torch.empty(ctx.workspace_bytes_mx8(T), dtype=torch.uint8, device="cuda")
    with pytest.raises(vit.VitError) as e:
        ctx.encoder_forward_mx8([dict(lw, w_o_codes=None)], x, y, vit.seqs(T, 1, T, cu, pos), ws)
    assert e.value.code == 1
    torch.cuda.synchronize()
    assert torch.all(y == 3.0)
    ctx.close()
    c32 = vit.Context(256, 4, 64, 1024, vit.F32)
    assert c32.workspace_bytes_mx8(100) == 0
    c32.close()
