"""The projector composition after the 2x2 merge (vit_projector: LayerNorm,
linear + GELU, linear) against the fp64 oracle, vit_ref.projector, on a
GPU through the C ABI.  Widths are test choices (the pages give none): the
merged c2 tokens (975 x 4608) to a 1024-wide output, ragged small widths,
and the fp32 mode."""
import numpy as np
import pytest
import torch

import synth
from oracle import vit_ref as R
from tests.gpu_util import assert_close, from_dev, to_dev

pytestmark = pytest.mark.gpu

vit = pytest.importorskip("vision_transformer_encoder_layernorm_b200")


def _case(dt, M, d_in, d_hid, d_out, seed):
    ctx = (vit.Context(1152, 16, 72, 4304, vit.BF16) if dt == "bf16"
           else vit.Context(256, 4, 64, 1024, vit.F32))
    w = synth.make_projector_weights(d_in, d_hid, d_out, seed, dt)
    xh = synth.random_tensor((M, d_in), seed + 1, dt)
    wd = {k: to_dev(v, dt) for k, v in w.items()}
    x = to_dev(xh, dt)
    y = torch.full((M, d_out), float("nan"), dtype=x.dtype, device="cuda")
    ws = torch.empty(ctx.projector_workspace_bytes(M, d_in, d_hid), dtype=torch.uint8,
                     device="cuda")
    ctx.projector(wd, x, y, ws)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    ref = R.projector(synth.to_f64(xh, dt), {k: synth.to_f64(v, dt) for k, v in w.items()})
    ctx.close()
    return from_dev(y), ref


@pytest.mark.parametrize("M,d_in,d_hid,d_out", [(975, 4608, 4608, 1024), (37, 192, 136, 72),
                                                (300, 4608, 1024, 2048)])
def test_projector_bf16(M, d_in, d_hid, d_out):
    got, ref = _case("bf16", M, d_in, d_hid, d_out, 90)
    # the chain of an MLP half-layer: LN and GELU outputs rounded to bf16 once
    assert_close(got, ref, 2e-2, 0.9999, f"projector {M}x{d_in}->{d_hid}->{d_out}")


def test_projector_f32():
    got, ref = _case("f32", 50, 1024, 512, 256, 91)
    assert_close(got, ref, 1e-4, None, "projector fp32")


def test_projector_errors():
    ctx = vit.Context(1152, 16, 72, 4304, vit.BF16)
    w = {k: to_dev(v, "bf16") for k, v in synth.make_projector_weights(64, 32, 16, 3, "bf16").items()}
    x = to_dev(synth.random_tensor((10, 64), 4, "bf16"), "bf16")
    y = torch.full((10, 16), 7.0, dtype=torch.bfloat16, device="cuda")
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(vit.VitError) as e:
        ctx.projector(w, x, y, small)
    assert e.value.code == 4  # VIT_ERR_WORKSPACE
    w_odd = dict(w, w1=to_dev(synth.random_tensor((36, 64), 5, "bf16"), "bf16"))
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(vit.VitError) as e:
        ctx.projector(dict(w_odd, w2=torch.zeros((16, 36), dtype=torch.bfloat16, device="cuda")),
                      x, y, ws)
    assert e.value.code == 3  # d_hidden % 8: VIT_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)
    ctx.close()
