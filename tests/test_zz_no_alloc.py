"""vit_layer_forward_noalloc, the layer call for callers that cannot allocate
device memory at call time (its scratch is a fixed array inside libvit).

It is checked against vit_layer_forward with a caller-allocated workspace,
on two calls in a row with different inputs, so that a second call that
picked up the first call's leftovers in the shared scratch would show up.
The file is named to be collected last."""
import os

import numpy as np
import pytest
import torch

import synth
from tests.gpu_util import assert_close, context_for, from_dev, int_dev, layer_dev, to_dev

pytestmark = pytest.mark.gpu

vit = pytest.importorskip("vision_transformer_encoder_layernorm_b200")


def test_noalloc_layer_matches_workspace_layer_twice():
    wl = synth.get("c1")                         # 960 tokens: fits the 32 MiB scratch
    inp = synth.make_inputs(wl)
    ctx = context_for(wl)
    T, C = wl.tokens, wl.hidden
    from oracle import run as orun
    from oracle import vit_ref as R
    cu_r, pos_r = R.positions_from_grids(wl.grids)
    sq = vit.seqs(T, 1, T, int_dev(cu_r), int_dev(pos_r))
    lw = layer_dev(inp, 0)
    ws = torch.empty(ctx.workspace_bytes(T), dtype=torch.uint8, device="cuda")
    x_b = synth.random_tensor((T, C), 123, wl.dtype)
    # Both calls launch the same kernels in the same order on the same
    # inputs (the workspace call takes the split attention schedule only when
    # VIT_ATTN_SPLIT is set), so the outputs agree bit for bit: a call that
    # read a stale value left in the shared scratch by the call before it
    # would differ.
    exact = not os.environ.get("VIT_ATTN_SPLIT")
    for xh in (inp.x, x_b):                      # two calls in a row
        x = to_dev(xh, wl.dtype)
        ref = torch.empty_like(x)
        got = torch.full_like(x, float("nan"))
        ctx.layer_forward(lw, x, ref, sq, ws)
        ctx.layer_forward_noalloc(lw, x, got, sq)
        torch.cuda.synchronize()
        if exact:
            assert torch.equal(got, ref), "noalloc output differs from the workspace call"
        else:
            assert_close(from_dev(got), from_dev(ref), 2e-2, 0.9999, "noalloc vs workspace layer")
        # and against the fp64 oracle at the per-layer bar
        want = orun.run_layers(inp, x=synth.to_f64(xh, wl.dtype), n_layers=1)
        assert_close(from_dev(got), want, 2e-2, 0.9999, "noalloc layer vs oracle")
    assert ctx.device_status() == 0
    ctx.close()


def test_noalloc_rejects_more_tokens_than_the_scratch_holds():
    wl = synth.get("c2")                         # 3900 tokens need 96 MB of scratch
    ctx = context_for(wl)
    T, C = wl.tokens, wl.hidden
    assert ctx.workspace_bytes(T) > 32 << 20
    x = torch.zeros((T, C), dtype=torch.bfloat16, device="cuda")
    y = torch.full((T, C), 5.0, dtype=torch.bfloat16, device="cuda")
    lw = layer_dev(synth.make_inputs(wl, layers=1), 0)
    cu = int_dev(np.array([0, T]))
    pos = torch.zeros((T, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(vit.VitError) as e:
        ctx.layer_forward_noalloc(lw, x, y, vit.seqs(T, 1, T, cu, pos))
    assert e.value.code == 4                     # VIT_ERR_WORKSPACE, nothing launched
    torch.cuda.synchronize()
    assert torch.all(y == 5.0)
    ctx.close()
