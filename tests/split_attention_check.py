"""Runs one 3900-token layer with the split attention schedule switched on
(VIT_ATTN_SPLIT=1, read once per process) and prints its error metrics
against the fp64 oracle.  Called by tests/test_gpu_layer.py in a child
process."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
os.environ["VIT_ATTN_SPLIT"] = "1"

import torch  # noqa: E402

import synth  # noqa: E402
from oracle import run as orun  # noqa: E402
from tests.gpu_util import context_for, from_dev, layer_dev, metrics, to_dev  # noqa: E402

import vision_transformer_encoder_layernorm_b200 as vit  # noqa: E402

wl = synth.get("c2").with_(layers=1)
inp = synth.make_inputs(wl, layers=1)
ctx = context_for(wl)
T = wl.tokens
cu = torch.empty(2, dtype=torch.int32, device="cuda")
pos = torch.empty((T, 2), dtype=torch.int32, device="cuda")
ctx.positions_from_grids(wl.grids, cu, pos)
sq = vit.seqs(T, 1, T, cu, pos)
x = to_dev(inp.x, wl.dtype)
y = torch.empty_like(x)
ws = torch.empty(ctx.workspace_bytes(T), dtype=torch.uint8, device="cuda")
for _ in range(2):  # the counters must come back to zero between calls
    ctx.layer_forward(layer_dev(inp, 0), x, y, sq, ws)
torch.cuda.synchronize()
rel, cos = metrics(from_dev(y), orun.run_layers(inp))
print(f"{rel} {cos} {ctx.device_status()} {ctx.workspace_bytes(T)}")
