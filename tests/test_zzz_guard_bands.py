"""Out-of-bounds writes, checked without a sanitizer: every output (and
workspace) of every entry point is a view in the middle of a larger buffer
whose margins hold a canary byte pattern.  After the call the margins must be
unchanged, and floating-point outputs, pre-filled with NaN, must hold no NaN
(every element written).  Runs last: these cases repeat shapes of the parity
tests, with ragged tails in every dimension."""
import math

import numpy as np
import pytest
import torch

import synth
from tests.gpu_util import context_for, int_dev, layer_dev, to_dev

pytestmark = pytest.mark.gpu

vit = pytest.importorskip("vision_transformer_encoder_layernorm_b200")

MARGIN = 64 << 10  # bytes of canary on each side
CANARY = 0xA5


class Band:
    """A `shape` x `dtype` view inside a canary-guarded byte buffer."""

    def __init__(self, shape, dtype, device="cuda", poison=True):
        self.n = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
        self.buf = torch.full((2 * MARGIN + self.n,), CANARY, dtype=torch.uint8, device=device)
        self.t = self.buf[MARGIN:MARGIN + self.n].view(dtype).view(shape)
        self.floating = dtype.is_floating_point and poison
        if poison:
            self.t.view(torch.uint8).fill_(0xFF)  # NaN for fp32 / bf16; -1 for integers

    def check(self, what):
        if self.buf.is_cuda:
            torch.cuda.synchronize()
        lo, hi = self.buf[:MARGIN], self.buf[MARGIN + self.n:]
        bad_lo = int((lo != CANARY).sum())
        bad_hi = int((hi != CANARY).sum())
        assert bad_lo == 0 and bad_hi == 0, f"{what}: {bad_lo} bytes before / {bad_hi} after changed"
        if self.floating:
            assert bool(torch.isfinite(self.t.float()).all()), f"{what}: output elements not written"


def _bf16(shape, seed, scale=1.0):
    return to_dev(synth.random_tensor(shape, seed, "bf16", scale), "bf16")


def _f32(shape, seed, scale=1.0):
    return to_dev(synth.random_tensor(shape, seed, "f32", scale), "f32")


@pytest.fixture(scope="module")
def ctx():
    c = vit.Context(1152, 16, 72, 4304, vit.BF16)
    yield c
    c.close()


@pytest.mark.parametrize("M,N,K,epi", [(300, 392, 200, 0), (129, 264, 72, 1), (257, 136, 64, 2),
                                       (3900, 3456, 1152, 0), (3900, 1152, 4304, 2), (1, 8, 8, 1)])
def test_guard_linear_bf16(ctx, M, N, K, epi):
    x, w, b = _bf16((M, K), 1), _bf16((N, K), 2, 0.02), _bf16((N,), 3, 0.01)
    res = _bf16((M, N), 4) if epi == 2 else None
    y = Band((M, N), torch.bfloat16)
    ctx.linear(x, w, b, y.t, epi=epi, residual=res)
    y.check(f"linear {M}x{N}x{K} epi{epi}")
    assert ctx.device_status() == 0


def test_guard_layernorm(ctx):
    x, g, b = _bf16((300, 1152), 5), _bf16((1152,), 6), _bf16((1152,), 7)
    y = Band((300, 1152), torch.bfloat16)
    ctx.layernorm(x, y.t, g, b)
    y.check("layernorm")


@pytest.mark.parametrize("H,d,grids,P,Hkv", [
    (16, 72, [(15, 20), (7, 11)], 0, 0),   # ragged query tiles, two segments, RoPE on load
    (3, 128, [(10, 14), (7, 11)], 130, 3),  # prefix keys
    (3, 72, [(1, 1), (13, 10)], 0, 0),      # a one-token segment
])
def test_guard_attention(H, d, grids, P, Hkv):
    C = H * d
    lens = [r * c for r, c in grids]
    T = sum(lens)
    c = vit.Context(C, H, d, 4 * C, vit.BF16)
    qkv = _bf16((T, 3 * C), 8)
    cu = torch.empty(len(grids) + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, 2), dtype=torch.int32, device="cuda")
    c.positions_from_grids(grids, cu, pos)
    pkv = _bf16((len(grids), 2, P, Hkv, d), 9) if P else None
    o = Band((T, C), torch.bfloat16)
    c.attention(qkv, o.t, vit.seqs(T, len(grids), max(lens), cu, pos, pkv, P, Hkv))
    o.check(f"attention H{H} d{d} {grids} P{P}")
    assert c.device_status() == 0
    c.close()


def test_guard_layer_and_workspace():
    wl = synth.get("c1")
    inp = synth.make_inputs(wl, layers=1)
    c = context_for(wl)
    T = wl.tokens
    x = to_dev(inp.x, "bf16")
    cu = torch.empty(len(wl.grids) + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, 2), dtype=torch.int32, device="cuda")
    c.positions_from_grids(wl.grids, cu, pos)
    sq = vit.seqs(T, len(wl.grids), max(r * q for r, q in wl.grids), cu, pos)
    lw = layer_dev(inp, 0)
    ws = Band((c.workspace_bytes(T),), torch.uint8, poison=False)
    y = Band((T, wl.hidden), torch.bfloat16)
    c.layer_forward(lw, x, y.t, sq, ws.t)
    y.check("layer output")
    ws.check("layer workspace")
    y2 = Band((T, wl.hidden), torch.bfloat16)
    c.encoder_forward([lw, lw], x, y2.t, sq, ws.t)
    y2.check("two-layer encoder output")
    ws.check("encoder workspace")
    assert c.device_status() == 0
    c.close()


def test_guard_folded_layernorm_layer():
    # the fold's outputs, and a folded two-layer stack whose row statistics
    # live in the workspace (written by GEMM epilogues and the row-statistics
    # kernel)
    wl = synth.get("c1")
    inp = synth.make_inputs(wl, layers=1)
    c = context_for(wl)
    T, C, Fm = wl.tokens, wl.hidden, wl.mlp
    lw = layer_dev(inp, 0)
    wq, sq_ = Band((3 * C, C), torch.bfloat16), Band((2, 3 * C), torch.float32)
    w1, s1 = Band((Fm, C), torch.bfloat16), Band((2, Fm), torch.float32)
    import ctypes
    lws = vit.layer_weights(lw)
    assert vit.lib.vit_fold_layernorm(c.handle, ctypes.byref(lws), wq.t.data_ptr(), sq_.t.data_ptr(),
                                      w1.t.data_ptr(), s1.t.data_ptr(), None) == 0
    for band, what in [(wq, "folded w_qkv"), (sq_, "qkv s, c"), (w1, "folded w_fc1"), (s1, "fc1 s, c")]:
        band.check(what)
    f = dict(lw, w_qkv=wq.t, qkv_fold=sq_.t, w_fc1=w1.t, fc1_fold=s1.t, ln1_g=None, ln1_b=None,
             b_qkv=None, ln2_g=None, ln2_b=None, b_fc1=None)
    x = to_dev(inp.x, "bf16")
    cu = torch.empty(len(wl.grids) + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, 2), dtype=torch.int32, device="cuda")
    c.positions_from_grids(wl.grids, cu, pos)
    sq = vit.seqs(T, len(wl.grids), max(r * q for r, q in wl.grids), cu, pos)
    ws = Band((c.workspace_bytes(T),), torch.uint8, poison=False)
    y = Band((T, C), torch.bfloat16)
    c.encoder_forward([f, f], x, y.t, sq, ws.t)
    y.check("folded two-layer encoder output")
    ws.check("folded encoder workspace")
    assert c.device_status() == 0
    c.close()


def test_guard_merge_and_positions(ctx):
    grids = [(26, 30), (24, 36), (2, 2)]
    T = sum(r * q for r, q in grids)
    cu = Band((len(grids) + 1,), torch.int32)
    pos = Band((T, 2), torch.int32)
    ctx.positions_from_grids(grids, cu.t, pos.t)
    cu.check("cu_seqlens")
    pos.check("positions")
    assert int(pos.t.min()) >= 0 and int(cu.t[-1]) == T
    x = _bf16((T, 1152), 10)
    y = Band((T // 4, 4 * 1152), torch.bfloat16)
    ctx.spatial_merge_2x2(x, y.t, grids, 1152)
    y.check("merge")


@pytest.mark.parametrize("M,N,K", [(300, 384, 4304), (129, 136, 200), (3900, 4304, 1152)])
def test_guard_mx8(ctx, M, N, K):
    x, w, b = _bf16((M, K), 11), _bf16((N, K), 12, 0.02), _bf16((N,), 13)
    a = (Band((M, vit.mx8_row_bytes(K)), torch.uint8, poison=False),
         Band((vit.mx8_scale_bytes(M, K),), torch.uint8, poison=False))
    wq = (Band((N, vit.mx8_row_bytes(K)), torch.uint8, poison=False),
          Band((vit.mx8_scale_bytes(N, K),), torch.uint8, poison=False))
    ctx.mx8_quantize(x, a[0].t, a[1].t)
    ctx.mx8_quantize(w, wq[0].t, wq[1].t)
    for band, what in [(a[0], "A codes"), (a[1], "A scales"), (wq[0], "W codes"), (wq[1], "W scales")]:
        band.check(f"mx8 quantize {what} {M}x{K}")
    y = Band((M, N), torch.bfloat16)
    ctx.linear_mx8((a[0].t, a[1].t), (wq[0].t, wq[1].t), b, y.t, K, epi=vit.EPI_BIAS_GELU)
    y.check(f"linear mx8 {M}x{N}x{K}")
    assert ctx.device_status() == 0


def test_guard_embedding():
    grids = [(4, 6), (6, 4), (3, 5)]
    wl = synth.get("c1").with_(grids=grids)
    inp = synth.make_embed_inputs(wl, patch=14)
    c = context_for(wl)
    T = sum(r * q for r, q in grids)
    px = to_dev(np.concatenate([im.reshape(-1) for im in inp.images]), "bf16")
    w, b, t = (to_dev(v, "bf16") for v in (inp.w_pe, inp.b_pe, inp.table))
    ws = Band((c.embed_workspace_bytes(T, 14),), torch.uint8, poison=False)
    y = Band((T, wl.hidden), torch.bfloat16)
    c.patch_embed(px, grids, 14, w, b, t, y.t, ws.t)
    y.check("patch embedding")
    ws.check("embedding workspace")
    y2 = Band((T, wl.hidden), torch.bfloat16)
    c.pos_interp(t, grids, y2.t)
    y2.check("position interpolation")
    assert c.device_status() == 0
    c.close()


def test_guard_fp32_mode():
    c = vit.Context(256, 4, 64, 1024, vit.F32)
    M, N, K = 300, 392, 200
    x, w, b = _f32((M, K), 14), _f32((N, K), 15, 0.02), _f32((N,), 16)
    y = Band((M, N), torch.float32)
    c.linear(x, w, b, y.t, epi=vit.EPI_BIAS_GELU)
    y.check("linear f32")
    lens = [100, 37]
    T = sum(lens)
    qkv = _f32((T, 3 * 256), 17)
    cu = int_dev(np.array([0, 100, 137]))
    o = Band((T, 256), torch.float32)
    c.attention(qkv, o.t, vit.seqs(T, 2, 100, cu))
    o.check("attention f32")
    assert c.device_status() == 0
    c.close()
