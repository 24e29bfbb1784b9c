"""Step-level parity of the CUDA kernels against the fp64 oracle, through the
C ABI.  Sizes span several tiles and ragged tails; merge and positions are
compared bit-exactly."""
import numpy as np
import pytest
import torch

import synth
from oracle import vit_ref as R
from tests.gpu_util import assert_close, from_dev, int_dev, to_dev

pytestmark = pytest.mark.gpu

vit = pytest.importorskip("vision_transformer_encoder_layernorm_b200")


@pytest.fixture(scope="module")
def ctx_bf16():
    c = vit.Context(1152, 16, 72, 4304, vit.BF16)
    yield c
    c.close()


@pytest.fixture(scope="module")
def ctx_f32():
    c = vit.Context(256, 4, 64, 1024, vit.F32)
    yield c
    c.close()


def _t(shape, seed, dtype, scale=1.0):
    a = synth.random_tensor(shape, seed, dtype, scale)
    return a, to_dev(a, dtype), synth.to_f64(a, dtype)


# ------------------------------------------------------------------ GEMM
GEMM_CASES = [
    # (M, N, K) -- ragged in every dimension, then the encoder's shapes
    (300, 392, 200), (1, 8, 8), (129, 264, 72), (3900, 3456, 1152), (3900, 1152, 4304),
    (960, 4304, 1152), (4096, 9216, 3072),
]


@pytest.mark.parametrize("M,N,K", GEMM_CASES)
@pytest.mark.parametrize("epi", [0, 1, 2])
def test_linear_bf16(ctx_bf16, M, N, K, epi):
    if M * N * K > 4e10 and epi != 0:
        pytest.skip("large shape covered with the bias epilogue")
    _, x, xr = _t((M, K), 1, "bf16")
    _, w, wr = _t((N, K), 2, "bf16", 0.02)
    _, b, br = _t((N,), 3, "bf16", 0.01)
    _, res, rr = _t((M, N), 4, "bf16")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ctx_bf16.linear(x, w, b, y, epi=epi, residual=res if epi == 2 else None)
    torch.cuda.synchronize()
    # every output row is an independent dot-product set: large shapes are
    # checked on sampled rows (first and last tile rows included)
    rows = np.arange(M)
    if M > 1024:
        g = np.random.Generator(np.random.PCG64(M + N))
        rows = np.unique(np.concatenate([g.choice(M, 256, replace=False),
                                         [0, 127, 128, M - 129, M - 1]]))
    ref = R.linear(xr[rows], wr, br)
    if epi == 1:
        ref = R.gelu_tanh(ref)
    if epi == 2:
        ref = ref + rr[rows]
    assert_close(from_dev(y)[rows], ref, 1e-2, 0.99999, f"linear bf16 {M}x{N}x{K} epi{epi}")
    assert ctx_bf16.device_status() == 0


def test_linear_bf16_no_bias(ctx_bf16):
    _, x, xr = _t((200, 136), 5, "bf16")
    _, w, wr = _t((264, 136), 6, "bf16", 0.02)
    y = torch.empty((200, 264), dtype=torch.bfloat16, device="cuda")
    ctx_bf16.linear(x, w, None, y)
    torch.cuda.synchronize()
    assert_close(from_dev(y), R.linear(xr, wr), 1e-2, 0.99999, "linear no bias")


@pytest.mark.parametrize("epi", [0, 1, 2])
def test_linear_f32(ctx_f32, epi):
    M, N, K = 300, 392, 200
    _, x, xr = _t((M, K), 7, "f32")
    _, w, wr = _t((N, K), 8, "f32", 0.02)
    _, b, br = _t((N,), 9, "f32", 0.01)
    _, res, rr = _t((M, N), 10, "f32")
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    ctx_f32.linear(x, w, b, y, epi=epi, residual=res if epi == 2 else None)
    torch.cuda.synchronize()
    ref = R.linear(xr, wr, br)
    if epi == 1:
        ref = R.gelu_tanh(ref)
    if epi == 2:
        ref = ref + rr
    assert_close(from_dev(y), ref, 2e-6, None, f"linear f32 epi{epi}")


# ------------------------------------------------------------------ LayerNorm
@pytest.mark.parametrize("rows,cols,dt", [(1000, 1152, "bf16"), (77, 3072, "bf16"),
                                          (300, 256, "f32"), (5, 4096, "f32"),
                                          # rows wider than a warp holds: a block per row
                                          (975, 4608, "bf16"), (3, 16384, "f32"),
                                          (7, 4100, "bf16")])
def test_layernorm(ctx_bf16, ctx_f32, rows, cols, dt):
    ctx = ctx_bf16 if dt == "bf16" else ctx_f32
    _, x, xr = _t((rows, cols), 11, dt, 2.0)
    _, g, gr = _t((cols,), 12, dt, 0.02)
    g = g + 1
    gr = synth.to_f64(synth.from_f64(gr + 1, dt), dt) if dt == "bf16" else gr + 1
    _, b, br = _t((cols,), 13, dt, 0.01)
    y = torch.empty_like(x)
    ctx.layernorm(x, y, g, b, 1e-6)
    torch.cuda.synchronize()
    ref = R.layernorm(xr, from_dev(g), br, 1e-6)
    assert_close(from_dev(y), ref, 1e-2 if dt == "bf16" else 2e-6, 0.99999, "layernorm")


# ------------------------------------------------------------------ RoPE
@pytest.mark.parametrize("H,d,dt", [(16, 72, "bf16"), (4, 64, "f32"), (2, 128, "f32")])
def test_rope2d(H, d, dt):
    T = 157
    ctx = vit.Context(H * d, H, d, 4 * H * d, vit.BF16 if dt == "bf16" else vit.F32)
    a, qkv, qr = _t((T, 3 * H * d), 14, dt)
    pos = np.random.Generator(np.random.PCG64(15)).integers(0, 90, size=(T, 2)).astype(np.int32)
    before = qkv.clone()
    ctx.rope2d(qkv, int_dev(pos))
    torch.cuda.synchronize()
    q, k, v = R.split_qkv(qr, H, d)
    out = from_dev(qkv).reshape(T, 3, H, d)
    # fp32: the rotation angle p*w is carried in fp32 (3e-6 rad at p ~ 90)
    tol = 1e-2 if dt == "bf16" else 2e-5
    assert_close(out[:, 0], R.rope2d(q, pos), tol, 0.99999, "rope q")
    assert_close(out[:, 1], R.rope2d(k, pos), tol, 0.99999, "rope k")
    assert torch.equal(qkv.view(T, 3, H * d)[:, 2], before.view(T, 3, H * d)[:, 2])
    ctx.close()


# ------------------------------------------------------------------ merge / positions
@pytest.mark.parametrize("dt,C,grids", [
    ("bf16", 1152, [(50, 78)]), ("bf16", 1152, [(4, 6), (2, 2), (30, 32), (76, 58)]),
    ("f32", 256, [(16, 16)]), ("bf16", 12, [(2, 4), (6, 2)]), ("f32", 3, [(2, 2), (4, 2)]),
])
def test_merge_bit_exact(ctx_bf16, ctx_f32, dt, C, grids):
    ctx = ctx_bf16 if dt == "bf16" else ctx_f32
    T = synth.grid_tokens(grids)
    a, x, _ = _t((T, C), 16, dt)
    y = torch.full((T // 4, 4 * C), 7.0, dtype=x.dtype, device="cuda")
    ctx.spatial_merge_2x2(x, y, grids, C)
    torch.cuda.synchronize()
    ref = R.spatial_merge_2x2(a, grids)          # index map applied to the stored values
    got = y.cpu().view(torch.int16 if dt == "bf16" else torch.int32).numpy()
    exp = ref.view(np.int16 if dt == "bf16" else np.int32)
    np.testing.assert_array_equal(got, exp)


def test_merge_rejects_odd_grid(ctx_bf16):
    x = torch.zeros((3900, 1152), dtype=torch.bfloat16, device="cuda")
    y = torch.full((975, 4608), 3.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vit.VitError) as e:
        ctx_bf16.spatial_merge_2x2(x, y, [(60, 65)], 1152)
    assert e.value.code == 2
    torch.cuda.synchronize()
    assert torch.all(y == 3.0)                   # nothing was launched


@pytest.mark.parametrize("grids", [[(26, 30), (24, 37), (30, 32), (60, 65), (76, 58)],
                                   [(1, 1)], [(3, 1), (1, 5), (2, 2)]])
def test_positions_bit_exact(ctx_bf16, grids):
    T = synth.grid_tokens(grids)
    cu = torch.full((len(grids) + 1,), -1, dtype=torch.int32, device="cuda")
    pos = torch.full((T, 2), -1, dtype=torch.int32, device="cuda")
    ctx_bf16.positions_from_grids(grids, cu, pos)
    torch.cuda.synchronize()
    cu_r, pos_r = R.positions_from_grids(grids)
    np.testing.assert_array_equal(cu.cpu().numpy(), cu_r)
    np.testing.assert_array_equal(pos.cpu().numpy(), pos_r)


def test_positions_many_images(ctx_bf16):
    grids = [((i % 7) + 1, (i % 5) + 2) for i in range(600)]    # spans 3 launches
    T = synth.grid_tokens(grids)
    cu = torch.empty((601,), dtype=torch.int32, device="cuda")
    pos = torch.empty((T, 2), dtype=torch.int32, device="cuda")
    ctx_bf16.positions_from_grids(grids, cu, pos)
    torch.cuda.synchronize()
    cu_r, pos_r = R.positions_from_grids(grids)
    np.testing.assert_array_equal(cu.cpu().numpy(), cu_r)
    np.testing.assert_array_equal(pos.cpu().numpy(), pos_r)


# ------------------------------------------------------------------ attention
def _attention_case(dt, H, d, lens, P=0, Hkv=0, rope=False, seed=20):
    C = H * d
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    a, qkv, qr = _t((T, 3 * C), seed, dt)
    pos = np.random.Generator(np.random.PCG64(seed + 1)).integers(0, 100, size=(T, 2)).astype(np.int32)
    Hkv = Hkv or H
    pkv = pkv_r = None
    if P:
        _, pkv, pkv_r = _t((len(lens), 2, P, Hkv, d), seed + 2, dt)
    ctx = vit.Context(C, H, d, 4 * C, vit.BF16 if dt == "bf16" else vit.F32)
    o = torch.full((T, C), float("nan"), dtype=qkv.dtype, device="cuda")
    cu_d, pos_d = int_dev(cu), int_dev(pos)
    sq = vit.seqs(T, len(lens), int(max(lens)), cu_d, pos_d if rope else None, pkv, P, Hkv)
    ctx.attention(qkv, o, sq)
    torch.cuda.synchronize()
    st = ctx.device_status()
    ctx.close()
    q, k, v = R.split_qkv(qr, H, d)
    ref = R.attention(q, k, v, cu, pos if rope else None, pkv_r).reshape(T, C)
    return from_dev(o), ref, st


ATTN_CASES = [
    # (H, d, segment lengths, prefix P, prefix heads, rope on load)
    (3, 72, [300], 0, 0, False),
    (3, 72, [1, 130, 257, 300, 513], 0, 0, False),
    (3, 72, [200, 129], 0, 0, True),
    (2, 128, [257, 40], 0, 0, False),
    (2, 128, [300, 90], 100, 1, False),
    (2, 128, [256, 129], 256, 2, True),
    (3, 72, [140, 77], 130, 3, True),
    # 16 heads: pairs of query tiles; several lengths (and an empty image)
    # take the longest-first snake schedule, 70 sequences the plain order
    (16, 72, [700, 0, 300, 1300, 130, 1], 0, 0, False),
    (16, 72, [int(v) for v in np.random.Generator(np.random.PCG64(7)).integers(1, 200, 70)], 0, 0,
     False),
]


@pytest.mark.parametrize("H,d,lens,P,Hkv,rope", ATTN_CASES)
def test_attention_tc_bf16(H, d, lens, P, Hkv, rope):
    y, ref, st = _attention_case("bf16", H, d, lens, P, Hkv, rope)
    assert st == 0
    assert_close(y, ref, 2e-2, 0.9999, f"attention H{H} d{d} {lens} P{P} rope{rope}")


@pytest.mark.parametrize("d,lens,P,rope", [(64, [100, 37], 0, True), (64, [64, 1], 33, True),
                                           (72, [70], 0, False), (128, [50, 20], 40, False)])
def test_attention_simt_f32(d, lens, P, rope):
    H = 2
    y, ref, st = _attention_case("f32", H, d, lens, P, 1 if P else 0, rope, seed=30)
    assert_close(y, ref, 2e-5, None, f"attention f32 d{d}")


def test_attention_full_size_rows():
    # the encoder's attention at 3900 tokens, 16 x 72 heads (sampled query rows
    # against the oracle, which evaluates each query row independently)
    H, d, T = 16, 72, 3900
    C = H * d
    _, qkv, qr = _t((T, 3 * C), 40, "bf16")
    ctx = vit.Context(C, H, d, 4304, vit.BF16)
    o = torch.empty((T, C), dtype=torch.bfloat16, device="cuda")
    cu = np.array([0, T], np.int32)
    ctx.attention(qkv, o, vit.seqs(T, 1, T, int_dev(cu)))
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    ctx.close()
    q, k, v = R.split_qkv(qr, H, d)
    rows = np.random.Generator(np.random.PCG64(41)).choice(T, 64, replace=False)
    rows = np.concatenate([rows, [0, 127, 128, 255, 256, T - 1]])
    got = from_dev(o)[rows].reshape(len(rows), H, d)
    for h in range(H):
        ref = R.attention_segment(q[rows, h], k[:, h], v[:, h], 1 / np.sqrt(d))
        assert_close(got[:, h], ref, 2e-2, 0.9999, f"row sample head {h}")


# ------------------------------------------------------------------ every GEMM variant
VARIANT_CASES = [(300, 392, 200, 0), (257, 136, 64, 2), (3900, 3456, 1152, 0),
                 (3900, 1152, 4304, 2), (960, 4304, 1152, 1), (1, 8, 8, 0)]


@pytest.mark.parametrize("variant", ["1x128", "1x256", "2x128", "2x192", "2x256"])
@pytest.mark.parametrize("M,N,K,epi", VARIANT_CASES)
def test_linear_bf16_each_variant(ctx_bf16, monkeypatch, variant, M, N, K, epi):
    # VIT_GEMM_TILE pins the GEMM variant (CTAs per MMA x tile width)
    monkeypatch.setenv("VIT_GEMM_TILE", variant)
    _, x, xr = _t((M, K), 51, "bf16")
    _, w, wr = _t((N, K), 52, "bf16", 0.02)
    _, b, br = _t((N,), 53, "bf16", 0.01)
    _, res, rr = _t((M, N), 54, "bf16")
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ctx_bf16.linear(x, w, b, y, epi=epi, residual=res if epi == 2 else None)
    torch.cuda.synchronize()
    rows = np.arange(M)
    if M > 1024:
        g = np.random.Generator(np.random.PCG64(M + N + 7))
        rows = np.unique(np.concatenate([g.choice(M, 192, replace=False),
                                         [0, 127, 128, 255, 256, M - 129, M - 1]]))
    ref = R.linear(xr[rows], wr, br)
    if epi == 1:
        ref = R.gelu_tanh(ref)
    if epi == 2:
        ref = ref + rr[rows]
    got = from_dev(y)
    assert np.all(np.isfinite(got)), "unwritten outputs"
    assert_close(got[rows], ref, 1e-2, 0.99999, f"linear {variant} {M}x{N}x{K} epi{epi}")
    assert ctx_bf16.device_status() == 0
