"""Pins of the fp64 oracle against things other than itself: closed forms,
invariants, brute force on tiny inputs, library routines (torch fp64) and
hand-written fixtures in tests/golden/.  CPU only."""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import synth
from oracle import vit_ref as R
from oracle import run as orun
from tests import torch_fp64_layer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


# ------------------------------------------------------------------ LayerNorm
def test_layernorm_matches_torch():
    x = rng(1).standard_normal((7, 33)) * 3 + 1.5
    g = 1 + 0.1 * rng(2).standard_normal(33)
    b = 0.1 * rng(3).standard_normal(33)
    ref = F.layer_norm(torch.tensor(x), (33,), torch.tensor(g), torch.tensor(b), 1e-6).numpy()
    np.testing.assert_allclose(R.layernorm(x, g, b, 1e-6), ref, rtol=0, atol=1e-13)


def test_layernorm_moments_closed_form():
    # gamma = 1, beta = 0: per-row mean 0, biased variance v / (v + eps)
    x = rng(4).standard_normal((5, 1152)) * 2.0 - 0.7
    eps = 1e-2      # large eps so a dropped or misplaced eps is visible
    y = R.layernorm(x, np.ones(1152), np.zeros(1152), eps)
    v = x.var(axis=1)          # numpy var is the biased variance
    np.testing.assert_allclose(y.mean(axis=1), 0, atol=1e-13)
    np.testing.assert_allclose((y ** 2).mean(axis=1), v / (v + eps), rtol=1e-12)


def test_layernorm_affine_and_constant_row():
    x = np.tile(np.array([[2.5]]), (1, 8))            # constant row: x - mean = 0
    g = np.arange(8.0)
    b = np.linspace(-1, 1, 8)
    np.testing.assert_array_equal(R.layernorm(x, g, b), np.broadcast_to(b, (1, 8)))
    x = np.array([[1.0, -1.0]])                         # mean 0, var 1
    y = R.layernorm(x, np.array([2.0, 3.0]), np.array([0.5, -0.5]), eps=0.0)
    np.testing.assert_allclose(y, [[2.5, -3.5]], atol=1e-15)


# ------------------------------------------------------------------ GEMM
def test_linear_brute_force():
    x = rng(5).standard_normal((3, 4))
    w = rng(6).standard_normal((5, 4))
    b = rng(7).standard_normal(5)
    y = R.linear(x, w, b)
    for i in range(3):
        for j in range(5):
            acc = b[j]
            for k in range(4):
                acc += x[i, k] * w[j, k]
            assert abs(y[i, j] - acc) < 1e-13


def test_linear_matches_torch():
    x = rng(8).standard_normal((17, 40))
    w = rng(9).standard_normal((23, 40))
    b = rng(10).standard_normal(23)
    ref = F.linear(torch.tensor(x), torch.tensor(w), torch.tensor(b)).numpy()
    np.testing.assert_allclose(R.linear(x, w, b), ref, atol=1e-12)


# ------------------------------------------------------------------ GELU
def test_gelu_tanh_identities():
    u = np.linspace(-6, 6, 1001)
    g = R.gelu_tanh(u)
    assert R.gelu_tanh(np.array([0.0]))[0] == 0.0
    # 0.5u(1+tanh(a)) - (-0.5u)(1+tanh(-a)) = u exactly (tanh odd)
    np.testing.assert_allclose(g - R.gelu_tanh(-u), u, atol=1e-14)
    # the tanh form stays within 1e-3 of the exact erf form
    exact = np.array([0.5 * t * (1 + math.erf(t / math.sqrt(2))) for t in u])
    assert np.max(np.abs(g - exact)) < 1e-3
    # large |u| limits: identity and zero
    assert abs(R.gelu_tanh(np.array([30.0]))[0] - 30.0) < 1e-12
    assert abs(R.gelu_tanh(np.array([-30.0]))[0]) < 1e-12


def test_gelu_tanh_matches_torch():
    u = rng(11).standard_normal(1000) * 4
    ref = F.gelu(torch.tensor(u), approximate="tanh").numpy()
    np.testing.assert_allclose(R.gelu_tanh(u), ref, atol=1e-14)


# ------------------------------------------------------------------ RoPE
def _golden_rope():
    vals = []
    with open(os.path.join(GOLDEN, "rope2d_d8_example.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            i, _expr, v = line.split()
            vals.append((int(i), float(v)))
    return np.array([v for _, v in sorted(vals)])


def test_rope_golden_example():
    x = np.arange(1.0, 9.0).reshape(1, 1, 8)
    y = R.rope2d(x, np.array([[1, 2]]), theta=100.0)
    np.testing.assert_allclose(y[0, 0], _golden_rope(), atol=1e-14)


@pytest.mark.parametrize("d", [8, 64, 72, 128])
def test_rope_each_coordinate_angle(d):
    # unit vector in dim j of a half rotates into dim j + h/2 by angle p*w_j
    theta = 10000.0
    h = d // 2
    for axis in (0, 1):
        for j in range(h // 2):
            e = np.zeros((1, 1, d))
            e[0, 0, axis * h + j] = 1.0
            pos = np.array([[3, 0]]) if axis == 0 else np.array([[0, 5]])
            p = pos[0, axis]
            ang = p * theta ** (-2.0 * j / h)
            y = R.rope2d(e, pos, theta)[0, 0]
            expect = np.zeros(d)
            expect[axis * h + j] = math.cos(ang)
            expect[axis * h + h // 2 + j] = math.sin(ang)
            np.testing.assert_allclose(y, expect, atol=1e-14)


def test_rope_identity_norm_composition():
    d = 72
    x = rng(12).standard_normal((6, 3, d))
    np.testing.assert_array_equal(R.rope2d(x, np.zeros((6, 2), int)), x)
    pos = rng(13).integers(0, 80, size=(6, 2))
    y = R.rope2d(x, pos)
    # norm preserved per rotated pair
    h = d // 2
    for lo in (0, h):
        a0, b0 = x[..., lo:lo + h // 2], x[..., lo + h // 2:lo + h]
        a1, b1 = y[..., lo:lo + h // 2], y[..., lo + h // 2:lo + h]
        np.testing.assert_allclose(a0 ** 2 + b0 ** 2, a1 ** 2 + b1 ** 2, rtol=1e-12)
    # R(a) R(b) = R(a + b)
    p2 = rng(14).integers(-40, 40, size=(6, 2))
    np.testing.assert_allclose(R.rope2d(R.rope2d(x, pos), p2), R.rope2d(x, pos + p2), atol=1e-11)


def test_rope_relative_offset():
    # <R(p) q, R(p') k> depends only on p' - p: shifting both by s is invisible
    d = 72
    q = rng(15).standard_normal((1, 1, d))
    k = rng(16).standard_normal((1, 1, d))
    p, pk = np.array([[3, 7]]), np.array([[11, 2]])
    base = float(np.sum(R.rope2d(q, p) * R.rope2d(k, pk)))
    for s in ([1, 0], [0, 1], [5, -9], [40, 33]):
        s = np.array([s])
        v = float(np.sum(R.rope2d(q, p + s) * R.rope2d(k, pk + s)))
        assert abs(v - base) < 1e-11
    # and equals <q, R(p' - p) k>
    v = float(np.sum(q * R.rope2d(k, pk - p)))
    assert abs(v - base) < 1e-11


# ------------------------------------------------------------------ attention
def _brute_attention(q, k, v, scale):
    n, m = q.shape[0], k.shape[0]
    out = np.zeros((n, v.shape[1]))
    for i in range(n):
        s = [sum(q[i, t] * k[j, t] for t in range(q.shape[1])) * scale for j in range(m)]
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        z = sum(e)
        for j in range(m):
            out[i] += e[j] / z * v[j]
    return out


def test_attention_brute_force_tiny():
    T, H, d = 8, 2, 4
    q, k, v = (rng(s).standard_normal((T, H, d)) for s in (20, 21, 22))
    o = R.attention(q, k, v, [0, T])
    for h in range(H):
        np.testing.assert_allclose(o[:, h], _brute_attention(q[:, h], k[:, h], v[:, h], 0.5),
                                   atol=1e-13)


def test_attention_matches_torch_sdpa():
    T, H, d = 37, 3, 72
    q, k, v = (rng(s).standard_normal((T, H, d)) for s in (23, 24, 25))
    ref = F.scaled_dot_product_attention(*(torch.tensor(t).transpose(0, 1) for t in (q, k, v)))
    np.testing.assert_allclose(R.attention(q, k, v, [0, T]), ref.transpose(0, 1).numpy(),
                               atol=1e-13)


def test_attention_rows_sum_to_one():
    # with V = identity the output rows are the softmax rows themselves
    n, d = 6, 6
    q = rng(26).standard_normal((n, 1, d)) * 3
    k = rng(27).standard_normal((n, 1, d)) * 3
    v = np.eye(n).reshape(n, 1, d)
    p = R.attention(q, k, v, [0, n])[:, 0]
    assert np.all(p >= 0)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-14)


def test_attention_special_cases():
    n, d = 9, 8
    q = rng(28).standard_normal((n, 1, d))
    v = rng(29).standard_normal((n, 1, d))
    # all keys equal -> every output row is the mean of V
    k = np.tile(rng(30).standard_normal((1, 1, d)), (n, 1, 1))
    o = R.attention(q, k, v, [0, n])
    np.testing.assert_allclose(o[:, 0], np.tile(v[:, 0].mean(0), (n, 1)), atol=1e-14)
    # one dominant key -> its V row
    k = np.zeros((n, 1, d))
    k[4, 0, :] = 1.0
    qd = np.full((n, 1, d), 200.0)
    o = R.attention(qd, k, v, [0, n])
    np.testing.assert_allclose(o[:, 0], np.tile(v[4, 0], (n, 1)), atol=1e-12)
    # a scale argument multiplies the logits
    k = rng(31).standard_normal((n, 1, d))
    o1 = R.attention(q, k, v, [0, n], scale=0.7)
    o2 = R.attention(q * 0.7 * math.sqrt(d), k, v, [0, n])
    np.testing.assert_allclose(o1, o2, atol=1e-13)


def test_attention_permutations():
    n, H, d = 10, 2, 8
    q, k, v = (rng(s).standard_normal((n, H, d)) for s in (32, 33, 34))
    o = R.attention(q, k, v, [0, n])
    perm = rng(35).permutation(n)
    # permuting queries permutes outputs; permuting (K, V) jointly changes nothing
    np.testing.assert_allclose(R.attention(q[perm], k, v, [0, n]), o[perm], atol=1e-13)
    np.testing.assert_allclose(R.attention(q, k[perm], v[perm], [0, n]), o, atol=1e-13)


def test_attention_varlen_is_block_diagonal():
    lens = [5, 1, 7, 3]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, H, d = cu[-1], 2, 8
    q, k, v = (rng(s).standard_normal((T, H, d)) for s in (36, 37, 38))
    pos = rng(39).integers(0, 9, size=(T, 2))
    o = R.attention(q, k, v, cu, pos)
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        np.testing.assert_allclose(o[a:b], R.attention(q[a:b], k[a:b], v[a:b], [0, b - a],
                                                       pos[a:b]), atol=1e-13)
    # reversing the segment order reverses the output blocks
    order = list(range(len(lens)))[::-1]
    idx = np.concatenate([np.arange(cu[s], cu[s + 1]) for s in order])
    cu2 = np.concatenate([[0], np.cumsum([lens[s] for s in order])])
    o2 = R.attention(q[idx], k[idx], v[idx], cu2, pos[idx])
    np.testing.assert_allclose(o2, o[idx], atol=1e-13)


def test_attention_prefix_is_concatenation():
    lens, P, H, Hkv, d = [6, 4], 5, 4, 2, 8
    cu = np.concatenate([[0], np.cumsum(lens)])
    T = cu[-1]
    q, k, v = (rng(s).standard_normal((T, H, d)) for s in (40, 41, 42))
    pkv = rng(43).standard_normal((2, 2, P, Hkv, d))
    pos = rng(44).integers(0, 5, size=(T, 2))
    o = R.attention(q, k, v, cu, pos, pkv)
    qr, kr = R.rope2d(q, pos), R.rope2d(k, pos)
    for s in range(2):
        a, b = cu[s], cu[s + 1]
        for h in range(H):
            ks = np.concatenate([pkv[s, 0, :, h // 2], kr[a:b, h]])
            vs = np.concatenate([pkv[s, 1, :, h // 2], v[a:b, h]])
            np.testing.assert_allclose(o[a:b, h], _brute_attention(qr[a:b, h], ks, vs,
                                                                   1 / math.sqrt(d)), atol=1e-12)


# ------------------------------------------------------------------ merge / positions
def _golden_merge():
    maps = {}
    with open(os.path.join(GOLDEN, "merge_index_maps.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            grids, rest = line.split("|")
            o, ins = rest.split(":")
            maps.setdefault(grids.strip(), {})[int(o)] = [int(t) for t in ins.split()]
    return maps


def test_merge_golden_index_maps():
    for key, m in _golden_merge().items():
        grids = [tuple(int(a) for a in g.split("x")) for g in key.split(",")]
        T = synth.grid_tokens(grids)
        C = 3
        x = np.arange(T * C).reshape(T, C)     # token t holds t*C .. t*C+C-1
        y = R.spatial_merge_2x2(x, grids)
        assert y.shape == (T // 4, 4 * C)
        for o, ins in m.items():
            expect = np.concatenate([x[t] for t in ins])
            np.testing.assert_array_equal(y[o], expect)


def test_merge_is_a_permutation():
    grids = [(6, 8), (2, 2), (4, 10)]
    T = synth.grid_tokens(grids)
    C = 5
    x = np.arange(T * C).reshape(T, C)
    y = R.spatial_merge_2x2(x, grids)
    flat = y.reshape(-1)
    assert sorted(flat.tolist()) == list(range(T * C))        # bijection
    inv = np.empty(T * C, dtype=np.int64)
    inv[flat] = np.arange(T * C)
    np.testing.assert_array_equal(flat[inv].reshape(T, C), x)    # inverse recovers x
    with pytest.raises(ValueError):
        R.spatial_merge_2x2(np.zeros((60 * 65, 1)), [(60, 65)])


def test_positions_golden():
    with open(os.path.join(GOLDEN, "positions_2x3_1x2.txt")) as f:
        lines = [ln for ln in f if not ln.startswith("#")]
    cu_exp = [int(t) for t in lines[0].split(":")[1].split()]
    pos_exp = [tuple(int(a) for a in t.split(",")) for t in lines[1].split(":")[1].split()]
    cu, pos = R.positions_from_grids([(2, 3), (1, 2)])
    assert cu.tolist() == cu_exp
    assert [tuple(p) for p in pos.tolist()] == pos_exp


# ------------------------------------------------------------------ layer / stack
def _small_layer_inputs(seed, T_grids, C=64, H=4, d=16, Fm=96, dtype="f32", P=0, attn_only=False):
    wl = synth.Workload("t", seed, dtype, C, H, d, Fm, 2, tuple(T_grids),
                        prefix_len=P, kv_heads=(H // 2 if P else 0), attn_only=attn_only)
    return wl, synth.make_inputs(wl)


@pytest.mark.parametrize("P,attn_only", [(0, False), (3, True)])
def test_layer_matches_torch_restatement(P, attn_only):
    wl, inp = _small_layer_inputs(50, [(3, 4), (2, 5)], P=P, attn_only=attn_only)
    cu, pos = R.positions_from_grids(wl.grids)
    w = orun.layer_f64(inp, 0)
    x = synth.to_f64(inp.x, wl.dtype)
    pkv = None if inp.prefix_kv is None else synth.to_f64(inp.prefix_kv, wl.dtype)
    y = R.layer_forward(x, w, cu, pos, wl.heads, wl.head_dim, wl.ln_eps, wl.rope_theta, pkv,
                        attn_only)
    ref = torch_fp64_layer.layer(x, w, cu, pos, wl.heads, wl.head_dim, wl.ln_eps,
                                 wl.rope_theta, pkv, attn_only)
    np.testing.assert_allclose(y, ref, atol=1e-12)


@pytest.mark.parametrize("P,attn_only", [(0, False), (3, True)])
def test_stack_matches_torch_restatement_layer_by_layer(P, attn_only):
    # The stack oracle (vit_ref.encoder_forward, reached through
    # oracle.run.run_layers as every stack-level GPU test reaches it) against
    # the independent PyTorch restatement applied once per layer, with each
    # layer's own weights, over two packed images: a stack that reused one
    # layer's weights, dropped or repeated a layer, or fed a layer the wrong
    # input would differ.
    wl = synth.Workload("t", 51, "f32", 64, 4, 16, 96, 3, ((3, 4), (2, 5)), prefix_len=P,
                        kv_heads=(2 if P else 0), attn_only=attn_only)
    inp = synth.make_inputs(wl)
    got = orun.run_layers(inp)
    cu, pos = R.positions_from_grids(wl.grids)
    pkv = None if inp.prefix_kv is None else synth.to_f64(inp.prefix_kv, wl.dtype)
    ref = synth.to_f64(inp.x, wl.dtype)
    outs = []
    for i in range(wl.layers):
        ref = torch_fp64_layer.layer(ref, orun.layer_f64(inp, i), cu, pos, wl.heads, wl.head_dim,
                                     wl.ln_eps, wl.rope_theta, pkv, attn_only)
        outs.append(ref)
    np.testing.assert_allclose(got, ref, atol=1e-11)
    # every layer changes the activations, so the comparison above covers
    # each layer of the chain
    for a, b in zip(outs, outs[1:]):
        assert np.max(np.abs(a - b)) > 1e-3
    # a shorter stack stops after its own last layer
    np.testing.assert_allclose(orun.run_layers(inp, n_layers=2), outs[1], atol=1e-11)


def test_projector_matches_torch_restatement():
    # the composition LN -> linear + GELU -> linear against PyTorch's routines,
    # with ragged widths; and its two closed-form cases
    w = {k: synth.to_f64(v, "f32") for k, v in
         synth.make_projector_weights(40, 24, 12, 55, "f32").items()}
    x = rng(56).standard_normal((7, 40)) * 3.0 + 1.0
    np.testing.assert_allclose(R.projector(x, w, 1e-6), torch_fp64_layer.projector(x, w, 1e-6),
                               atol=1e-12)
    # zero second weight: y = b2 for every row
    w0 = dict(w, w2=np.zeros_like(w["w2"]))
    np.testing.assert_allclose(R.projector(x, w0), np.broadcast_to(w["b2"], (7, 12)), atol=0)
    # a constant row normalises to beta: y = W2 GELU(W1 beta + b1) + b2
    xc = np.full((1, 40), 2.5)
    want = R.linear(R.gelu_tanh(R.linear(w["ln_b"][None, :], w["w1"], w["b1"])), w["w2"], w["b2"])
    np.testing.assert_allclose(R.projector(xc, w), want, atol=1e-12)


def test_c1_layer_matches_torch_restatement():
    wl = synth.get("c1")
    inp = synth.make_inputs(wl)
    cu, pos = R.positions_from_grids(wl.grids)
    w = orun.layer_f64(inp, 0)
    x = synth.to_f64(inp.x, wl.dtype)
    y = R.layer_forward(x, w, cu, pos, wl.heads, wl.head_dim)
    ref = torch_fp64_layer.layer(x, w, cu, pos, wl.heads, wl.head_dim, 1e-6, 1e4)
    np.testing.assert_allclose(y, ref, atol=1e-10)


# ------------------------------------------------------------------ synth
def test_bf16_rounding_matches_torch():
    a = rng(60).standard_normal(100000) * 10.0 ** rng(61).integers(-6, 6, 100000)
    bits = synth.round_bf16_bits(a)
    ref = torch.tensor(a.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    np.testing.assert_array_equal(bits, ref.view(np.uint16))
    np.testing.assert_array_equal(synth.bf16_bits_to_f64(bits),
                                  torch.tensor(a.astype(np.float32)).to(torch.bfloat16)
                                  .to(torch.float64).numpy())


def test_workload_flop_counts():
    # per-layer algorithmic FLOP of the 3900-token layer, by hand:
    # GEMM 2*T*C*(3C + C + 2F); attention 4*T^2*C
    f = synth.get("c2").flops()
    T, C, Fm = 3900, 1152, 4304
    assert f["gemm"] == 27 * 2.0 * T * C * (4 * C + 2 * Fm)
    assert f["attn"] == 27 * 4.0 * T * T * C
    assert abs(f["total"] - 5.0987e12) / 5.0987e12 < 1e-4


# ------------------------------------------------------------------ embedding
from oracle import embed_ref as E  # noqa: E402


@pytest.mark.parametrize("p,rows,cols,C", [(14, 3, 5, 24), (4, 2, 2, 8), (2, 1, 3, 5)])
def test_patch_embed_matches_conv2d(p, rows, cols, C):
    r = rng(70 + p)
    img = r.standard_normal((3, rows * p, cols * p))
    w = r.standard_normal((C, 3, p, p))
    b = r.standard_normal(C)
    got = E.patch_embed(img, w.reshape(C, -1), b, p)
    ref = F.conv2d(torch.tensor(img)[None], torch.tensor(w), torch.tensor(b), stride=p)
    ref = ref[0].permute(1, 2, 0).reshape(rows * cols, C).numpy()  # tokens row-major
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("gh,gw,oh,ow", [(27, 27, 50, 78), (27, 27, 6, 4), (5, 7, 5, 7),
                                         (4, 3, 9, 2), (1, 1, 3, 3), (6, 6, 1, 1)])
def test_bilinear_matches_torch_interpolate(gh, gw, oh, ow):
    t = rng(80 + oh).standard_normal((gh, gw, 3))
    got = E.bilinear_resize(t, oh, ow)
    ref = F.interpolate(torch.tensor(t).permute(2, 0, 1)[None], size=(oh, ow), mode="bilinear",
                        align_corners=False)[0].permute(1, 2, 0).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_bilinear_affine_closed_form():
    # table value 2y + x on a 2x2 grid; 4 outputs per axis sit at the clamped
    # half-pixel source coordinates 0, 1/4, 3/4, 1, where bilinear
    # interpolation reproduces the affine function exactly
    t = np.array([[0.0, 1.0], [2.0, 3.0]])[:, :, None]
    got = E.bilinear_resize(t, 4, 4)[:, :, 0]
    c = np.array([0.0, 0.25, 0.75, 1.0])
    np.testing.assert_array_equal(got, 2 * c[:, None] + c[None, :])


def test_bilinear_identity_and_constant():
    t = rng(90).standard_normal((5, 6, 4))
    np.testing.assert_array_equal(E.bilinear_resize(t, 5, 6), t)  # s = i exactly
    k = np.full((3, 4, 2), 1.75)
    np.testing.assert_allclose(E.bilinear_resize(k, 7, 11), 1.75, rtol=0, atol=1e-15)


def test_embed_images_packs_images_in_order():
    r = rng(91)
    p, C = 2, 6
    grids = [(2, 3), (1, 2)]
    imgs = [r.standard_normal((3, a * p, b * p)) for a, b in grids]
    w, b, t = r.standard_normal((C, 12)), r.standard_normal(C), r.standard_normal((4, 4, C))
    got = E.embed_images(imgs, grids, p, w, b, t)
    assert got.shape == (8, C)
    first = E.patch_embed(imgs[0], w, b, p) + E.bilinear_resize(t, 2, 3).reshape(6, C)
    second = E.patch_embed(imgs[1], w, b, p) + E.bilinear_resize(t, 1, 2).reshape(2, C)
    np.testing.assert_array_equal(got, np.concatenate([first, second]))


# ------------------------------------------------------------------ MXFP8 (block-scaled 8-bit)
from oracle import mxfp8_ref as MX  # noqa: E402


def _torch_e4m3(x):
    """PyTorch's float8_e4m3fn conversion (round to nearest even, no clamp)."""
    return torch.tensor(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_table_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.tensor(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = MX.e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))
    # the definition's landmarks: 1.0, largest normal, smallest normal and subnormal
    assert MX.e4m3_decode([0x38, 0x7E, 0x08, 0x01]).tolist() == [1.0, 448.0, 2.0 ** -6, 2.0 ** -9]


def test_e4m3_round_trip_of_every_code():
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)
    assert np.array_equal(MX.e4m3_encode(MX.e4m3_decode(codes)), codes)


def test_e4m3_rounding_matches_torch():
    # every midpoint between neighbouring values (ties), points just off them,
    # and random values over the whole range, up to 464 (torch does not clamp)
    v = np.unique(MX.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = (v[1:] + v[:-1]) / 2
    pts = np.concatenate([v, mids, mids * (1 + 2.0 ** -12), mids * (1 - 2.0 ** -12),
                          [464.0, 460.0, 449.0]])
    r = rng(40)
    pts = np.concatenate([pts, np.exp2(r.uniform(-12, np.log2(464), 4000))])
    pts = np.concatenate([pts, -pts]).astype(np.float32).astype(np.float64)
    assert np.array_equal(MX.e4m3_encode(pts), _torch_e4m3(pts))


def test_e4m3_clamps_above_the_largest_normal():
    x = np.array([465.0, 480.0, 1e6, -500.0, np.inf])
    assert MX.e4m3_encode(x).tolist() == [0x7E, 0x7E, 0x7E, 0xFE, 0x7E]
    assert MX.e4m3_encode([np.nan]).tolist() == [0x7F]


def test_mx_block_exponent_closed_form():
    # amax = f * 2^k with f in [1, 2) gives X = k - 8: the scaled maximum lands in [256, 512)
    r = rng(41)
    k = r.integers(-100, 100, 64)
    f = r.uniform(1.0, 2.0, 64)
    x = np.zeros((64, 40))
    x[:, 0] = -f * np.exp2(k)           # the block maximum, negative on purpose
    x[:, 1:32] = r.uniform(-1, 1, (64, 31)) * np.exp2(k)[:, None]
    x[:, 32:] = 3.0                     # second block: 8 elements (K = 40)
    X = MX.mx_block_exponents(x)
    assert X.shape == (64, 2)
    assert np.array_equal(X[:, 0], k - 8)
    assert np.all(X[:, 1] == 1 - 8)     # log2(3) = 1.58: only the block's own elements count
    assert MX.mx_block_exponents(np.zeros((1, 32)))[0, 0] == -127
    assert MX.mx_block_exponents(np.full((1, 32), 2.0 ** 200))[0, 0] == 127


def test_mx_quantize_exact_on_representable_blocks():
    # elements that are E4M3 values times the block's own scale survive exactly
    r = rng(42)
    codes = r.integers(0, 0x7F, (16, 96)).astype(np.uint8) | (r.integers(0, 2, (16, 96)) << 7).astype(np.uint8)
    codes[:, ::32] = 0x78 | (codes[:, ::32] & 0x80)       # each block holds +-256: X is the block's own
    X = r.integers(-20, 20, (16, 3))
    x = MX.e4m3_decode(codes) * np.exp2(np.repeat(X, 32, axis=1).astype(np.float64))
    q, s = MX.mx_quantize(x)
    assert np.array_equal(s.astype(np.int64) - 127, X)
    assert np.array_equal(MX.mx_dequantize(q, s), x)


def test_mx_quantize_error_bound():
    # round to nearest: |x - deq| <= half the E4M3 spacing at x, times 2^X,
    # except where the clamp at 448 * 2^X applies
    r = rng(43)
    x = r.standard_normal((32, 128)) * np.exp2(r.integers(-10, 10, (32, 1)))
    q, s = MX.mx_quantize(x)
    d = MX.mx_dequantize(q, s)
    X = np.repeat(s.astype(np.int64) - 127, 32, axis=1).astype(np.float64)
    sx = np.abs(x) / np.exp2(X)
    clamp = sx > 448
    spacing = np.exp2(np.maximum(np.floor(np.log2(np.maximum(sx, 2.0 ** -30))), -6) - 3)
    err = np.abs(d - x) / np.exp2(X)
    assert np.all(err[~clamp] <= spacing[~clamp] / 2)
    assert np.all(np.abs(d[clamp]) == 448 * np.exp2(X[clamp]))
    assert np.all(np.sign(d[d != 0]) == np.sign(x[d != 0]))


def test_mx_linear_integer_closed_form():
    # integer E4M3 values with scale 2^0: deq(A).deq(W)^T is an integer matmul
    r = rng(44)
    vals = np.arange(-16, 17)
    a = r.choice(vals, (9, 70))
    w = r.choice(vals, (13, 70))
    a[:, [0, 32, 64]] = 288             # E4M3 block maxima in [256, 512) keep X = 0
    w[:, [0, 32, 64]] = -256
    qa, sa = MX.mx_quantize(a.astype(np.float64))
    qw, sw = MX.mx_quantize(w.astype(np.float64))
    assert np.all(sa == 127) and np.all(sw == 127)
    b = r.integers(-5, 5, 13)
    ref = (a.astype(np.int64) @ w.astype(np.int64).T + b).astype(np.float64)
    assert np.array_equal(MX.mx_linear(qa, sa, qw, sw, b), ref)
    res = r.standard_normal((9, 13))
    assert np.array_equal(MX.mx_linear(qa, sa, qw, sw, b, "residual", res), ref + res)
    g = MX.mx_linear(qa, sa, qw, sw, b, "gelu")
    np.testing.assert_allclose(g, R.gelu_tanh(ref), rtol=0, atol=0)


def test_mx_linear_power_of_two_rescaling():
    # raising one block's scale byte by n multiplies exactly that block's
    # contribution by 2^n
    r = rng(45)
    qa, sa = MX.mx_quantize(r.standard_normal((5, 64)))
    qw, sw = MX.mx_quantize(r.standard_normal((7, 64)))
    y = MX.mx_linear(qa, sa, qw, sw)
    sa2 = sa.copy()
    sa2[:, 1] += 3
    y2 = MX.mx_linear(qa, sa2, qw, sw)
    da = MX.mx_dequantize(qa, sa)
    dw = MX.mx_dequantize(qw, sw)
    part = da[:, 32:] @ dw[:, 32:].T
    np.testing.assert_allclose(y2, y + 7 * part, rtol=1e-12, atol=1e-12)


def _small_layer(seed, C=64, H=2, F=96, T=70):
    r = rng(seed)
    w = {"ln1_g": 1 + 0.02 * r.standard_normal(C), "ln1_b": 0.01 * r.standard_normal(C),
         "w_qkv": 0.05 * r.standard_normal((3 * C, C)), "b_qkv": 0.01 * r.standard_normal(3 * C),
         "w_o": 0.05 * r.standard_normal((C, C)), "b_o": 0.01 * r.standard_normal(C),
         "ln2_g": 1 + 0.02 * r.standard_normal(C), "ln2_b": 0.01 * r.standard_normal(C),
         "w_fc1": 0.05 * r.standard_normal((F, C)), "b_fc1": 0.01 * r.standard_normal(F),
         "w_fc2": 0.05 * r.standard_normal((C, F)), "b_fc2": 0.01 * r.standard_normal(C)}
    x = r.standard_normal((T, C))
    cu = np.array([0, 40, T])
    pos = np.stack([np.arange(T) // 7, np.arange(T) % 7], axis=1)
    return x, w, cu, pos, H, C // H


def test_mx_layer_with_plain_projections_is_the_fp64_layer():
    x, w, cu, pos, H, d = _small_layer(46)
    got = MX.layer_forward_mx8(x, w, cu, pos, H, d, project=R.linear)
    assert np.array_equal(got, R.layer_forward(x, w, cu, pos, H, d))
    got = MX.layer_forward_mx8(x, w, cu, pos, H, d, attn_only=True, project=R.linear)
    assert np.array_equal(got, R.layer_forward(x, w, cu, pos, H, d, attn_only=True))


def test_mx_layer_routes_every_projection_through_the_quantised_product():
    x, w, cu, pos, H, d = _small_layer(47)
    seen = []

    def spy(a, wt, b=None):
        seen.append((a.shape, wt.shape))
        return MX.mx_project(a, wt, b)

    MX.layer_forward_mx8(x, w, cu, pos, H, d, project=spy)
    T, C = x.shape
    F = w["w_fc1"].shape[0]
    assert seen == [((T, C), (3 * C, C)), ((T, C), (C, C)), ((T, C), (F, C)), ((T, F), (C, F))]


def test_mx_layer_error_is_bounded():
    # E4M3 rounding of every projection's operands: well below the signal,
    # but not zero
    x, w, cu, pos, H, d = _small_layer(48)
    ref = R.layer_forward(x, w, cu, pos, H, d)
    got = MX.layer_forward_mx8(x, w, cu, pos, H, d)
    dy, dr = got - x, ref - x          # the layer's own contribution, without the residual
    cos = float(np.sum(dy * dr) / np.sqrt(np.sum(dy * dy) * np.sum(dr * dr)))
    assert 0.99 <= cos < 1.0, cos
