"""MXFP8 (block-scaled E4M3) quantisation and GEMM through the C ABI against
the fp64 oracle of oracle/mxfp8_ref.py.

The quantiser takes integer decisions (codes and exponents) from exact
fp32 arithmetic, so it is compared bit for bit.  The GEMM computes on the
same codes as the oracle, so its bar is the bf16 GEMM's (fp32 accumulation,
one bf16 rounding of the output).  A separate, looser bound checks the
quantisation error against the unquantised fp64 product."""
import numpy as np
import pytest
import torch

import synth
from oracle import mxfp8_ref as MX
from oracle import vit_ref as R
from tests.gpu_util import assert_close, from_dev, metrics, to_dev

pytestmark = pytest.mark.gpu

vit = pytest.importorskip("vision_transformer_encoder_layernorm_b200")


@pytest.fixture(scope="module")
def ctx():
    c = vit.Context(1152, 16, 72, 4304, vit.BF16)
    yield c
    c.close()


def _t(shape, seed, scale=1.0):
    a = synth.random_tensor(shape, seed, "bf16", scale)
    return to_dev(a, "bf16"), synth.to_f64(a, "bf16")


def _scale_index(rows, K):
    """Byte offset of the scale of (row r, 32-column group j) in the block
    layout documented with vit_mx8_quantize, as an index array [rows, groups]."""
    nkb = (K + 127) // 128
    r = np.arange(rows)[:, None]
    j = np.arange((K + 31) // 32)[None, :]
    return ((r // 128) * nkb + j // 4) * 512 + (r % 128 % 32) * 16 + (r % 128 // 32) * 4 + j % 4


def _quantize(ctx, x, rows, K):
    codes = torch.empty((rows, vit.mx8_row_bytes(K)), dtype=torch.uint8, device="cuda")
    scales = torch.empty(vit.mx8_scale_bytes(rows, K), dtype=torch.uint8, device="cuda")
    ctx.mx8_quantize(x, codes, scales)
    return codes, scales


QUANT_CASES = [(300, 1152), (130, 4304), (5, 48), (1, 16), (257, 200)]


@pytest.mark.parametrize("rows,K", QUANT_CASES)
def test_mx8_quantize_bit_exact(ctx, rows, K):
    x, xr = _t((rows, K), 70 + K)
    # rows of very different magnitudes, a zero row and a row of tiny values
    mag = np.exp2(np.random.Generator(np.random.PCG64(rows)).integers(-30, 30, rows)).astype(np.float64)
    xr = xr * mag[:, None]
    xr[rows // 2] = 0.0
    if rows > 3:
        xr[3] *= 2.0 ** -100
    bits = synth.round_bf16_bits(xr)
    xr = synth.bf16_bits_to_f64(bits)
    x = to_dev(bits, "bf16")
    codes, scales = _quantize(ctx, x, rows, K)
    torch.cuda.synchronize()
    q_ref, s_ref = MX.mx_quantize(xr)
    q = codes.cpu().numpy()[:, :K]
    s = scales.cpu().numpy()
    idx = _scale_index(rows, K)
    assert np.array_equal(q, q_ref), f"codes differ at {np.argwhere(q != q_ref)[:5].tolist()}"
    assert np.array_equal(s[idx], s_ref)
    pad = np.ones(s.size, bool)
    pad[idx.ravel()] = False
    assert np.all(s[pad] == 127)  # padding blocks read as 2^0
    assert ctx.device_status() == 0


LN_MX_CASES = [(3900, 1152), (257, 200), (130, 36), (7, 4), (129, 1536)]


@pytest.mark.parametrize("rows,cols", LN_MX_CASES)
def test_layernorm_mx8_equals_layernorm_then_quantise(ctx, rows, cols):
    """vit_layernorm_mx8 gives the codes and scales of vit_mx8_quantize applied
    to vit_layernorm's bf16 output, bit for bit (padding scales included),
    across ragged row blocks, a partial last group and widths of 1 to 48
    groups; and the codes match the oracle's quantiser on that output."""
    x, _ = _t((rows, cols), 90 + cols, 3.0)
    g, _ = _t((cols,), 91 + cols)
    b, _ = _t((cols,), 92 + cols, 0.5)
    y = torch.empty_like(x)
    ctx.layernorm(x, y, g, b, eps=1e-6)
    c0, s0 = _quantize(ctx, y, rows, cols)
    c1 = torch.empty_like(c0)
    s1 = torch.full_like(s0, 0xFF)  # every byte must be written (no 0xFF is a valid scale here)
    ctx.layernorm_mx8(x, g, b, c1, s1, eps=1e-6)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    assert torch.equal(c0[:, :cols], c1[:, :cols])
    assert torch.equal(s0, s1)
    q_ref, s_ref = MX.mx_quantize(from_dev(y))
    assert np.array_equal(c1.cpu().numpy()[:, :cols], q_ref)
    assert np.array_equal(s1.cpu().numpy()[_scale_index(rows, cols)], s_ref)


def test_layernorm_mx8_errors(ctx):
    x, _ = _t((4, 1540), 95)
    g, _ = _t((1540,), 96)
    c = torch.empty((4, vit.mx8_row_bytes(1540)), dtype=torch.uint8, device="cuda")
    sc = torch.empty(vit.mx8_scale_bytes(4, 1540), dtype=torch.uint8, device="cuda")
    with pytest.raises(vit.VitError) as ei:
        ctx.layernorm_mx8(x, g, g, c, sc)
    assert ei.value.code == 3  # wider than 1536 columns: unsupported
    x2, _ = _t((4, 6), 97)
    g2, _ = _t((6,), 98)
    with pytest.raises(vit.VitError) as ei:
        ctx.layernorm_mx8(x2, g2, g2, c, sc)
    assert ei.value.code == 3  # cols % 4 != 0


GEMM_CASES = [
    # (M, N, K, epilogue): ragged M, several N tiles, K with a partial
    # 128-column block and a partial 32-element group; then fc1 of the
    # 3900-patch layer
    (300, 384, 1152, 0), (257, 256, 4304, 1), (130, 128, 48, 2), (129, 136, 200, 0),
    (3900, 4304, 1152, 1),
]


@pytest.mark.parametrize("M,N,K,epi", GEMM_CASES)
def test_linear_mx8_matches_oracle(ctx, M, N, K, epi):
    x, xr = _t((M, K), 80 + M)
    w, wr = _t((N, K), 81 + N, 0.02)
    b, br = _t((N,), 82)
    res, rr = _t((M, N), 83)
    a = _quantize(ctx, x, M, K)
    wq = _quantize(ctx, w, N, K)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ctx.linear_mx8(a, wq, b, y, K, epi=epi, residual=res if epi == 2 else None)
    torch.cuda.synchronize()
    rows = np.arange(M)
    if M > 1024:  # sampled rows, first and last tiles included
        g = np.random.Generator(np.random.PCG64(M + N))
        rows = np.unique(np.concatenate([g.choice(M, 256, replace=False),
                                         [0, 127, 128, M - 129, M - 1]]))
    qa, sa = MX.mx_quantize(xr[rows])
    qw, sw = MX.mx_quantize(wr)
    ref = MX.mx_linear(qa, sa, qw, sw, br, ["none", "gelu", "residual"][epi],
                       rr[rows] if epi == 2 else None)
    assert_close(from_dev(y)[rows], ref, 1e-2, 0.99999, f"linear mx8 {M}x{N}x{K} epi{epi}")
    assert ctx.device_status() == 0


def test_linear_mx8_quantisation_error(ctx):
    # E4M3 keeps 3 mantissa bits: each operand carries a relative rounding
    # error of at most 2^-4 (rms about 2^-4/sqrt(3) over a binade), so the
    # product's noise-to-signal ratio is about 0.04-0.05 and its cosine to
    # the unquantised product about 0.999; the bar leaves room for that
    M, N, K = 300, 384, 1152
    x, xr = _t((M, K), 90)
    w, wr = _t((N, K), 91, 0.02)
    b, br = _t((N,), 92, 0.01)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ctx.linear_mx8(_quantize(ctx, x, M, K), _quantize(ctx, w, N, K), b, y, K)
    torch.cuda.synchronize()
    rel, cos = metrics(from_dev(y), R.linear(xr, wr, br))
    assert cos >= 0.995 and rel <= 0.15, (rel, cos)


def test_linear_mx8_zero_input_gives_bias(ctx):
    M, N, K = 130, 128, 256
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    w, _ = _t((N, K), 93)
    b, br = _t((N,), 94)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ctx.linear_mx8(_quantize(ctx, x, M, K), _quantize(ctx, w, N, K), b, y, K)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(y), np.broadcast_to(br, (M, N)))


def test_mx8_errors_launch_nothing(ctx):
    M, N, K = 16, 16, 64
    x, _ = _t((M, K), 95)
    a = _quantize(ctx, x, M, K)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vit.VitError) as e:
        ctx.linear_mx8(a, a, None, torch.empty((M, 12), dtype=torch.bfloat16, device="cuda"), K)  # N % 8
    assert e.value.code == 3
    with pytest.raises(vit.VitError) as e:
        ctx.linear_mx8(a, a, None, y, K, epi=vit.EPI_BIAS_RESIDUAL)   # residual missing
    assert e.value.code == 1
    with pytest.raises(vit.VitError) as e:
        ctx.linear_mx8((a[0].view(-1)[1:], a[1]), a, None, y, K)      # misaligned codes
    assert e.value.code == 1
    with pytest.raises(vit.VitError) as e:                         # misaligned input rows
        xm = torch.empty(M * K + 8, dtype=torch.bfloat16, device="cuda")[1:1 + M * K].view(M, K)
        ctx.mx8_quantize(xm, a[0], a[1])
    assert e.value.code == 1
    f32 = vit.Context(256, 4, 64, 1024, vit.F32)
    try:
        with pytest.raises(vit.VitError) as e:
            f32.mx8_quantize(x, a[0], a[1])
        assert e.value.code == 3
    finally:
        f32.close()
    # M = 0 with valid pointers: VIT_OK and no launch (an empty torch view
    # has a null data pointer, so the C entry is called directly)
    ctx.profile_read(reset=True)
    code = vit.lib.vit_linear_mx8(ctx._h, a[0].data_ptr(), a[1].data_ptr(), a[0].data_ptr(),
                                  a[1].data_ptr(), None, None, y.data_ptr(), 0, N, K,
                                  vit.EPI_BIAS, None)
    assert code == 0
    assert ctx.profile_read(reset=True)["gemm_mx8"][0] == 0
    assert ctx.device_status() == 0
