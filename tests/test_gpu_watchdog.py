"""Failure detection on a GPU without a fault: a bounded wait inside the
tcgen05 GEMM is made to run out, and the kernel must end, free its tensor
memory and report VIT_ERR_TIMEOUT through the context's status word, after
which the context keeps working.

The wait is made unreachable by fault injection on the host side
(vit_debug_lost_tx): the stage barrier of the one-CTA GEMM is told to expect
more bytes than its copies deliver.  Nothing traps, no address is invalid and
every wait involved ends by its own time limit (2 s per wait)."""
import time

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

vit = pytest.importorskip("vision_transformer_encoder_layernorm_b200")

TIMEOUT = 6  # VIT_ERR_TIMEOUT


def _operands(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    w = (0.05 * torch.randn(N, K, generator=g)).to(torch.bfloat16).cuda()
    b = (0.01 * torch.randn(N, generator=g)).to(torch.bfloat16).cuda()
    return x, w, b


def _check_product(x, w, b, y):
    ref = x.double() @ w.double().T + b.double()
    err = (y.double() - ref).abs().max().item() / ref.abs().max().item()
    assert err <= 1e-2, err


def test_unreachable_stage_barrier_times_out_and_context_recovers():
    ctx = vit.Context(1152, 16, 72, 4304, vit.BF16)
    M, N, K = 64, 128, 256                      # <= 128 rows: the one-CTA kernel
    x, w, b = _operands(M, N, K, 5)
    y = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    ctx.linear(x, w, b, y)                      # a normal call first
    assert ctx.device_status() == 0
    _check_product(x, w, b, y)

    ctx.debug_lost_tx(16)
    t0 = time.monotonic()
    ctx.linear(x, w, b, y)                      # the launch itself succeeds
    status = ctx.device_status()                # synchronises: the kernel has ended
    waited = time.monotonic() - t0
    assert status == TIMEOUT, vit.lib.vit_status_string(status)
    assert 1.5 <= waited <= 30.0, waited        # one 2 s wait ran out, bounded drains

    ctx.debug_lost_tx(0)                        # injection off: the context still works
    y.zero_()
    ctx.linear(x, w, b, y)
    assert ctx.device_status() == 0
    _check_product(x, w, b, y)
    # and the status word was cleared by the read above
    assert ctx.device_status() == 0
    ctx.close()


def test_fault_injection_argument_checked():
    ctx = vit.Context(1152, 16, 72, 4304, vit.BF16)
    with pytest.raises(vit.VitError) as e:
        ctx.debug_lost_tx(65537)
    assert e.value.code == 1
    ctx.close()
