"""Helpers shared by the GPU parity tests: seeded synth inputs -> device
tensors, and the error metrics (max-relative and cosine, in fp64)."""
import numpy as np
import torch

import synth


def to_dev(a, dtype: str, device="cuda"):
    """Storage-dtype numpy array (float32, or uint16 bf16 bits) -> device tensor."""
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def from_dev(t) -> np.ndarray:
    """Device tensor (fp32 or bf16) -> fp64 numpy (exact)."""
    return t.detach().to(torch.float64).cpu().numpy()


def int_dev(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def metrics(y, r):
    y = np.asarray(y, dtype=np.float64).ravel()
    r = np.asarray(r, dtype=np.float64).ravel()
    rel = float(np.max(np.abs(y - r)) / max(np.max(np.abs(r)), 1e-300))
    cos = float(np.dot(y, r) / max(np.linalg.norm(y) * np.linalg.norm(r), 1e-300))
    return rel, cos


def assert_close(y, r, rel_max, cos_min=None, what=""):
    rel, cos = metrics(y, r)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    assert rel <= rel_max, f"{what}: rel {rel:.3e} > {rel_max:.1e} (cos {cos:.7f})"
    if cos_min is not None:
        assert cos >= cos_min, f"{what}: cos {cos:.7f} < {cos_min} (rel {rel:.3e})"
    return rel, cos


def layer_dev(inputs, i, device="cuda"):
    dt = inputs.workload.dtype
    return {k: (to_dev(v, dt, device) if v.size else None) for k, v in inputs.layers[i].items()}


def dtype_code(dt):
    import vision_transformer_encoder_layernorm_b200 as vit
    return vit.F32 if dt == "f32" else vit.BF16


def context_for(wl, **kw):
    import vision_transformer_encoder_layernorm_b200 as vit
    flags = 0
    if wl.attn_only:
        flags |= vit.FLAG_NO_MLP
    if not wl.rope:
        flags |= vit.FLAG_NO_ROPE
    return vit.Context(wl.hidden, wl.heads, wl.head_dim, wl.mlp if not wl.attn_only else 0,
                       dtype_code(wl.dtype), wl.ln_eps, wl.rope_theta, flags, **kw)
