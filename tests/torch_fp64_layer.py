"""An independent restatement of one encoder layer with PyTorch CPU library
routines (layer_norm, linear, gelu, scaled_dot_product_attention) and 2D
RoPE written as a complex-number rotation.  In fp64 it pins the oracle, with
which it shares no code; in fp32 the benchmark times it as the CPU figure at
the pages' own precision."""
import torch
import torch.nn.functional as F


def rope2d_complex(x, pos_rc, theta, dtype=torch.float64):
    # x [T, H, d]; each half of the head is viewed as h/2 complex numbers
    # (dim j, dim j + h/2) and multiplied by exp(i * p * theta^(-2j/h)).
    T, H, d = x.shape
    h = d // 2
    out = []
    for axis in range(2):
        half = x[..., axis * h:(axis + 1) * h]
        z = torch.complex(half[..., : h // 2], half[..., h // 2:])
        j = torch.arange(h // 2, dtype=dtype)
        freq = theta ** (-(2.0 * j) / h)
        ang = pos_rc[:, axis].to(dtype)[:, None] * freq[None, :]
        z = z * torch.polar(torch.ones_like(ang), ang)[:, None, :]
        out.append(torch.cat([z.real, z.imag], dim=-1))
    return torch.cat(out, dim=-1)


def layer(x, w, cu_seqlens, pos_rc, heads, head_dim, eps, theta,
          prefix_kv=None, attn_only=False, dtype=torch.float64):
    t = {k: torch.as_tensor(v, dtype=dtype) for k, v in w.items()}
    x = torch.as_tensor(x, dtype=dtype)
    T, C = x.shape
    h = F.layer_norm(x, (C,), t["ln1_g"], t["ln1_b"], eps)
    qkv = F.linear(h, t["w_qkv"], t["b_qkv"]).view(T, 3, heads, head_dim)
    q, k, v = qkv[:, 0], qkv[:, 1], qkv[:, 2]
    if pos_rc is not None:
        pos = torch.as_tensor(pos_rc)
        q = rope2d_complex(q, pos, theta, dtype)
        k = rope2d_complex(k, pos, theta, dtype)
    o = torch.empty_like(q)
    cu = [int(c) for c in cu_seqlens]
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        ks, vs = k[a:b], v[a:b]
        if prefix_kv is not None:
            p = torch.as_tensor(prefix_kv[s], dtype=dtype)
            g = heads // p.shape[2]
            ks = torch.cat([p[0].repeat_interleave(g, dim=1), ks], 0)
            vs = torch.cat([p[1].repeat_interleave(g, dim=1), vs], 0)
        o[a:b] = F.scaled_dot_product_attention(
            q[a:b].transpose(0, 1), ks.transpose(0, 1), vs.transpose(0, 1)
        ).transpose(0, 1)
    x1 = x + F.linear(o.reshape(T, C), t["w_o"], t["b_o"])
    if attn_only:
        return x1.numpy()
    h2 = F.layer_norm(x1, (C,), t["ln2_g"], t["ln2_b"], eps)
    g = F.gelu(F.linear(h2, t["w_fc1"], t["b_fc1"]), approximate="tanh")
    return (x1 + F.linear(g, t["w_fc2"], t["b_fc2"])).numpy()


def projector(x, w, eps, dtype=torch.float64):
    # LayerNorm, linear + GELU (tanh), linear, with PyTorch's library routines
    t = {k: torch.as_tensor(v, dtype=dtype) for k, v in w.items()}
    x = torch.as_tensor(x, dtype=dtype)
    h = F.layer_norm(x, (x.shape[1],), t["ln_g"], t["ln_b"], eps)
    g = F.gelu(F.linear(h, t["w1"], t["b1"]), approximate="tanh")
    return F.linear(g, t["w2"], t["b2"]).numpy()
