"""fp64 full-sequence causal forward in torch (test infrastructure, not product code).

The same statement of the decoder as ``naive.causal_forward`` -- whole matrices, float64,
the attention of every position at once with a causal mask over an optional KV prefix --
written with torch so that it can run on a GPU for the large workloads. It widens one
layer's bf16 weights to float64 at a time, so an 8B model never needs its float64 copy
whole (60 GB). It shares no code with the CUDA decode library (torch matrix products are
library steps). It is pinned to ``naive.causal_forward`` on the tiny model with and without
a prefix (tests/test_oracle.py).

Why it exists: the C oracle sums every dot product in ascending order in fp32, and over
rows of 4096-14336 terms (the 2B and 8B shapes) that order loses up to ~3e-3 of relative
accuracy in the logits at some steps. The full-size parity tests therefore measure both the
GPU and the oracle against this float64 forward: the GPU must be within the tolerance of the
exact result, and within the tolerance of the oracle widened to twice the oracle's own error.

Conventions as in ``naive.py``: rotate-half RoPE (pairs i, i + hd/2, frequency
theta^(-2i/hd), angles in float64), q head h reads kv head floor(h * Hkv / Hq), scale
1/sqrt(hd), RMSNorm x / sqrt(mean(x^2) + eps) * g, SwiGLU silu(gate) * up, untied LM head;
with ``round_kv`` the K (after RoPE) and V rows are rounded to bf16 through fp32, as a
decoder that keeps a bf16 cache of fp32 activations does.
"""

from __future__ import annotations

import math

import numpy as np


def causal_forward(dims: dict, weights: dict, tokens, pos0: int = 0, kv_prefix=None, round_kv: bool = True,
                   device: str = "cpu") -> np.ndarray:
    """Logits [n][V] (float64, numpy) of every position of ``tokens`` placed at pos0, pos0 + 1, ...

    weights: bf16 torch tensors (any device). kv_prefix: optional (K, V) bf16 [L][Hkv][pos0][hd]
    holding positions [0, pos0)."""
    import torch
    f64 = torch.float64
    dev = torch.device(device)
    L, d = dims["n_layers"], dims["d_model"]
    Hq, Hkv, hd = dims["n_heads"], dims["n_kv_heads"], dims["head_dim"]
    eps, theta = float(dims["rms_eps"]), float(dims["rope_theta"])
    tok = torch.as_tensor(np.asarray(tokens, np.int64), device=dev)
    n = tok.numel()
    if kv_prefix is None:
        assert pos0 == 0
    else:
        assert kv_prefix[0].shape[2] == pos0

    def w64(t):
        return t.to(dev).to(f64)

    def rms(x, g):
        return x / torch.sqrt((x * x).mean(dim=-1, keepdim=True) + eps) * w64(g)

    def to_bf16_values(x):
        return x.to(torch.float32).to(torch.bfloat16).to(f64)

    positions = torch.arange(pos0, pos0 + n, dtype=f64, device=dev)
    freq = theta ** (-2.0 * torch.arange(hd // 2, dtype=f64, device=dev) / hd)
    ang = positions[:, None] * freq[None, :]
    cos, sin = torch.cos(ang)[:, None, :], torch.sin(ang)[:, None, :]

    def rope(x):  # [n][H][hd]
        a, b = x[..., : hd // 2], x[..., hd // 2:]
        return torch.cat([a * cos - b * sin, b * cos + a * sin], dim=-1)

    key_pos = torch.arange(pos0 + n, device=dev)
    mask = key_pos[None, :] <= (pos0 + torch.arange(n, device=dev))[:, None]  # [n][T]
    group = [h * Hkv // Hq for h in range(Hq)]

    x = w64(weights["embed"][tok.to(weights["embed"].device)])  # [n][d]
    for l in range(L):
        xn = rms(x, weights["attn_norm"][l])
        q = rope((xn @ w64(weights["wq"][l]).T).reshape(n, Hq, hd))
        k = rope((xn @ w64(weights["wk"][l]).T).reshape(n, Hkv, hd))
        v = (xn @ w64(weights["wv"][l]).T).reshape(n, Hkv, hd)
        if round_kv:
            k, v = to_bf16_values(k), to_bf16_values(v)
        if kv_prefix is not None:
            K = torch.cat([w64(kv_prefix[0][l]), k.transpose(0, 1)], dim=1)  # [Hkv][T][hd]
            V = torch.cat([w64(kv_prefix[1][l]), v.transpose(0, 1)], dim=1)
        else:
            K, V = k.transpose(0, 1), v.transpose(0, 1)
        o = torch.empty(n, Hq, hd, dtype=f64, device=dev)
        for h in range(Hq):
            s = (q[:, h, :] @ K[group[h]].T) / math.sqrt(hd)  # [n][T]
            s = s.masked_fill(~mask, float("-inf"))
            p = torch.softmax(s, dim=1)
            o[:, h, :] = p @ V[group[h]]
        x = x + o.reshape(n, Hq * hd) @ w64(weights["wo"][l]).T
        xn = rms(x, weights["ffn_norm"][l])
        gt = xn @ w64(weights["wg"][l]).T
        up = xn @ w64(weights["wu"][l]).T
        x = x + ((gt / (1.0 + torch.exp(-gt))) * up) @ w64(weights["wd"][l]).T
    xn = rms(x, weights["final_norm"])
    out = torch.empty(n, weights["lm_head"].shape[0], dtype=f64, device=dev)
    step = 16384
    for r0 in range(0, out.shape[1], step):  # the LM head a slice of rows at a time
        out[:, r0:r0 + step] = xn @ w64(weights["lm_head"][r0:r0 + step]).T
    return out.cpu().numpy()
