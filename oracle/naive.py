"""Independent fp64 full-sequence causal forward (test infrastructure, not product code).

A second statement of the same decoder, written the other way round from ``oracle.c``:
whole matrices instead of scalar loops, float64 instead of float32, and the attention of
every position computed at once over the full sequence with a causal mask instead of
step by step against a KV cache. Row t of its output must equal decode step t of the
C oracle (KV-cache decode is an exact reorganisation of the causal forward; the pages
require the engine to keep the model's output exact -- "Kog inference engine: no
precision cut, 3000 tokens/s per request", zdabc.icu, opening section).

With ``round_kv=True`` the K (after RoPE) and V rows are rounded to bf16 before use,
through fp32 first, as a decoder that stores a bf16 cache of fp32 activations does. With
``round_kv=False`` this is the plain fp64 model, which a library Llama-style
implementation in fp64 must reproduce.

Conventions (the pages are silent on all of them): rotate-half RoPE with frequency
theta^(-2i/hd) on pairs (i, i+hd/2); q head h uses kv head floor(h*Hkv/Hq); scale
1/sqrt(hd); RMSNorm x/sqrt(mean(x^2)+eps)*g; SwiGLU silu(gate)*up; untied LM head.
"""

from __future__ import annotations

import numpy as np


def _f64(t) -> np.ndarray:
    """bf16 tensor or uint16 bit-pattern array -> float64 array."""
    if not isinstance(t, np.ndarray):
        import torch
        t = t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    return (t.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _to_bf16_values(x: np.ndarray) -> np.ndarray:
    """Round float64 values to fp32 (nearest) and then to bf16 (nearest, ties to even)."""
    f = np.ascontiguousarray(x, np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _rms(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * g


def _rope_tables(positions: np.ndarray, hd: int, theta: float):
    i = np.arange(hd // 2, dtype=np.float64)
    freq = theta ** (-2.0 * i / hd)
    ang = positions.astype(np.float64)[:, None] * freq[None, :]
    return np.cos(ang), np.sin(ang)


def _rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """x [n][H][hd]; rotate pairs (i, i+hd/2) by the angle of each row's position."""
    h = x.shape[-1] // 2
    a, b = x[..., :h], x[..., h:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def causal_forward(dims: dict, weights: dict, tokens, pos0: int = 0, kv_prefix=None,
                   round_kv: bool = True) -> np.ndarray:
    """Logits [n][V] (float64) of every position of ``tokens`` placed at pos0, pos0+1, ...

    kv_prefix: optional (K, V) bf16 [L][Hkv][pos0][hd] occupying positions [0, pos0)."""
    L, d = dims["n_layers"], dims["d_model"]
    Hq, Hkv, hd = dims["n_heads"], dims["n_kv_heads"], dims["head_dim"]
    eps, theta = dims["rms_eps"], dims["rope_theta"]
    tokens = np.asarray(tokens, np.int64)
    n = tokens.size
    W = {k: _f64(v) for k, v in weights.items()}
    if kv_prefix is not None:
        Kp, Vp = _f64(kv_prefix[0]), _f64(kv_prefix[1])
        assert Kp.shape[2] == pos0
    else:
        assert pos0 == 0
        Kp = Vp = np.zeros((L, Hkv, 0, hd))
    positions = pos0 + np.arange(n)
    cos, sin = _rope_tables(positions, hd, theta)
    # causal mask over all cached positions: row i sees key positions <= pos0 + i
    key_pos = np.arange(pos0 + n)
    mask = key_pos[None, :] <= positions[:, None]
    group = np.arange(Hq) * Hkv // Hq

    x = W["embed"][tokens]                                     # [n][d]
    for l in range(L):
        xn = _rms(x, W["attn_norm"][l], eps)
        q = (xn @ W["wq"][l].T).reshape(n, Hq, hd)
        k = (xn @ W["wk"][l].T).reshape(n, Hkv, hd)
        v = (xn @ W["wv"][l].T).reshape(n, Hkv, hd)
        q, k = _rope(q, cos, sin), _rope(k, cos, sin)
        if round_kv:
            k, v = _to_bf16_values(k), _to_bf16_values(v)
        K = np.concatenate([Kp[l], k.transpose(1, 0, 2)], axis=1)  # [Hkv][T][hd]
        V = np.concatenate([Vp[l], v.transpose(1, 0, 2)], axis=1)
        o = np.empty((n, Hq, hd))
        for h in range(Hq):
            s = (q[:, h, :] @ K[group[h]].T) / np.sqrt(hd)           # [n][T]
            s = np.where(mask, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            o[:, h, :] = p @ V[group[h]]
        x = x + o.reshape(n, Hq * hd) @ W["wo"][l].T
        xn = _rms(x, W["ffn_norm"][l], eps)
        gt = xn @ W["wg"][l].T
        up = xn @ W["wu"][l].T
        x = x + ((gt / (1.0 + np.exp(-gt))) * up) @ W["wd"][l].T
    return _rms(x, W["final_norm"], eps) @ W["lm_head"].T
