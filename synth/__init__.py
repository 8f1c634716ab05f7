"""Seeded synthetic inputs for batch-1 decode: workload shapes, weights, prompts, KV caches.

This module holds no arithmetic of the decode method. It only defines the workload shapes
and draws seeded random tensors; the oracle and the CUDA library both receive the very
same bytes from here. The bytes, not the random number generator, are the contract:
``tensor_digest`` gives a SHA-256 of each tensor so runs can be compared.

Workloads (a dense decoder-only transformer with RMSNorm, GQA attention with RoPE, a
SwiGLU FFN and an untied LM head; greedy decode of a single request):

* ``tiny``   -- 2 layers, d 256, 4/2 heads of 64, FFN 1024, vocab 4096; 16-token prompt,
  64 generated tokens.
* ``0.5b``   -- 16 layers, d 1536, 12/4 heads of 128, FFN 4096, vocab 32000; 128-token
  prompt, 256 generated tokens.
* ``2b-4k``  -- 28 layers, d 2048, 16/8 heads of 128, FFN 8192, vocab 32000 (the pages'
  "2B model" shape); 4096 cached positions of N(0,1) K/V, 1024 generated tokens.
* ``2b-32k`` -- the same model with 32768 cached positions, 512 generated tokens.
* ``8b-4k``  -- 32 layers, d 4096, 32/8 heads of 128, FFN 14336, vocab 128256, RoPE theta
  500000; 4096 cached positions, 512 generated tokens.

Recipe: every weight matrix (embedding and LM head included) is N(0, 0.02) drawn in fp32
and rounded to bf16; norm gains are 1.0. Weights use seed 0, prompt / start token seed 1,
the KV cache seed 2. Matrices are drawn in a fixed order, one layer slice at a time, so the
result does not depend on how much memory is free. Shapes up to ``0.5b`` draw on the CPU
generator; the larger ones draw on the CUDA generator (same order), because drawing 4-16 GB
on one CPU thread takes minutes. Random-KV workloads fill positions [0, P) of K and V with
N(0, 1) in bf16 (K is taken as already rotated) and start decoding at position P from one
seeded uniform token id.
"""

from __future__ import annotations

import hashlib
from dataclasses import dataclass, asdict

import torch

__all__ = ["Workload", "WORKLOADS", "get", "make_weights", "make_prompt", "make_kv",
           "tensor_digest", "WEIGHT_KEYS", "generator_device"]


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn_dim: int
    vocab: int
    rms_eps: float = 1e-5
    rope_theta: float = 10000.0
    prompt_len: int = 0      # prompt tokens run through the decode step (0: random-KV workload)
    kv_len: int = 0          # pre-filled KV positions (random-KV workloads)
    n_gen: int = 64          # generated tokens

    @property
    def n_pending(self) -> int:
        """Tokens fed before the first generated one: the prompt, or the one start token."""
        return self.prompt_len if self.prompt_len > 0 else 1

    @property
    def start_pos(self) -> int:
        return self.kv_len

    @property
    def n_steps(self) -> int:
        """Decode steps (forward passes) to produce n_gen tokens."""
        return self.n_pending + self.n_gen - 1

    @property
    def capacity(self) -> int:
        """KV positions needed: every step appends one entry."""
        return self.start_pos + self.n_steps

    def dims(self) -> dict:
        d = asdict(self)
        for k in ("name", "prompt_len", "kv_len", "n_gen"):
            d.pop(k)
        return d

    def replace(self, **kw) -> "Workload":
        d = asdict(self)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "tiny": Workload("tiny", 2, 256, 4, 2, 64, 1024, 4096, prompt_len=16, n_gen=64),
    "0.5b": Workload("0.5b", 16, 1536, 12, 4, 128, 4096, 32000, prompt_len=128, n_gen=256),
    "2b-4k": Workload("2b-4k", 28, 2048, 16, 8, 128, 8192, 32000, kv_len=4096, n_gen=1024),
    "2b-32k": Workload("2b-32k", 28, 2048, 16, 8, 128, 8192, 32000, kv_len=32768, n_gen=512),
    "8b-4k": Workload("8b-4k", 32, 4096, 32, 8, 128, 14336, 128256, rope_theta=500000.0,
                      kv_len=4096, n_gen=512),
}

# Stacked weight tensors, in drawing order. Shapes: see ``weight_shapes``.
WEIGHT_KEYS = ("embed", "attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "wg", "wu", "wd",
               "final_norm", "lm_head")


def get(name: str) -> Workload:
    return WORKLOADS[name]


def weight_shapes(w: Workload) -> dict:
    L, d, F, V = w.n_layers, w.d_model, w.ffn_dim, w.vocab
    qd, kd = w.n_heads * w.head_dim, w.n_kv_heads * w.head_dim
    return {
        "embed": (V, d), "attn_norm": (L, d), "wq": (L, qd, d), "wk": (L, kd, d),
        "wv": (L, kd, d), "wo": (L, d, qd), "ffn_norm": (L, d), "wg": (L, F, d),
        "wu": (L, F, d), "wd": (L, d, F), "final_norm": (d,), "lm_head": (V, d),
    }


def generator_device(w: Workload) -> str:
    """CPU for shapes up to 0.5B, CUDA above (same drawing order either way)."""
    n = sum(int(torch.Size(s).numel()) for s in weight_shapes(w).values())
    return "cpu" if n <= 600_000_000 else "cuda"


def _normal_bf16(shape, std, gen, device) -> torch.Tensor:
    return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std).to(
        torch.bfloat16)


def make_weights(w: Workload, seed: int = 0, device: str | None = None) -> dict:
    """All weights as bf16 tensors on ``device`` (default: ``generator_device``)."""
    device = device or generator_device(w)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    shapes = weight_shapes(w)
    out = {}
    for key in WEIGHT_KEYS:
        shape = shapes[key]
        if key.endswith("norm"):
            out[key] = torch.ones(shape, dtype=torch.bfloat16, device=device)
        elif len(shape) == 3:  # one layer slice at a time
            t = torch.empty(shape, dtype=torch.bfloat16, device=device)
            for l in range(shape[0]):
                t[l] = _normal_bf16(shape[1:], 0.02, gen, device)
            out[key] = t
        else:
            out[key] = _normal_bf16(shape, 0.02, gen, device)
    return out


def make_prompt(w: Workload, seed: int = 1) -> torch.Tensor:
    """int32 token ids fed before generation: the prompt, or the single start token."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return torch.randint(0, w.vocab, (w.n_pending,), generator=gen, dtype=torch.int64).to(torch.int32)


def make_tokens(w: Workload, n: int, seed: int = 3) -> torch.Tensor:
    """n uniform token ids, e.g. a forced input sequence for teacher-forced parity runs."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return torch.randint(0, w.vocab, (n,), generator=gen, dtype=torch.int64).to(torch.int32)


def make_kv(w: Workload, seed: int = 2, device: str | None = None, n_pos: int | None = None):
    """Pre-filled cache: (K, V), each bf16 [L][Hkv][P][hd] drawn from N(0, 1).

    Drawn layer by layer, K before V."""
    n_pos = w.kv_len if n_pos is None else n_pos
    device = device or generator_device(w)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    shape = (w.n_kv_heads, n_pos, w.head_dim)
    K = torch.empty((w.n_layers,) + shape, dtype=torch.bfloat16, device=device)
    V = torch.empty_like(K)
    for l in range(w.n_layers):
        K[l] = _normal_bf16(shape, 1.0, gen, device)
        V[l] = _normal_bf16(shape, 1.0, gen, device)
    return K, V


def tensor_digest(t: torch.Tensor) -> str:
    """SHA-256 of a tensor's raw bytes (moved to the CPU)."""
    b = t.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes()
    return hashlib.sha256(b).hexdigest()
