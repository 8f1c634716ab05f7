"""Temperature sampling on the oracle side (test infrastructure, not product code).

The pages put sampling inside the monokernel, with no trip to the CPU ("3000 tokens per
second: how to speed up LLMs on ordinary GPUs", aikraft.ru, section 04 "Monokernel"), and
name no sampling rule. The reading taken here: a generated token is drawn from
softmax(logits / T) by the Gumbel-max rule -- the argmax over the vocabulary of
logit_i / T + g_i with g_i = -log(-log(u_i)) and u_i uniform on (0, 1) -- which draws exactly
from that distribution. T = 0 means greedy argmax. Ties go to the lowest index, as in greedy.

The uniforms come from a counter-based generator, so that the GPU and this oracle draw the
same numbers without passing them around: Philox4x32-10 as published by Salmon, Moraes, Dror
and Shaw ("Parallel random numbers: as easy as 1, 2, 3", SC 2011): a 128-bit counter and a
64-bit key, ten rounds, each round two 32x32 -> 64-bit products with the multipliers
0xD2511F53 and 0xCD9E8D57, the key bumped between rounds by 0x9E3779B9 and 0xBB67AE85.
Stream layout (the same on both sides): key = (seed mod 2^32, seed div 2^32); vocabulary
index i at absolute position p uses output word i mod 4 of the counter (i div 4, p, 0, 0);
u = (top 23 bits + 0.5) / 2^23, exact in fp32 and never 0 or 1 (with 24 bits, k + 0.5 rounds
for k >= 2^23 and u can reach 1, where g is infinite). The perturbed values are formed in fp32
(logit * (1/T) + g, 1/T itself an fp32 division), the precision the kernel decides the argmax
in.

Written with numpy; shares no code with the CUDA library.
"""

from __future__ import annotations

import numpy as np

M0, M1 = 0xD2511F53, 0xCD9E8D57
W0, W1 = 0x9E3779B9, 0xBB67AE85
MASK = 0xFFFFFFFF


def _mulhilo(a: int, b: np.ndarray):
    p = np.uint64(a) * b.astype(np.uint64)
    return (p >> np.uint64(32)).astype(np.uint32), (p & np.uint64(MASK)).astype(np.uint32)


def philox4x32_round(c, k):
    """One round on counter words c = (c0, c1, c2, c3) (uint32 arrays) with key k = (k0, k1)."""
    hi0, lo0 = _mulhilo(M0, c[0])
    hi1, lo1 = _mulhilo(M1, c[2])
    return (hi1 ^ c[1] ^ np.uint32(k[0]), lo1, hi0 ^ c[3] ^ np.uint32(k[1]), lo0)


def philox4x32(counter, key, rounds: int = 10):
    """Philox4x32 with `rounds` rounds. counter: 4 uint32 arrays (broadcastable); key: 2 ints."""
    c = tuple(np.asarray(x, np.uint32) for x in counter)
    k0, k1 = int(key[0]) & MASK, int(key[1]) & MASK
    for r in range(rounds):
        if r > 0:
            k0, k1 = (k0 + W0) & MASK, (k1 + W1) & MASK
        c = philox4x32_round(c, (k0, k1))
    return c


def uniforms(seed: int, pos: int, n: int) -> np.ndarray:
    """u_i in (0, 1), fp32, for vocabulary indices 0 .. n-1 at absolute position pos."""
    i = np.arange(n, dtype=np.uint64)
    blk = (i >> np.uint64(2)).astype(np.uint32)
    z = np.zeros_like(blk)
    out = philox4x32((blk, np.full_like(blk, pos & MASK), z, z), (seed & MASK, (seed >> 32) & MASK))
    words = np.stack(out, axis=1)  # [n][4]
    w = words[np.arange(n), (i & np.uint64(3)).astype(np.int64)]
    return ((w >> np.uint32(9)).astype(np.float32) + np.float32(0.5)) * np.float32(2.0 ** -23)


def gumbel(seed: int, pos: int, n: int) -> np.ndarray:
    """g_i = -log(-log(u_i)), fp32."""
    u = uniforms(seed, pos, n)
    return -np.log(-np.log(u))


def sample(logits, pos: int, temperature: float, seed: int) -> int:
    """The token drawn at absolute position pos from fp32 logits [V]: argmax of
    logit * (1/T) + g (lowest index on a tie); plain argmax at T = 0."""
    y = np.asarray(logits, np.float32)
    if temperature <= 0:
        return int(np.argmax(y))
    z = y * (np.float32(1.0) / np.float32(temperature)) + gumbel(seed, pos, y.size)
    return int(np.argmax(z))


def perturbed(logits, pos: int, temperature: float, seed: int) -> np.ndarray:
    """The values the sampled token is the argmax of (for margin checks)."""
    y = np.asarray(logits, np.float32)
    if temperature <= 0:
        return y
    return y * (np.float32(1.0) / np.float32(temperature)) + gumbel(seed, pos, y.size)
