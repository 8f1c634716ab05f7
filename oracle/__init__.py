"""CPU oracle for batch-1 decode (test infrastructure, not product code).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg import
this package. The CUDA decode library never imports, links or runs it; the two share no
code. What the oracle computes and how each part is pinned is stated at the top of
``oracle.c`` (the C reference) and ``naive.py`` (an independent fp64 full-sequence forward).

``Oracle`` wraps the C library through ctypes. Weights are passed as bf16 tensors or uint16
arrays holding bf16 bit patterns; the wrapper keeps references so the C side can read them
in place.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# Strict IEEE fp32: no fused multiply-add contraction, no fast-math reassociation.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-pthread"]


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc into ``out`` (default: oracle/liboracle.so)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


class _Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim", "ffn_dim", "vocab",
        "capacity", "n_threads")] + [("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float)]


_WKEYS = ("embed", "attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "wg", "wu", "wd",
          "final_norm", "lm_head")


class _Weights(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in _WKEYS]


_u16p = ctypes.POINTER(ctypes.c_uint16)
_f32p = ctypes.POINTER(ctypes.c_float)


def load(path: str | None = None) -> ctypes.CDLL:
    lib = ctypes.CDLL(path or build())
    lib.orc_new.restype = ctypes.c_void_p
    lib.orc_new.argtypes = [ctypes.POINTER(_Config)]
    lib.orc_free.argtypes = [ctypes.c_void_p]
    lib.orc_set_weights.argtypes = [ctypes.c_void_p, ctypes.POINTER(_Weights)]
    lib.orc_set_kv.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
                               ctypes.c_int32]
    lib.orc_get_kv.argtypes = lib.orc_set_kv.argtypes
    lib.orc_step.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
                             ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_double)]
    lib.orc_bf16_to_f32.restype = ctypes.c_float
    lib.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
    lib.orc_bf16_round.restype = ctypes.c_uint16
    lib.orc_bf16_round.argtypes = [ctypes.c_float]
    lib.orc_silu.restype = ctypes.c_float
    lib.orc_silu.argtypes = [ctypes.c_float]
    lib.orc_argmax.restype = ctypes.c_int32
    lib.orc_argmax.argtypes = [ctypes.c_void_p, ctypes.c_int32]
    lib.orc_rmsnorm.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_float,
                                ctypes.c_void_p]
    lib.orc_rope.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_float]
    lib.orc_matvec.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                               ctypes.c_void_p]
    lib.orc_attend.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                               ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
    return lib


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load()
    return _lib


def as_u16(t) -> np.ndarray:
    """bf16 torch tensor (any device) or uint16 array -> contiguous uint16 numpy array."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch
    assert t.dtype == torch.bfloat16, t.dtype
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


# ---------------------------------------------------------------- stage functions

def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    return (np.asarray(u16, np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32)
    return np.array([lib().orc_bf16_round(float(v)) for v in x.ravel()], np.uint16).reshape(x.shape)


def silu(z: float) -> float:
    return lib().orc_silu(z)


def argmax(v: np.ndarray) -> int:
    v = np.ascontiguousarray(v, np.float32)
    return lib().orc_argmax(_ptr(v), v.size)


def rmsnorm(x: np.ndarray, g_u16: np.ndarray, eps: float) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32)
    g = np.ascontiguousarray(g_u16, np.uint16)
    out = np.empty_like(x)
    lib().orc_rmsnorm(_ptr(x), _ptr(g), x.size, eps, _ptr(out))
    return out


def rope(v: np.ndarray, pos: int, theta: float) -> np.ndarray:
    v = np.array(v, np.float32, copy=True)
    lib().orc_rope(_ptr(v), v.size, pos, theta)
    return v


def matvec(W_u16: np.ndarray, x: np.ndarray) -> np.ndarray:
    W = np.ascontiguousarray(W_u16, np.uint16)
    x = np.ascontiguousarray(x, np.float32)
    y = np.empty(W.shape[0], np.float32)
    lib().orc_matvec(_ptr(W), _ptr(x), W.shape[0], W.shape[1], _ptr(y))
    return y


def attend(q: np.ndarray, K_u16: np.ndarray, V_u16: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, np.float32)
    K = np.ascontiguousarray(K_u16, np.uint16)
    V = np.ascontiguousarray(V_u16, np.uint16)
    T, hd = K.shape
    out = np.empty(hd, np.float32)
    scratch = np.empty(max(T, 1), np.float32)
    lib().orc_attend(_ptr(q), _ptr(K), _ptr(V), T, hd, _ptr(out), _ptr(scratch))
    return out


# ---------------------------------------------------------------- decoder

class Oracle:
    """Step-by-step decoder with its own KV cache (fp32 math over bf16 weights)."""

    def __init__(self, dims: dict, weights: dict, capacity: int, n_threads: int = 1,
                 library: ctypes.CDLL | None = None):
        self._lib = library or lib()
        self.dims = dict(dims)
        self.capacity = int(capacity)
        c = _Config(dims["n_layers"], dims["d_model"], dims["n_heads"], dims["n_kv_heads"],
                    dims["head_dim"], dims["ffn_dim"], dims["vocab"], self.capacity,
                    int(n_threads), float(dims["rms_eps"]), float(dims["rope_theta"]))
        self._h = self._lib.orc_new(ctypes.byref(c))
        if not self._h:
            raise ValueError("oracle rejected config %r" % (dims,))
        self._w = {k: as_u16(weights[k]) for k in _WKEYS}
        w = _Weights(*[_ptr(self._w[k]) for k in _WKEYS])
        if self._lib.orc_set_weights(self._h, ctypes.byref(w)) != 0:
            raise ValueError("oracle rejected weights")

    def close(self):
        if getattr(self, "_h", None):
            self._lib.orc_free(self._h)
            self._h = None

    __del__ = close

    def set_kv(self, K, V):
        """Pre-fill positions [0, P) of every layer: K, V bf16 [L][Hkv][P][hd]."""
        K, V = as_u16(K), as_u16(V)
        P = K.shape[2]
        for l in range(K.shape[0]):
            for which, arr in ((0, K[l]), (1, V[l])):
                a = np.ascontiguousarray(arr)
                if self._lib.orc_set_kv(self._h, l, which, _ptr(a), P) != 0:
                    raise ValueError("bad KV fill")

    def get_kv(self, layer: int, which: int, n: int) -> np.ndarray:
        hkv, hd = self.dims["n_kv_heads"], self.dims["head_dim"]
        out = np.empty((hkv, n, hd), np.uint16)
        if self._lib.orc_get_kv(self._h, layer, which, _ptr(out), n) != 0:
            raise ValueError("bad KV read")
        return out

    def step(self, token: int, pos: int, head: bool = True):
        """Run one position. Returns (logits fp32 [V] or None, argmax or None, bytes read)."""
        nb = ctypes.c_double(0.0)
        if not head:
            rc = self._lib.orc_step(self._h, int(token), int(pos), None, None, ctypes.byref(nb))
            if rc:
                raise ValueError("oracle step failed")
            return None, None, nb.value
        logits = np.empty(self.dims["vocab"], np.float32)
        nxt = ctypes.c_int32(-1)
        rc = self._lib.orc_step(self._h, int(token), int(pos), _ptr(logits), ctypes.byref(nxt),
                                ctypes.byref(nb))
        if rc:
            raise ValueError("oracle step failed")
        return logits, nxt.value, nb.value

    def forced(self, tokens, pos0: int, heads=None):
        """Feed a fixed token sequence from position pos0; logits [n][V] at every step
        (or only where ``heads[i]`` is true; other rows stay NaN)."""
        n = len(tokens)
        out = np.full((n, self.dims["vocab"]), np.nan, np.float32)
        for i, t in enumerate(tokens):
            h = True if heads is None else bool(heads[i])
            lg, _, _ = self.step(int(t), pos0 + i, head=h)
            if h:
                out[i] = lg
        return out

    def greedy(self, pending, pos0: int, n_gen: int, keep_logits: bool = True):
        """Feed ``pending`` tokens, then generate n_gen tokens greedily.

        Returns (tokens [n_gen] int32, logits [n_gen][V] of the steps that chose them)."""
        pending = [int(t) for t in pending]
        toks, logits = [], []
        pos = pos0
        for i, t in enumerate(pending[:-1]):
            self.step(t, pos, head=False)
            pos += 1
        cur = pending[-1]
        for g in range(n_gen):
            lg, nxt, _ = self.step(cur, pos, head=True)
            pos += 1
            toks.append(nxt)
            if keep_logits:
                logits.append(lg)
            cur = nxt
        return np.array(toks, np.int32), (np.stack(logits) if keep_logits else None)
