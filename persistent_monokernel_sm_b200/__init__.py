"""Python binding of libkd, the batch-1 decode monokernel library for B200 (sm_100a).

Argument marshalling only: every step of the decode path runs in libkd's CUDA kernels.
The ``kd_*`` functions mirror the C ABI in ``include/kd.h`` one to one; ``Decoder`` is a
small convenience that lets PyTorch allocate the device memory (arena, outputs) and
passes raw pointers and the current stream through. There is no CPU fallback: if libkd.so
is missing the binding raises.
"""

from __future__ import annotations

import ctypes
import os

__all__ = ["KdError", "kd_config", "kd_weights", "kd_info", "load_library", "Decoder", "config_from",
           "kd_arena_bytes", "kd_step_bytes", "kd_create", "kd_load_weights", "kd_set_kv", "kd_reset",
           "kd_decode", "kd_generate", "kd_sync", "kd_position", "kd_set_trace", "kd_set_timeout", "kd_set_sampling", "kd_decode_noalloc", "kd_get_info", "kd_kv_ptr",
           "kd_last_error", "kd_strerror", "kd_destroy", "LIB_PATH", "ERRORS"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkd.so")

ERRORS = {0: "KD_OK", -1: "KD_EINVAL", -2: "KD_ENOMEM", -3: "KD_ECAPACITY", -4: "KD_ECOOP",
          -5: "KD_ECUDA", -6: "KD_ETIMEOUT", -7: "KD_ESTATE",
          -8: "KD_ETOKEN"}


class kd_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim",
                                               "ffn_dim", "vocab", "max_seq")] + \
               [("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float)]


WEIGHT_FIELDS = ("embed", "attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "wg", "wu", "wd",
                 "final_norm", "lm_head")


class kd_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_FIELDS]


class kd_info(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("grid", "threads", "smem_bytes", "stages", "stage_bytes",
                                               "attn_pieces")] + \
               [(n, ctypes.c_int64) for n in ("arena_bytes", "weight_bytes", "kv_bytes", "launches", "ctl_offset")] + \
               [("sync_replicas", ctypes.c_int32), ("sync_offset", ctypes.c_int64 * 2)]


class KdError(RuntimeError):
    def __init__(self, code, msg=""):
        super().__init__("%s (%d): %s" % (ERRORS.get(code, "?"), code, msg))
        self.code = code


_lib = None
_P = ctypes.c_void_p
_CFG = ctypes.POINTER(kd_config)


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libkd.so (raises if it was not built: the CUDA path has no substitute)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError("libkd.so not found at %s; build it with persistent_monokernel_sm_b200/build.py"
                          % path)
    lib = ctypes.CDLL(path)
    sig = {
        "kd_arena_bytes": (ctypes.c_size_t, [_CFG]),
        "kd_step_bytes": (ctypes.c_double, [_CFG, ctypes.c_int64, ctypes.c_int]),
        "kd_create": (ctypes.c_int, [_CFG, _P, ctypes.c_size_t, _P, ctypes.POINTER(_P)]),
        "kd_load_weights": (ctypes.c_int, [_P, ctypes.POINTER(kd_weights)]),
        "kd_set_kv": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32, _P, ctypes.c_int32]),
        "kd_reset": (ctypes.c_int, [_P, _P, ctypes.c_int32, ctypes.c_int32]),
        "kd_decode": (ctypes.c_int, [_P, ctypes.c_int32, _P, _P]),
        "kd_generate": (ctypes.c_int, [_P, _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _P]),
        "kd_sync": (ctypes.c_int, [_P]),
        "kd_position": (ctypes.c_int32, [_P]),
        "kd_set_trace": (ctypes.c_int, [_P, _P, ctypes.c_int64, ctypes.c_int32]),
        "kd_set_timeout": (ctypes.c_int, [_P, ctypes.c_int64]),
        "kd_set_sampling": (ctypes.c_int, [_P, ctypes.c_float, ctypes.c_uint64]),
        "kd_decode_noalloc": (ctypes.c_int, [_P, _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _P, _P]),
        "kd_get_info": (ctypes.c_int, [_P, ctypes.POINTER(kd_info)]),
        "kd_kv_ptr": (_P, [_P, ctypes.c_int32, ctypes.c_int32]),
        "kd_last_error": (ctypes.c_char_p, [_P]),
        "kd_strerror": (ctypes.c_char_p, [ctypes.c_int]),
        "kd_destroy": (None, [_P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


# ---------------------------------------------------------------- the C ABI, same names

def kd_arena_bytes(cfg: kd_config) -> int:
    return load_library().kd_arena_bytes(ctypes.byref(cfg))


def kd_step_bytes(cfg: kd_config, kv_positions: int, with_head: bool = True) -> float:
    return load_library().kd_step_bytes(ctypes.byref(cfg), int(kv_positions), int(bool(with_head)))


def kd_create(cfg: kd_config, d_arena: int, arena_bytes: int, stream: int):
    h = _P()
    rc = load_library().kd_create(ctypes.byref(cfg), d_arena, arena_bytes, stream, ctypes.byref(h))
    if rc:
        raise KdError(rc, "kd_create")
    return h


def _check(h, rc, what):
    if rc:
        raise KdError(rc, "%s: %s" % (what, kd_last_error(h)))
    return rc


def kd_load_weights(h, w: kd_weights) -> int:
    return _check(h, load_library().kd_load_weights(h, ctypes.byref(w)), "kd_load_weights")


def kd_set_kv(h, layer: int, which: int, d_src: int, n_pos: int) -> int:
    return _check(h, load_library().kd_set_kv(h, layer, which, d_src, n_pos), "kd_set_kv")


def kd_reset(h, d_tokens: int, n_tokens: int, kv_len: int) -> int:
    return _check(h, load_library().kd_reset(h, d_tokens, n_tokens, kv_len), "kd_reset")


def kd_decode(h, n_gen: int, d_tokens_out: int, d_logits_out: int | None) -> int:
    return _check(h, load_library().kd_decode(h, n_gen, d_tokens_out, d_logits_out), "kd_decode")


def kd_generate(h, h_tokens: int, n_tokens: int, kv_len: int, n_gen: int, h_tokens_out: int) -> int:
    return _check(h, load_library().kd_generate(h, h_tokens, n_tokens, kv_len, n_gen, h_tokens_out),
                  "kd_generate")


def kd_sync(h) -> int:
    return _check(h, load_library().kd_sync(h), "kd_sync")


def kd_decode_noalloc(h, d_tokens: int, n_tokens: int, kv_len: int, n_gen: int, d_tokens_out: int,
                      d_logits_out: int | None) -> int:
    """kd_decode for callers that cannot allocate device memory: scratch lives in a fixed
    array inside libkd (see kd.h). Waits for the launch and raises on its device status."""
    return _check(h, load_library().kd_decode_noalloc(h, d_tokens, n_tokens, kv_len, n_gen, d_tokens_out,
                                                      d_logits_out), "kd_decode_noalloc")


def kd_set_timeout(h, ns: int) -> int:
    return _check(h, load_library().kd_set_timeout(h, ns), "kd_set_timeout")


def kd_set_sampling(h, temperature: float, seed: int) -> int:
    return _check(h, load_library().kd_set_sampling(h, float(temperature), int(seed) & 0xFFFFFFFFFFFFFFFF),
                  "kd_set_sampling")


def kd_set_trace(h, d_buf: int | None, n_words: int, every: int) -> int:
    return _check(h, load_library().kd_set_trace(h, d_buf, n_words, every), "kd_set_trace")


def kd_position(h) -> int:
    return load_library().kd_position(h)


def kd_get_info(h) -> kd_info:
    info = kd_info()
    _check(h, load_library().kd_get_info(h, ctypes.byref(info)), "kd_get_info")
    return info


def kd_kv_ptr(h, layer: int, which: int) -> int:
    return load_library().kd_kv_ptr(h, layer, which)


def kd_last_error(h) -> str:
    return (load_library().kd_last_error(h) or b"").decode()


def kd_strerror(code: int) -> str:
    return load_library().kd_strerror(code).decode()


def kd_destroy(h) -> None:
    load_library().kd_destroy(h)


# ---------------------------------------------------------------- convenience

def config_from(dims: dict, max_seq: int) -> kd_config:
    return kd_config(dims["n_layers"], dims["d_model"], dims["n_heads"], dims["n_kv_heads"],
                     dims["head_dim"], dims["ffn_dim"], dims["vocab"], int(max_seq),
                     float(dims["rms_eps"]), float(dims["rope_theta"]))


class Decoder:
    """One request's decoder on the current CUDA device and stream.

    PyTorch allocates the arena and the output buffers; libkd does the rest."""

    def __init__(self, dims: dict, max_seq: int, device=None, stream=None):
        import torch
        self.torch = torch
        self.device = torch.device(device or "cuda")
        self.cfg = config_from(dims, max_seq)
        self.dims = dict(dims)
        nbytes = kd_arena_bytes(self.cfg)
        if nbytes == 0:
            raise KdError(-1, "unsupported configuration %r" % (dims,))
        self.stream = stream or torch.cuda.current_stream(self.device)
        self.arena = torch.empty(nbytes + 256, dtype=torch.uint8, device=self.device)
        base = self.arena.data_ptr()
        self._arena_ptr = (base + 255) & ~255
        with torch.cuda.device(self.device):
            self.h = kd_create(self.cfg, self._arena_ptr, nbytes, self.stream.cuda_stream)
        self._keep = []
        self.pending = 0

    def close(self):
        h = getattr(self, "h", None)
        if h:
            self.h = None
            if kd_destroy is not None:  # None while the interpreter is shutting down
                kd_destroy(h)

    __del__ = close

    def info(self) -> kd_info:
        return kd_get_info(self.h)

    def load_weights(self, weights: dict):
        torch = self.torch
        w = kd_weights()
        keep = []
        for name in WEIGHT_FIELDS:
            t = weights[name]
            assert t.dtype == torch.bfloat16
            t = t.to(self.device).contiguous()
            keep.append(t)
            setattr(w, name, t.data_ptr())
        kd_load_weights(self.h, w)
        self.stream.synchronize()  # the repack reads the tensors; they may go away after this

    def set_kv(self, K, V):
        """Fill positions [0, P) of every layer from bf16 [L][Hkv][P][hd] tensors."""
        for l in range(K.shape[0]):
            for which, t in ((0, K[l]), (1, V[l])):
                t = t.to(self.device).contiguous()
                kd_set_kv(self.h, l, which, t.data_ptr(), t.shape[1])
                self._keep.append(t)
        self.stream.synchronize()
        self._keep.clear()

    def reset(self, tokens, kv_len: int = 0):
        torch = self.torch
        t = torch.as_tensor(tokens, dtype=torch.int32).to(self.device).contiguous()
        self._tokens = t  # kept alive until the copy has run
        kd_reset(self.h, t.data_ptr(), t.numel(), kv_len)
        self.pending = t.numel()

    def decode(self, n_gen: int, logits: bool = False, out=None):
        """Enqueue one decode launch; returns (tokens [n_gen] int32, logits [steps][V] or None)."""
        torch = self.torch
        steps = self.pending + n_gen - 1
        toks = out if out is not None else torch.empty(max(n_gen, 1), dtype=torch.int32, device=self.device)
        lg = torch.empty((steps, self.dims["vocab"]), dtype=torch.float32, device=self.device) if logits else None
        kd_decode(self.h, n_gen, toks.data_ptr(), lg.data_ptr() if lg is not None else None)
        if steps > 0:
            self.pending = 1  # the last generated (or last fed) token
        return toks[:n_gen], lg

    def sync(self):
        kd_sync(self.h)

    def set_sampling(self, temperature: float, seed: int = 0):
        """Greedy at temperature 0 (the default); else in-kernel draws from softmax(logits / T)."""
        kd_set_sampling(self.h, temperature, seed)

    def position(self) -> int:
        return kd_position(self.h)

    def generate(self, h_tokens, kv_len: int, n_gen: int, h_out=None):
        """Host buffers in and out (pinned tensors recommended): the end-to-end user call."""
        torch = self.torch
        h_tokens = torch.as_tensor(h_tokens, dtype=torch.int32).contiguous()
        if h_out is None:
            h_out = torch.empty(n_gen, dtype=torch.int32)
        kd_generate(self.h, h_tokens.data_ptr(), h_tokens.numel(), kv_len, n_gen, h_out.data_ptr())
        self.pending = 1
        return h_out
