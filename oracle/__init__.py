"""CPU oracle for the decode megakernel -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's ``cpu_baseline`` leg and
reference arm may import this package.  The product path (the CUDA library and its
Python binding) never imports it, and it imports nothing from the product path.

``oracle.cpp`` is a plain C++ decoder written from the pages (see its header for the
passages followed and the readings taken where the pages are silent).  This module
compiles it with g++ and wraps it with ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "oracle.cpp")
    hdr = os.path.join(_HERE, "oracle.h")
    newest = max(os.path.getmtime(src), os.path.getmtime(hdr))
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < newest:
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
                               src, "-o", _SO])
    return _SO


class _Config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("hidden", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("ffn", ctypes.c_int),
                ("vocab", ctypes.c_int), ("rms_eps", ctypes.c_double), ("rope_theta", ctypes.c_double)]


_PP = ctypes.POINTER(ctypes.c_void_p)


class _Weights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("lm_head", ctypes.c_void_p), ("final_norm", ctypes.c_void_p),
                ("attn_norm", _PP), ("wq", _PP), ("wk", _PP), ("wv", _PP), ("wo", _PP),
                ("mlp_norm", _PP), ("wg", _PP), ("wu", _PP), ("wd", _PP),
                ("q_norm_w", _PP), ("q_norm_b", _PP), ("k_norm_w", _PP), ("k_norm_b", _PP)]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        vp, i32, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.or_create.argtypes = [ctypes.POINTER(_Config), ctypes.POINTER(_Weights), i32, i32, i32, i32]
        L.or_create.restype = vp
        L.or_destroy.argtypes = [vp]
        L.or_set_threads.argtypes = [i32]
        L.or_prefill.argtypes = [vp, vp, i32, vp]
        L.or_decode.argtypes = [vp, vp, vp]
        L.or_decode_f64.argtypes = [vp, vp, vp]
        L.or_set_cache.argtypes = [vp, vp, i32]
        L.or_get_cache.argtypes = [vp, vp, i32]
        L.or_set_positions.argtypes = [vp, vp]
        L.or_position.argtypes = [vp, i32]
        L.or_argmax.argtypes = [vp, i32]
        L.or_get_qk.argtypes = [vp, i32, vp, vp]
        L.or_layernorm.argtypes = [vp, vp, vp, i32, dbl, vp]
        L.or_layernorm.restype = None
        L.or_rmsnorm.argtypes = [vp, vp, i32, dbl, vp]
        L.or_rmsnorm.restype = None
        L.or_matvec_bf16.argtypes = [vp, vp, i32, i32, vp]
        L.or_matvec_bf16.restype = None
        L.or_rope.argtypes = [vp, i32, i32, dbl]
        L.or_rope.restype = None
        L.or_rope_cos_sin.argtypes = [i32, i32, dbl, vp, vp]
        L.or_rope_cos_sin.restype = None
        L.or_attention_head.argtypes = [vp, vp, vp, i32, i32, dbl, vp, vp]
        L.or_attention_head.restype = None
        L.or_silu.argtypes = [dbl]
        L.or_silu.restype = dbl
        L.or_attention_decode_f16.argtypes = [vp, vp, vp, i32, i32, i32, dbl, vp]
        _lib = L
    return _lib


def set_threads(n: int) -> None:
    lib().or_set_threads(int(n))


def _ptr(a: np.ndarray):
    return a.ctypes.data


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


class Decoder:
    """One oracle decoder instance (batch of sequences with their own positions and cache).

    ``weights`` is an ``mk_inputs.Weights``-like object holding bf16 bit arrays.
    """

    def __init__(self, weights, batch: int, max_seq: int, f64: bool = False, kv_round: bool = True):
        s = weights.shape
        self.shape, self.batch, self.max_seq = s, batch, max_seq
        self._keep = weights  # keep the arrays alive while C holds their pointers
        self._cfg = _Config(s.n_layers, s.hidden, s.n_q_heads, s.n_kv_heads, s.head_dim, s.ffn, s.vocab,
                            s.rms_eps, s.rope_theta)
        n = s.n_layers

        def arr(lst):
            a = (ctypes.c_void_p * n)(*[x.ctypes.data for x in lst])
            return ctypes.cast(a, _PP), a

        self._arrs = []
        fields = {}
        names = ["attn_norm", "wq", "wk", "wv", "wo", "mlp_norm", "wg", "wu", "wd"]
        if getattr(weights, "q_norm_w", None):  # QK-norm model
            names += ["q_norm_w", "q_norm_b", "k_norm_w", "k_norm_b"]
        for name in names:
            p, a = arr(getattr(weights, name))
            self._arrs.append(a)
            fields[name] = p
        self._w = _Weights(weights.embed.ctypes.data, weights.lm_head.ctypes.data, weights.final_norm.ctypes.data,
                           **fields)
        self._h = lib().or_create(ctypes.byref(self._cfg), ctypes.byref(self._w), batch, max_seq, int(f64),
                                  int(kv_round))
        if not self._h:
            raise ValueError("or_create rejected the configuration")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            lib().or_destroy(h)
            self._h = None

    def prefill(self, tokens: np.ndarray) -> np.ndarray:
        tokens = _c(tokens, np.int32).reshape(self.batch, -1)
        out = np.empty((self.batch, self.shape.vocab), dtype=np.float32)
        rc = lib().or_prefill(self._h, _ptr(tokens), tokens.shape[1], _ptr(out))
        if rc != 0:
            raise RuntimeError(f"or_prefill failed: {rc}")
        return out

    def decode(self, tokens) -> np.ndarray:
        tokens = _c(np.atleast_1d(tokens), np.int32)
        out = np.empty((self.batch, self.shape.vocab), dtype=np.float32)
        rc = lib().or_decode(self._h, _ptr(tokens), _ptr(out))
        if rc != 0:
            raise RuntimeError(f"or_decode failed: {rc}")
        return out

    def decode_f64(self, tokens) -> np.ndarray:
        tokens = _c(np.atleast_1d(tokens), np.int32)
        out = np.empty((self.batch, self.shape.vocab), dtype=np.float64)
        rc = lib().or_decode_f64(self._h, _ptr(tokens), _ptr(out))
        if rc != 0:
            raise RuntimeError(f"or_decode_f64 failed: {rc}")
        return out

    def set_cache(self, kv_bf16: np.ndarray, length: int) -> None:
        kv = _c(kv_bf16, np.uint16)
        if lib().or_set_cache(self._h, _ptr(kv), int(length)) != 0:
            raise ValueError("or_set_cache rejected its arguments")

    def get_cache(self, length: int) -> np.ndarray:
        s = self.shape
        out = np.empty((s.n_layers, 2, self.batch, s.n_kv_heads, length, s.head_dim), dtype=np.uint16)
        if lib().or_get_cache(self._h, _ptr(out), int(length)) != 0:
            raise ValueError("or_get_cache rejected its arguments")
        return out

    def set_positions(self, positions) -> None:
        pos = _c(np.asarray(positions), np.int32)
        if pos.size != self.batch or lib().or_set_positions(self._h, _ptr(pos)) != 0:
            raise ValueError("or_set_positions rejected its arguments")

    def position(self, b: int = 0) -> int:
        return lib().or_position(self._h, b)

    def get_qk(self, layer: int):
        """q [batch, n_q_heads*head_dim] and k [batch, n_kv_heads*head_dim] of layer `layer` for the
        last token of the last call (after QK-norm and RoPE, before the cache's bf16 rounding)."""
        s = self.shape
        q = np.empty((self.batch, s.n_q_heads * s.head_dim), dtype=np.float64)
        k = np.empty((self.batch, s.n_kv_heads * s.head_dim), dtype=np.float64)
        if lib().or_get_qk(self._h, int(layer), _ptr(q), _ptr(k)) != 0:
            raise ValueError("or_get_qk rejected its arguments")
        return q, k


def argmax(logits: np.ndarray) -> int:
    x = _c(logits, np.float32)
    return int(lib().or_argmax(_ptr(x), x.size))


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    x, g = _c(x, np.float64), _c(g, np.float64)
    y = np.empty_like(x)
    lib().or_rmsnorm(_ptr(x), _ptr(g), x.size, eps, _ptr(y))
    return y


def layernorm(x: np.ndarray, g: np.ndarray, b: np.ndarray, eps: float) -> np.ndarray:
    x, g, b = _c(x, np.float64), _c(g, np.float64), _c(b, np.float64)
    y = np.empty_like(x)
    lib().or_layernorm(_ptr(x), _ptr(g), _ptr(b), x.size, eps, _ptr(y))
    return y


def matvec_bf16(w_bf16: np.ndarray, x: np.ndarray) -> np.ndarray:
    w, x = _c(w_bf16, np.uint16), _c(x, np.float64)
    y = np.empty(w.shape[0], dtype=np.float64)
    lib().or_matvec_bf16(_ptr(w), _ptr(x), w.shape[0], w.shape[1], _ptr(y))
    return y


def rope(v: np.ndarray, pos: int, theta: float) -> np.ndarray:
    v = _c(v, np.float64).copy()
    lib().or_rope(_ptr(v), v.size, int(pos), theta)
    return v


def rope_cos_sin(head_dim: int, pos: int, theta: float):
    c = np.empty(head_dim // 2, dtype=np.float32)
    s = np.empty(head_dim // 2, dtype=np.float32)
    lib().or_rope_cos_sin(head_dim, pos, theta, _ptr(c), _ptr(s))
    return c, s


def attention_head(q, k, v, scale: float):
    q, k, v = _c(q, np.float64), _c(k, np.float64), _c(v, np.float64)
    L, d = k.shape
    o = np.empty(d, dtype=np.float64)
    p = np.empty(L, dtype=np.float64)
    lib().or_attention_head(_ptr(q), _ptr(k), _ptr(v), L, d, scale, _ptr(o), _ptr(p))
    return o, p


def silu(z: float) -> float:
    return float(lib().or_silu(float(z)))


def attention_decode_f16(q: np.ndarray, k_t: np.ndarray, v: np.ndarray, scale: float = 1.0) -> np.ndarray:
    """q [BH,d], k_t [BH,d,L], v [BH,L,d] as fp16 bit arrays (uint16) -> o [BH,d] float64."""
    q, k_t, v = _c(q, np.uint16), _c(k_t, np.uint16), _c(v, np.uint16)
    BH, d, L = k_t.shape
    o = np.empty((BH, d), dtype=np.float64)
    rc = lib().or_attention_decode_f16(_ptr(q), _ptr(k_t), _ptr(v), BH, d, L, scale, _ptr(o))
    if rc != 0:
        raise ValueError("or_attention_decode_f16 rejected its arguments")
    return o
