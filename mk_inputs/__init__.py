"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

This package holds random-number generation only (SplitMix64 streams, Box-Muller
normals, bf16/fp16 rounding, token ids); none of the decoder's arithmetic lives
here.  `mk_inputs.c` states the generator's exact definition.  Weights for a
decoder of a given shape are produced by `make_weights`, with one tensor id per
tensor, so the oracle and the GPU library are fed the very same bytes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libmk_inputs.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile libmk_inputs.so in place with gcc."""
    src = os.path.join(_HERE, "mk_inputs.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-pthread", src, "-o", _SO, "-lm"])
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        u64, i32, dbl, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        L.mki_splitmix64_next.argtypes = [ctypes.POINTER(u64)]
        L.mki_splitmix64_next.restype = u64
        L.mki_stream_base.argtypes = [u64, u64]
        L.mki_stream_base.restype = u64
        L.mki_stream_u64.argtypes = [u64, u64]
        L.mki_stream_u64.restype = u64
        for name in ("mki_normal_bf16", "mki_normal_f16", "mki_normal_f32"):
            f = getattr(L, name)
            f.argtypes = [u64, u64, u64, dbl, dbl, vp, i32]
            f.restype = None
        L.mki_tokens.argtypes = [u64, u64, u64, ctypes.c_uint32, vp]
        L.mki_tokens.restype = None
        L.mki_const_bf16.argtypes = [u64, ctypes.c_float, vp]
        L.mki_const_bf16.restype = None
        _lib = L
    return _lib


def _threads() -> int:
    return int(os.environ.get("MK_INPUT_THREADS", os.cpu_count() or 1))


def normal_bf16(seed: int, tensor_id: int, shape, sigma: float = 1.0, mean: float = 0.0) -> np.ndarray:
    """bf16 bit patterns (uint16) of round(mean + sigma*N(0,1))."""
    out = np.empty(shape, dtype=np.uint16)
    lib().mki_normal_bf16(seed, tensor_id, out.size, mean, sigma, out.ctypes.data, _threads())
    return out


def normal_f16(seed: int, tensor_id: int, shape, sigma: float = 1.0, mean: float = 0.0) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint16)
    lib().mki_normal_f16(seed, tensor_id, out.size, mean, sigma, out.ctypes.data, _threads())
    return out


def normal_f32(seed: int, tensor_id: int, shape, sigma: float = 1.0, mean: float = 0.0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    lib().mki_normal_f32(seed, tensor_id, out.size, mean, sigma, out.ctypes.data, _threads())
    return out


def tokens(seed: int, tensor_id: int, n: int, vocab: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    lib().mki_tokens(seed, tensor_id, n, vocab, out.ctypes.data)
    return out


def const_bf16(shape, value: float) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint16)
    lib().mki_const_bf16(out.size, value, out.ctypes.data)
    return out


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32 (a shift; no rounding involved)."""
    return (a.astype(np.uint32) << 16).view(np.float32)


def f16_to_f32(a: np.ndarray) -> np.ndarray:
    return a.view(np.float16).astype(np.float32)


# ---------------------------------------------------------------------------
# Decoder shapes and weights
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class Shape:
    """Llama-style decoder shape (sizes only; no arithmetic)."""
    name: str
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rms_eps: float
    rope_theta: float
    qk_norm: bool = False  # LayerNorm on every query and key head before RoPE (Chameleon)

    def with_layers(self, n: int) -> "Shape":
        d = dict(self.__dict__)
        d["n_layers"] = n
        d["name"] = f"{self.name}-{n}L"
        return Shape(**d)


TINY = Shape("tiny", 2, 256, 4, 2, 64, 768, 1024, 1e-6, 1e4)
LLAMA8B = Shape("llama3-8b", 32, 4096, 32, 8, 128, 14336, 128256, 1e-5, 5e5)
CHAMELEON7B = Shape("chameleon-7b", 32, 4096, 32, 32, 128, 11008, 65536, 1e-5, 1e4)
CHAMELEON7B_QK = Shape("chameleon-7b-qknorm", 32, 4096, 32, 32, 128, 11008, 65536, 1e-5, 1e4, qk_norm=True)
TINY_QK = Shape("tiny-qknorm", 2, 256, 4, 2, 64, 768, 1024, 1e-5, 1e4, qk_norm=True)

# tensor ids: one stream per tensor so any subset can be regenerated independently
TID_EMBED, TID_LM_HEAD = 1, 2
TID_PROMPT_BASE = 1 << 20
TID_KV_BASE = 1 << 24


def _layer_tid(layer: int, which: int) -> int:
    return 1000 + 16 * layer + which


W_Q, W_K, W_V, W_O, W_G, W_U, W_D, W_QN_G, W_QN_B, W_KN_G, W_KN_B = range(11)


@dataclass
class Weights:
    """bf16 bit patterns, canonical [out, in] row-major, gains exactly 1."""
    shape: Shape
    embed: np.ndarray
    lm_head: np.ndarray
    final_norm: np.ndarray
    attn_norm: list = field(default_factory=list)
    wq: list = field(default_factory=list)
    wk: list = field(default_factory=list)
    wv: list = field(default_factory=list)
    wo: list = field(default_factory=list)
    mlp_norm: list = field(default_factory=list)
    wg: list = field(default_factory=list)
    wu: list = field(default_factory=list)
    wd: list = field(default_factory=list)
    # QK-norm models only: LayerNorm gain and bias per head, [heads * head_dim] each
    q_norm_w: list = field(default_factory=list)
    q_norm_b: list = field(default_factory=list)
    k_norm_w: list = field(default_factory=list)
    k_norm_b: list = field(default_factory=list)


def make_weights(s: Shape, seed: int = 0, sigma: float = 0.02, norm_sigma: float = 0.2) -> Weights:
    """Weights of shape `s`; for a QK-norm shape the norm gains are 1 + N(0, norm_sigma^2) and
    the biases N(0, norm_sigma^2), per head and element."""
    H, F, D = s.hidden, s.ffn, s.head_dim
    w = Weights(s, normal_bf16(seed, TID_EMBED, (s.vocab, H), sigma),
                normal_bf16(seed, TID_LM_HEAD, (s.vocab, H), sigma), const_bf16((H,), 1.0))
    for l in range(s.n_layers):
        w.attn_norm.append(const_bf16((H,), 1.0))
        w.mlp_norm.append(const_bf16((H,), 1.0))
        w.wq.append(normal_bf16(seed, _layer_tid(l, W_Q), (s.n_q_heads * D, H), sigma))
        w.wk.append(normal_bf16(seed, _layer_tid(l, W_K), (s.n_kv_heads * D, H), sigma))
        w.wv.append(normal_bf16(seed, _layer_tid(l, W_V), (s.n_kv_heads * D, H), sigma))
        w.wo.append(normal_bf16(seed, _layer_tid(l, W_O), (H, s.n_q_heads * D), sigma))
        w.wg.append(normal_bf16(seed, _layer_tid(l, W_G), (F, H), sigma))
        w.wu.append(normal_bf16(seed, _layer_tid(l, W_U), (F, H), sigma))
        w.wd.append(normal_bf16(seed, _layer_tid(l, W_D), (H, F), sigma))
        if s.qk_norm:
            nq, nkv = s.n_q_heads * D, s.n_kv_heads * D
            w.q_norm_w.append(normal_bf16(seed, _layer_tid(l, W_QN_G), (nq,), norm_sigma, mean=1.0))
            w.q_norm_b.append(normal_bf16(seed, _layer_tid(l, W_QN_B), (nq,), norm_sigma))
            w.k_norm_w.append(normal_bf16(seed, _layer_tid(l, W_KN_G), (nkv,), norm_sigma, mean=1.0))
            w.k_norm_b.append(normal_bf16(seed, _layer_tid(l, W_KN_B), (nkv,), norm_sigma))
    return w


def prompt(seed: int, index: int, n: int, vocab: int) -> np.ndarray:
    """Prompt token ids: sequence `index` of a batch gets its own stream."""
    return tokens(seed, TID_PROMPT_BASE + index, n, vocab)


def kv_cache_values(seed: int, s: Shape, batch: int, length: int, sigma: float = 1.0):
    """A synthetic, already-filled bf16 KV cache in the canonical layout
    [layer][K|V][seq][kv_head][pos][head_dim] with `length` positions per sequence;
    used where a prompt is too long for the oracle to prefill on a CPU."""
    shp = (s.n_layers, 2, batch, s.n_kv_heads, length, s.head_dim)
    return normal_bf16(seed, TID_KV_BASE, shp, sigma)
