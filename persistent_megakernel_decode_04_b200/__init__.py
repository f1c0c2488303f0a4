"""Persistent decode megakernel for B200 (sm_100a): Python binding of the C ABI in include/mk.h.

The binding only marshals arguments: every step of decode (and of prefill and the
standalone attention) runs in the CUDA kernels of ``libmk.so``.  PyTorch supplies device
memory and streams.  If ``libmk.so`` is missing, importing this package raises
ImportError: there is no fallback path.

Functions carry the C names (``mk_build_taskgraph``, ``mk_load_weights``, ``mk_prefill``,
``mk_decode_step``, ``mk_destroy`` ...); they raise :class:`MkError` on a non-zero status.
Pointer arguments accept a torch tensor (its ``data_ptr()``), an int or None (NULL);
``stream`` accepts a ``torch.cuda.Stream``, an int handle or None (legacy default stream).
:class:`Megakernel` wraps one model instance with torch-allocated buffers.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmk.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m persistent_megakernel_decode_04_b200.build` "
                      "(nvcc, sm_100a); there is no CPU fallback")
_lib = ctypes.CDLL(LIB_PATH)

MK_OK = 0
MK_ERR_INVALID_ARG = -1
MK_ERR_CUDA = -2
MK_ERR_DEVICE_TIMEOUT = -3
MK_ERR_NOT_RESIDENT = -4
MK_ERR_STATE = -5
MK_ERR_UNSUPPORTED = -6
MK_MAX_BATCH = 16
MK_DISPATCH_STATIC = 0
MK_DISPATCH_CLAIM = 1
MK_DISPATCH_CLAIM_PACED = 2
MK_DISPATCH_CLAIM_PRIORITY = 3

TASK_KINDS = {1: "embed", 2: "qkv", 3: "attn", 4: "oproj", 5: "gateup", 6: "down", 7: "lmhead", 8: "pool"}


class MkError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{msg} (status {code})")
        self.code = code


class mk_config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("hidden", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("ffn", ctypes.c_int),
                ("vocab", ctypes.c_int), ("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("max_batch", ctypes.c_int), ("max_seq", ctypes.c_int), ("tie_embeddings", ctypes.c_int),
                ("qk_norm", ctypes.c_int), ("tc_min_batch", ctypes.c_int)]


_PP = ctypes.POINTER(ctypes.c_void_p)


class mk_host_weights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("lm_head", ctypes.c_void_p), ("final_norm", ctypes.c_void_p),
                ("attn_norm", _PP), ("wq", _PP), ("wk", _PP), ("wv", _PP), ("wo", _PP),
                ("mlp_norm", _PP), ("wg", _PP), ("wu", _PP), ("wd", _PP),
                ("q_norm_w", _PP), ("q_norm_b", _PP), ("k_norm_w", _PP), ("k_norm_b", _PP)]


class mk_graph_info(ctypes.Structure):
    _fields_ = [("n_sms", ctypes.c_int), ("n_tasks", ctypes.c_int), ("n_events", ctypes.c_int),
                ("task_capacity", ctypes.c_int), ("attn_chunks", ctypes.c_int), ("kernel_variant", ctypes.c_int),
                ("weight_bytes_per_step", ctypes.c_uint64), ("smem_bytes", ctypes.c_uint64)]


_vp, _i32, _sz, _u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64
_SIGS = {
    "mk_build_taskgraph": ([ctypes.POINTER(mk_config), _i32, ctypes.POINTER(_vp)], _i32),
    "mk_weight_arena_bytes": ([_vp], _sz),
    "mk_workspace_bytes": ([_vp], _sz),
    "mk_kv_cache_bytes": ([_vp], _sz),
    "mk_load_weights": ([_vp, ctypes.POINTER(mk_host_weights), _vp, _vp, _vp], _i32),
    "mk_prefill": ([_vp, _vp, _i32, _i32, _vp, _vp, _vp], _i32),
    "mk_set_positions": ([_vp, _vp, _i32], _i32),
    "mk_get_positions": ([_vp, _vp, _i32], _i32),
    "mk_decode_step": ([_vp, _vp, _vp, _vp, _vp, _vp], _i32),
    "mk_decode_steps": ([_vp, _vp, _i32, _vp, _vp, _vp, _vp], _i32),
    "mk_sync_status": ([_vp, _vp], _i32),
    "mk_set_wait_timeout_ns": ([_vp, _u64], _i32),
    "mk_debug_drop_notify": ([_vp, _i32, _i32], _i32),
    "mk_set_l2_prefetch": ([_vp, _i32], _i32),
    "mk_set_attn_chunk_keys": ([_vp, _i32], _i32),
    "mk_set_attn_head_keys": ([_vp, _i32], _i32),
    "mk_set_dispatch": ([_vp, _i32, _i32, _vp], _i32),
    "mk_set_sm_weights": ([_vp, _vp, _i32, _vp], _i32),
    "mk_set_op_sm_weights": ([_vp, _i32, _vp, _i32, _vp], _i32),
    "mk_set_trace": ([_vp, _vp], _i32),
    "mk_get_graph_info": ([_vp, ctypes.POINTER(mk_graph_info)], _i32),
    "mk_export_taskgraph": ([_vp, _vp, _i32, _vp, _i32], _i32),
    "mk_validate_taskgraph": ([_vp, _vp, _i32, _vp, _i32], _i32),
    "mk_build_taskgraph_tp": ([ctypes.POINTER(mk_config), _i32, _i32, ctypes.POINTER(_vp)], _i32),
    "mk_export_taskgraph_tp": ([_vp, _vp, _i32, _vp, _i32], _i32),
    "mk_validate_taskgraph_tp": ([_vp, _vp, _i32, _vp, _i32], _i32),
    "mk_attention_workspace_bytes": ([_i32, _i32, _i32], _sz),
    "mk_attention_decode": ([_vp, _vp, _vp, _vp, _i32, _i32, _i32, ctypes.c_float, _vp, _vp], _i32),
    "mk_attention_status": ([_vp, _i32, _i32, _i32, _vp], _i32),
    "mk_attention_decode_noalloc": ([_vp, _vp, _vp, _vp, _i32, _i32, _i32, ctypes.c_float, _vp], _i32),
    "mk_attention_noalloc_status": ([_vp], _i32),
    "mk_attention_set_wait_timeout_ns": ([_u64], _i32),
    "mk_attention_debug_drop_unit": ([_i32], _i32),
    "mk_last_error": ([_vp], ctypes.c_char_p),
    "mk_destroy": ([_vp], None),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res


def exported_symbols():
    """Names of the C entry points this binding found in libmk.so."""
    return sorted(_SIGS)


def _ptr(x) -> int | None:
    if x is None:
        return None
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        return x.ctypes.data
    return int(x)


def _stream(s) -> int | None:
    if s is None:
        return None
    if hasattr(s, "cuda_stream"):
        return s.cuda_stream
    return int(s)


def _check(rc: int, ctx=None):
    if rc != MK_OK:
        msg = _lib.mk_last_error(ctx)
        raise MkError(rc, msg.decode() if msg else "error")
    return rc


# ------------------------------------------------------------------------------ C entry points

def mk_build_taskgraph(cfg: mk_config, device: int) -> int:
    h = _vp()
    _check(_lib.mk_build_taskgraph(ctypes.byref(cfg), int(device), ctypes.byref(h)))
    return h.value


def mk_weight_arena_bytes(ctx) -> int:
    return _lib.mk_weight_arena_bytes(ctx)


def mk_workspace_bytes(ctx) -> int:
    return _lib.mk_workspace_bytes(ctx)


def mk_kv_cache_bytes(ctx) -> int:
    return _lib.mk_kv_cache_bytes(ctx)


def _host_weights(w, n_layers):
    keep = []

    def arr(lst):
        a = (ctypes.c_void_p * n_layers)(*[_ptr(x) for x in lst])
        keep.append(a)
        return ctypes.cast(a, _PP)

    qk = [arr(getattr(w, name)) if getattr(w, "q_norm_w", None) else None
          for name in ("q_norm_w", "q_norm_b", "k_norm_w", "k_norm_b")]
    hw = mk_host_weights(_ptr(w.embed), _ptr(w.lm_head), _ptr(w.final_norm),
                         arr(w.attn_norm), arr(w.wq), arr(w.wk), arr(w.wv), arr(w.wo),
                         arr(w.mlp_norm), arr(w.wg), arr(w.wu), arr(w.wd), *qk)
    return hw, keep


def mk_load_weights(ctx, weights, weight_arena, workspace, stream=None, n_layers: int | None = None):
    """``weights``: object with bf16 (uint16) host arrays embed, lm_head, final_norm and per-layer
    lists attn_norm, wq, wk, wv, wo, mlp_norm, wg, wu, wd (canonical [out, in] row-major); for a
    QK-norm model also q_norm_w, q_norm_b ([n_q_heads*head_dim]) and k_norm_w, k_norm_b
    ([n_kv_heads*head_dim])."""
    n = n_layers if n_layers is not None else len(weights.wq)
    hw, keep = _host_weights(weights, n)
    _check(_lib.mk_load_weights(ctx, ctypes.byref(hw), _ptr(weight_arena), _ptr(workspace), _stream(stream)), ctx)
    del keep


def mk_prefill(ctx, tokens, B: int, T: int, kv_cache, last_logits, stream=None):
    _check(_lib.mk_prefill(ctx, _ptr(tokens), int(B), int(T), _ptr(kv_cache), _ptr(last_logits), _stream(stream)),
           ctx)


def mk_set_positions(ctx, positions):
    a = (ctypes.c_int32 * len(positions))(*[int(p) for p in positions])
    _check(_lib.mk_set_positions(ctx, ctypes.cast(a, _vp), len(positions)), ctx)


def mk_get_positions(ctx, capacity: int = MK_MAX_BATCH):
    a = (ctypes.c_int32 * capacity)()
    n = _lib.mk_get_positions(ctx, ctypes.cast(a, _vp), capacity)
    if n < 0:
        raise MkError(n, "mk_get_positions")
    return list(a[:n])


def mk_decode_step(ctx, tokens, kv_cache, logits, next_tokens=None, stream=None):
    _check(_lib.mk_decode_step(ctx, _ptr(tokens), _ptr(kv_cache), _ptr(logits), _ptr(next_tokens),
                               _stream(stream)), ctx)


def mk_decode_steps(ctx, tokens, n_steps: int, kv_cache, logits, tokens_out, stream=None):
    _check(_lib.mk_decode_steps(ctx, _ptr(tokens), int(n_steps), _ptr(kv_cache), _ptr(logits), _ptr(tokens_out),
                                _stream(stream)), ctx)


def mk_sync_status(ctx, stream=None) -> int:
    """Returns the status code (MK_OK or MK_ERR_DEVICE_TIMEOUT) instead of raising on a timeout."""
    rc = _lib.mk_sync_status(ctx, _stream(stream))
    if rc not in (MK_OK, MK_ERR_DEVICE_TIMEOUT):
        _check(rc, ctx)
    return rc


def mk_set_wait_timeout_ns(ctx, ns: int):
    _check(_lib.mk_set_wait_timeout_ns(ctx, int(ns)), ctx)


def mk_debug_drop_notify(ctx, event_id: int, on: bool):
    _check(_lib.mk_debug_drop_notify(ctx, int(event_id), int(bool(on))), ctx)


def mk_set_sm_weights(ctx, weights, stream=None):
    import numpy as np
    w = np.ascontiguousarray(weights, dtype=np.float32)
    _check(_lib.mk_set_sm_weights(ctx, w.ctypes.data, w.size, _stream(stream)), ctx)


def mk_set_op_sm_weights(ctx, op_kind: int, weights, stream=None):
    import numpy as np
    w = np.ascontiguousarray(weights, dtype=np.float32)
    _check(_lib.mk_set_op_sm_weights(ctx, int(op_kind), w.ctypes.data, w.size, _stream(stream)), ctx)


def mk_set_l2_prefetch(ctx, stages: int):
    _check(_lib.mk_set_l2_prefetch(ctx, int(stages)), ctx)


def mk_set_attn_chunk_keys(ctx, keys: int):
    _check(_lib.mk_set_attn_chunk_keys(ctx, int(keys)), ctx)


def mk_set_attn_head_keys(ctx, keys: int):
    _check(_lib.mk_set_attn_head_keys(ctx, int(keys)), ctx)


def mk_set_dispatch(ctx, mode: int, tasks_per_sm: int = 2, stream=None):
    """MK_DISPATCH_STATIC (fixed per-SM queues), MK_DISPATCH_CLAIM (projection tasks claimed at
    run time from per-op pools of tasks_per_sm * n_sms tasks) or MK_DISPATCH_CLAIM_PACED (claims
    paced by the SM's workers)."""
    _check(_lib.mk_set_dispatch(ctx, int(mode), int(tasks_per_sm), _stream(stream)), ctx)


def mk_set_trace(ctx, device_buffer):
    _check(_lib.mk_set_trace(ctx, _ptr(device_buffer)), ctx)


def mk_get_graph_info(ctx) -> dict:
    info = mk_graph_info()
    _check(_lib.mk_get_graph_info(ctx, ctypes.byref(info)), ctx)
    return {name: getattr(info, name) for name, _ in mk_graph_info._fields_}


def mk_export_taskgraph(ctx):
    """Returns (tasks int32 [n, 11], event_counts int32 [n_events]) as numpy arrays."""
    import numpy as np
    n = _lib.mk_export_taskgraph(ctx, None, 0, None, 0)
    info = mk_get_graph_info(ctx)
    tasks = np.zeros((n, 11), dtype=np.int32)
    counts = np.zeros(info["n_events"], dtype=np.int32)
    _lib.mk_export_taskgraph(ctx, tasks.ctypes.data, n, counts.ctypes.data, counts.size)
    return tasks, counts


def mk_validate_taskgraph(ctx, tasks, counts) -> int:
    import numpy as np
    tasks = np.ascontiguousarray(tasks, dtype=np.int32)
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    return _lib.mk_validate_taskgraph(ctx, tasks.ctypes.data, tasks.shape[0], counts.ctypes.data, counts.size)


def mk_build_taskgraph_tp(cfg: mk_config, n_ranks: int, device: int) -> int:
    h = _vp()
    _check(_lib.mk_build_taskgraph_tp(ctypes.byref(cfg), int(n_ranks), int(device), ctypes.byref(h)))
    return h.value


TP_FIELDS = ("rank", "kind", "layer", "sm", "row0", "nrows", "n_wait", "wait0", "wait1", "n_notify", "notify0",
             "notify1", "remote", "row_lo", "row_hi")


def mk_export_taskgraph_tp(ctx):
    """Returns (tasks int32 [n, 15] with the columns TP_FIELDS, event_counts int32 [n_events])."""
    import numpy as np
    n = _lib.mk_export_taskgraph_tp(ctx, None, 0, None, 0)
    if n < 0:
        raise MkError(n, "mk_export_taskgraph_tp")
    info = mk_get_graph_info(ctx)
    tasks = np.zeros((n, 15), dtype=np.int32)
    counts = np.zeros(info["n_events"], dtype=np.int32)
    _lib.mk_export_taskgraph_tp(ctx, tasks.ctypes.data, n, counts.ctypes.data, counts.size)
    return tasks, counts


def mk_validate_taskgraph_tp(ctx, tasks, counts) -> int:
    import numpy as np
    tasks = np.ascontiguousarray(tasks, dtype=np.int32)
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    return _lib.mk_validate_taskgraph_tp(ctx, tasks.ctypes.data, tasks.shape[0], counts.ctypes.data, counts.size)


def mk_attention_workspace_bytes(BH: int, d: int, L: int) -> int:
    return _lib.mk_attention_workspace_bytes(int(BH), int(d), int(L))


def mk_attention_decode(q, k_t, v, o, BH: int, d: int, L: int, scale: float, workspace, stream=None):
    _check(_lib.mk_attention_decode(_ptr(q), _ptr(k_t), _ptr(v), _ptr(o), int(BH), int(d), int(L), float(scale),
                                    _ptr(workspace), _stream(stream)))


def mk_attention_decode_noalloc(q, k_t, v, o, BH: int, d: int, L: int, scale: float, stream=None):
    """Same as mk_attention_decode for callers that may not allocate: the scratch is a fixed
    4 MiB array inside libmk.so (sizes needing more are rejected)."""
    _check(_lib.mk_attention_decode_noalloc(_ptr(q), _ptr(k_t), _ptr(v), _ptr(o), int(BH), int(d), int(L),
                                            float(scale), _stream(stream)))


def mk_attention_status(workspace, BH: int, d: int, L: int, stream=None) -> int:
    return _lib.mk_attention_status(_ptr(workspace), int(BH), int(d), int(L), _stream(stream))


def mk_attention_noalloc_status(stream=None) -> int:
    """MK_OK, or MK_ERR_DEVICE_TIMEOUT if a no-alloc call since the last status call had a device
    wait run out (returned, not raised)."""
    return _lib.mk_attention_noalloc_status(_stream(stream))


def mk_attention_set_wait_timeout_ns(ns: int):
    _check(_lib.mk_attention_set_wait_timeout_ns(int(ns)))


def mk_attention_debug_drop_unit(unit: int):
    _check(_lib.mk_attention_debug_drop_unit(int(unit)))


def mk_last_error(ctx=None) -> str:
    m = _lib.mk_last_error(ctx)
    return m.decode() if m else ""


def mk_destroy(ctx):
    _lib.mk_destroy(ctx)


# ------------------------------------------------------------------------------ convenience

@dataclass
class Config:
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rms_eps: float
    rope_theta: float
    max_batch: int = 1
    max_seq: int = 1024
    qk_norm: bool = False
    tc_min_batch: int = 0  # 0: default (every batched width on the tensor cores); 5: CUDA-core GEMV up to 4

    @classmethod
    def from_shape(cls, shape, max_batch: int = 1, max_seq: int = 1024) -> "Config":
        return cls(shape.n_layers, shape.hidden, shape.n_q_heads, shape.n_kv_heads, shape.head_dim, shape.ffn,
                   shape.vocab, shape.rms_eps, shape.rope_theta, max_batch, max_seq,
                   bool(getattr(shape, "qk_norm", False)))

    def c(self) -> mk_config:
        return mk_config(self.n_layers, self.hidden, self.n_q_heads, self.n_kv_heads, self.head_dim, self.ffn,
                         self.vocab, self.rms_eps, self.rope_theta, self.max_batch, self.max_seq, 0,
                         int(self.qk_norm), int(self.tc_min_batch))


class Megakernel:
    """One model instance: task graph + torch-allocated weight arena, workspace and KV cache."""

    def __init__(self, cfg: Config, weights=None, device: int = 0, stream=None, tp_ranks: int = 1):
        """tp_ranks > 1: an emulated tensor-parallel model (mk_build_taskgraph_tp), every rank on
        this device; kv_view() then has a leading rank axis."""
        import torch
        self.cfg = cfg
        self.device = device
        self.tp_ranks = tp_ranks
        self.ctx = mk_build_taskgraph_tp(cfg.c(), tp_ranks, device) if tp_ranks > 1 else \
            mk_build_taskgraph(cfg.c(), device)
        dev = torch.device("cuda", device)
        self.arena = torch.empty(mk_weight_arena_bytes(self.ctx), dtype=torch.uint8, device=dev)
        self.workspace = torch.zeros(mk_workspace_bytes(self.ctx), dtype=torch.uint8, device=dev)
        self.kv = torch.zeros(mk_kv_cache_bytes(self.ctx) // 2, dtype=torch.int16, device=dev)
        self.logits = torch.empty((cfg.max_batch, cfg.vocab), dtype=torch.float32, device=dev)
        self.next_tokens = torch.zeros(cfg.max_batch, dtype=torch.int32, device=dev)
        self.stream = stream
        if weights is not None:
            self.load(weights)

    def load(self, weights):
        mk_load_weights(self.ctx, weights, self.arena, self.workspace, self.stream, self.cfg.n_layers)

    def kv_view(self):
        """The cache as int16 bf16 bits [layer][K|V][max_batch][n_kv][max_seq][head_dim]; with
        tensor parallelism [rank][layer][K|V][1][n_kv / ranks][max_seq][head_dim]."""
        c = self.cfg
        if self.tp_ranks > 1:
            R = self.tp_ranks
            per = c.n_layers * 2 * c.max_batch * (c.n_kv_heads // R) * c.max_seq * c.head_dim
            return self.kv.view(-1)[: R * per].view(R, c.n_layers, 2, c.max_batch, c.n_kv_heads // R, c.max_seq,
                                                   c.head_dim)
        return self.kv.view(c.n_layers, 2, c.max_batch, c.n_kv_heads, c.max_seq, c.head_dim)

    def prefill(self, tokens):
        """tokens: int32 CUDA tensor [B, T]; returns fp32 logits [B, vocab] of the last token."""
        B, T = tokens.shape
        out = self.logits[:B]
        mk_prefill(self.ctx, tokens, B, T, self.kv, out, self.stream)
        return out

    def decode(self, tokens):
        """tokens: int32 CUDA tensor [B]; returns (logits [B, vocab], next_tokens [B])."""
        B = tokens.shape[0]
        mk_decode_step(self.ctx, tokens, self.kv, self.logits, self.next_tokens, self.stream)
        return self.logits[:B], self.next_tokens[:B]

    def decode_steps(self, tokens, n_steps: int):
        """n_steps greedy decode steps in one launch, starting from tokens (int32 CUDA [B]);
        returns (logits of the last step [B, vocab], picked tokens [n_steps, B])."""
        import torch
        B = tokens.shape[0]
        out = torch.empty((n_steps, self.cfg.max_batch), dtype=torch.int32, device=tokens.device)
        mk_decode_steps(self.ctx, tokens, n_steps, self.kv, self.logits, out, self.stream)
        return self.logits[:B], out[:, :B]

    def calibrate(self, tokens, steps: int = 2, rounds: int = 3):
        """Measure each SM's busy time on each projection (QKV, O, gate/up, down, LM head) over
        `steps` traced decode steps (decoding `tokens`, which advances the positions) and
        re-partition that projection's rows so that every SM finishes it together; `rounds`
        measure/re-partition passes.  Returns the weights, one row per projection kind.  (With
        run-time claims the pools stay cut in equal shares: the weights apply once the static
        schedule is selected again.)"""
        import numpy as np
        import torch
        info = self.info()
        n = info["n_sms"]
        kinds = (2, 4, 5, 6, 7)
        w = {k: np.ones(n) for k in kinds}
        trace = torch.zeros(info["task_capacity"] * 6, dtype=torch.int64, device=tokens.device)
        for _ in range(rounds):
            tasks, _ = mk_export_taskgraph(self.ctx)
            mk_set_trace(self.ctx, trace)
            busy = {k: np.zeros(n) for k in kinds}
            for _ in range(steps):
                self.decode(tokens)
                self.sync_status()
                T = trace[: tasks.shape[0] * 6].view(-1, 6).cpu().numpy()
                sm = (T[:, 3].astype(np.uint64) >> np.uint64(32)).astype(np.int64)  # the SM that ran it
                for k in kinds:
                    sel = tasks[:, 0] == k
                    np.add.at(busy[k], sm[sel], (T[sel, 2] - T[sel, 1]).astype(np.float64))
            mk_set_trace(self.ctx, None)
            for k in kinds:
                b = busy[k]
                if b.min() <= 0:  # an SM without tasks of this kind: keep its weights
                    continue
                w[k] = w[k] * b.mean() / b  # slower SMs (more busy time) get fewer rows
                w[k] = w[k] / w[k].mean()
                mk_set_op_sm_weights(self.ctx, k, w[k], self.stream)
        return np.stack([w[k] for k in kinds])

    def set_positions(self, positions):
        mk_set_positions(self.ctx, positions)

    def positions(self):
        return mk_get_positions(self.ctx)

    def sync_status(self) -> int:
        return mk_sync_status(self.ctx, self.stream)

    def info(self) -> dict:
        return mk_get_graph_info(self.ctx)

    def set_dispatch(self, mode: int, tasks_per_sm: int = 2):
        """Scheduling variant: MK_DISPATCH_STATIC or MK_DISPATCH_CLAIM (see mk_set_dispatch)."""
        mk_set_dispatch(self.ctx, mode, tasks_per_sm, self.stream)

    def close(self):
        if getattr(self, "ctx", None):
            mk_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
