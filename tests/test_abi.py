"""C-ABI library: loads without a GPU, exports every entry point of include/mk.h, checks
configs, and its task-graph validator accepts the built graphs and rejects corrupted ones."""
import os
import re

import numpy as np
import pytest

import mk_inputs as mi
import persistent_megakernel_decode_04_b200 as mk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "mk.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mk_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_entry_point():
    names = header_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(mk._lib, n), f"libmk.so lacks {n}"
    assert set(names) == set(mk.exported_symbols())


def _cfg(**kw):
    c = mk.Config.from_shape(mi.TINY, 1, 64)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value", [("head_dim", 96), ("hidden", 250), ("n_kv_heads", 3), ("max_batch", 0),
                                         ("max_batch", 17), ("max_seq", 0), ("rms_eps", 0.0), ("vocab", 1),
                                         ("qk_norm", 2), ("tc_min_batch", 1), ("tc_min_batch", 6)])
def test_bad_configs_are_rejected(field, value):
    with pytest.raises(mk.MkError) as e:
        mk.mk_build_taskgraph(_cfg(**{field: value}).c(), -1)
    assert e.value.code == mk.MK_ERR_INVALID_ARG


@pytest.mark.parametrize("max_batch", [1, 4, 16])
def test_qk_norm_config_sizes(max_batch):
    # QK-norm adds the per-layer gains and biases to the arena (q and k heads, gain + bias, bf16)
    # and a raw-key buffer [layer][batch][n_kv_heads*head_dim] fp32 to the workspace
    s = mi.TINY_QK
    sizes = []
    for qk in (False, True):
        c = mk.Config.from_shape(s, max_batch, 64)
        c.qk_norm = qk
        ctx = mk.mk_build_taskgraph(c.c(), -1)
        try:
            sizes.append((mk.mk_weight_arena_bytes(ctx), mk.mk_workspace_bytes(ctx), mk.mk_kv_cache_bytes(ctx)))
        finally:
            mk.mk_destroy(ctx)
    (a0, w0, k0), (a1, w1, k1) = sizes
    per_layer = 2 * (s.n_q_heads + s.n_kv_heads) * s.head_dim * 2
    assert a1 - a0 >= s.n_layers * per_layer and a1 - a0 < s.n_layers * (per_layer + 256)
    assert w1 - w0 >= s.n_layers * max_batch * s.n_kv_heads * s.head_dim * 4 - 256
    assert k1 == k0
    assert mk.Config.from_shape(s, 1, 8).qk_norm and not mk.Config.from_shape(mi.TINY, 1, 8).qk_norm


def test_null_context_calls_fail_cleanly():
    assert mk._lib.mk_decode_step(None, None, None, None, None, None) == mk.MK_ERR_INVALID_ARG
    assert mk._lib.mk_prefill(None, None, 1, 1, None, None, None) == mk.MK_ERR_INVALID_ARG
    assert mk.mk_last_error(None)


def test_decode_before_load_is_a_state_error():
    ctx = mk.mk_build_taskgraph(_cfg().c(), -1)
    try:
        rc = mk._lib.mk_decode_step(ctx, 1, 1, 1, None, None)
        assert rc == mk.MK_ERR_STATE
    finally:
        mk.mk_destroy(ctx)


@pytest.fixture(params=["tiny", "llama3-8b", "chameleon-7b-b1", "tiny-b4", "llama3-8b-b4", "chameleon-7b-b4",
                        "tiny-b16", "llama3-8b-b16", "chameleon-7b-b16"])
def graph(request):
    name, B = request.param, 1
    for suffix, b in (("-b4", 4), ("-b16", 16)):
        if name.endswith(suffix):
            name, B = name[: -len(suffix)], b
    shape, ms = {"tiny": (mi.TINY, 64), "llama3-8b": (mi.LLAMA8B, 1024),
                 "chameleon-7b-b1": (mi.CHAMELEON7B, 1280), "chameleon-7b": (mi.CHAMELEON7B, 1280)}[name]
    ctx = mk.mk_build_taskgraph(mk.Config.from_shape(shape, B, ms).c(), -1)
    tasks, counts = mk.mk_export_taskgraph(ctx)
    yield ctx, tasks, counts, shape, B
    mk.mk_destroy(ctx)


def test_built_graph_validates_and_balances_bytes(graph):
    ctx, tasks, counts, shape, B = graph
    assert mk.mk_validate_taskgraph(ctx, tasks, counts) == 0
    info = mk.mk_get_graph_info(ctx)
    # weight bytes streamed per step = every projection once (plain definition of the step)
    s = shape
    per_layer = ((s.n_q_heads + 2 * s.n_kv_heads) * s.head_dim * s.hidden + s.hidden * s.n_q_heads * s.head_dim
                 + 2 * s.ffn * s.hidden + s.hidden * s.ffn) * 2
    assert info["weight_bytes_per_step"] == s.n_layers * per_layer + s.vocab * s.hidden * 2
    # each SM streams nearly the same number of weight bytes (within 3 %); with 2..4 sequences
    # the down projection runs in K chunks, one task per chunk of the same rows; tensor-core
    # tasks (more than 4 sequences) stream nrows whole 32 KB weight blocks
    down = tasks[tasks[:, 0] == 6]
    ndc = len(down) // len({(int(t[1]), int(t[3])) for t in down})
    K = {2: s.hidden, 4: s.hidden, 5: s.hidden, 6: s.ffn / ndc, 7: s.hidden}
    per_sm = np.zeros(info["n_sms"])
    for t in tasks:
        if t[0] in K:
            per_sm[t[2]] += t[4] * (32768 if B > 4 else K[t[0]] * 2)
    if s.hidden >= 4096:
        assert per_sm.max() / per_sm.mean() < 1.03


def _reject(ctx, tasks, counts, needle):
    rc = mk.mk_validate_taskgraph(ctx, tasks, counts)
    assert rc == mk.MK_ERR_INVALID_ARG
    assert needle in mk.mk_last_error(ctx), mk.mk_last_error(ctx)


def test_validator_rejects_a_dropped_notify(graph):
    ctx, tasks, counts, _, B = graph
    t = tasks.copy()
    i = int(np.nonzero(t[:, 0] == 4)[0][0])  # an O-projection task
    t[i, 8] = 0
    _reject(ctx, t, counts, "producers per step")


def test_validator_rejects_a_missing_dependency(graph):
    ctx, tasks, counts, _, B = graph
    t = tasks.copy()
    i = int(np.nonzero(t[:, 0] == 3)[0][-1])  # an attention task loses its wait on QKV
    t[i, 5] = 0
    _reject(ctx, t, counts, "before its producers finish")


def test_validator_rejects_a_queue_that_deadlocks(graph):
    ctx, tasks, counts, _, B = graph
    t = tasks.copy()
    # find a task that waits on an event an earlier task of the same SM raises, and move it
    # in front of that producer: the SM then waits on itself
    pick = None
    for sm in range(int(t[:, 2].max()) + 1):
        q = [int(i) for i in np.nonzero(t[:, 2] == sm)[0]]
        for a_pos, a in enumerate(q):
            raised = set(int(e) for e in t[a, 9 : 9 + t[a, 8]])
            for b in q[a_pos + 1 :]:
                if raised & set(int(e) for e in t[b, 6 : 6 + t[b, 5]]):
                    pick = (a, b)
                    break
            if pick:
                break
        if pick:
            break
    assert pick is not None
    a, b = pick
    order = list(range(len(t)))
    order.remove(b)
    order.insert(order.index(a), b)
    _reject(ctx, t[order], counts, "deadlock")


def test_validator_rejects_overlapping_rows(graph):
    ctx, tasks, counts, _, B = graph
    t = tasks.copy()
    i = int(np.nonzero(t[:, 0] == 7)[0][3])
    t[i, 3] -= 2  # LM-head tile shifted onto its neighbour's rows (or blocks)
    rc = mk.mk_validate_taskgraph(ctx, t, counts)
    assert rc == mk.MK_ERR_INVALID_ARG
    msg = mk.mk_last_error(ctx)
    # row graphs: rows covered twice; block graphs: a task across two tiles, or an LM tile
    # count that no longer matches the token-pick threshold
    assert "covered" in msg or "spans two tiles" in msg or "threshold" in msg, msg


def test_validator_rejects_a_wrong_threshold(graph):
    ctx, tasks, counts, _, B = graph
    c = counts.copy()
    c[1] += 1
    _reject(ctx, tasks, c, "threshold")


def test_weighted_partition_follows_the_sm_weights():
    ctx = mk.mk_build_taskgraph(mk.Config.from_shape(mi.LLAMA8B, 1, 1024).c(), -1)
    try:
        info = mk.mk_get_graph_info(ctx)
        n = info["n_sms"]
        w = np.random.default_rng(0).uniform(0.6, 1.4, n).astype(np.float32)
        mk.mk_set_sm_weights(ctx, w)
        tasks, counts = mk.mk_export_taskgraph(ctx)
        assert mk.mk_validate_taskgraph(ctx, tasks, counts) == 0
        assert len(tasks) <= mk.mk_get_graph_info(ctx)["task_capacity"]
        K = {2: 4096, 4: 4096, 5: 4096, 6: 14336, 7: 4096}
        per_sm = np.zeros(n)
        for t in tasks:
            if t[0] in K:
                per_sm[t[2]] += t[4] * K[t[0]] * 2
        share = per_sm / per_sm.sum()
        assert np.allclose(share, w / w.sum(), rtol=0.02)
        with pytest.raises(mk.MkError):
            mk.mk_set_sm_weights(ctx, np.zeros(n, dtype=np.float32))
        with pytest.raises(mk.MkError):
            mk.mk_set_sm_weights(ctx, np.ones(n - 1, dtype=np.float32))
    finally:
        mk.mk_destroy(ctx)


def test_per_op_weights_repartition_only_that_op():
    ctx = mk.mk_build_taskgraph(mk.Config.from_shape(mi.LLAMA8B, 1, 1024).c(), -1)
    try:
        n = mk.mk_get_graph_info(ctx)["n_sms"]
        before, _ = mk.mk_export_taskgraph(ctx)
        w = np.random.default_rng(1).uniform(0.6, 1.4, n).astype(np.float32)
        mk.mk_set_op_sm_weights(ctx, 5, w)  # gate/up only
        tasks, counts = mk.mk_export_taskgraph(ctx)
        assert mk.mk_validate_taskgraph(ctx, tasks, counts) == 0
        per_sm = np.zeros(n)
        for t in tasks:
            if t[0] == 5:
                per_sm[t[2]] += t[4]
        assert np.allclose(per_sm / per_sm.sum(), w / w.sum(), rtol=0.03)
        for k in (2, 4, 6, 7):  # the other projections keep their partition
            assert np.array_equal(before[before[:, 0] == k][:, 2:5], tasks[tasks[:, 0] == k][:, 2:5])
        with pytest.raises(mk.MkError):
            mk.mk_set_op_sm_weights(ctx, 3, w)  # attention is not a projection
        mk.mk_set_sm_weights(ctx, np.ones(n, dtype=np.float32))  # resets every projection
        again, _ = mk.mk_export_taskgraph(ctx)
        assert np.array_equal(again, before)
    finally:
        mk.mk_destroy(ctx)


# ---------------------------------------------------------------- run-time claims (scheduling variant)

def _rows(shape, kind):
    D = shape.head_dim
    return {2: (shape.n_q_heads + 2 * shape.n_kv_heads) * D, 4: shape.hidden, 5: 2 * shape.ffn, 6: shape.hidden}[kind]


@pytest.mark.parametrize("shape,tps", [(mi.TINY, 1), (mi.TINY, 2), (mi.LLAMA8B.with_layers(3), 2),
                                       (mi.LLAMA8B.with_layers(2), 4)])
def test_claim_dispatch_pools_cover_every_projection(shape, tps):
    ctx = mk.mk_build_taskgraph(mk.Config.from_shape(shape, 1, 256).c(), -1)
    try:
        n0 = mk.mk_get_graph_info(ctx)["n_tasks"]
        mk.mk_set_dispatch(ctx, mk.MK_DISPATCH_CLAIM, tps)
        tasks, counts = mk.mk_export_taskgraph(ctx)
        n_sms = mk.mk_get_graph_info(ctx)["n_sms"]
        L = shape.n_layers
        entries = tasks[tasks[:, 0] == 8]
        pooled = tasks[tasks[:, 2] == -1]
        # one claim entry per SM for each projection of each layer, on every SM
        assert len(entries) == n_sms * 4 * L
        assert sorted(set(entries[:, 2].tolist())) == list(range(n_sms))
        assert set(pooled[:, 0].tolist()) == {2, 4, 5, 6}
        for kind in (2, 4, 5, 6):
            for l in range(L):
                sel = pooled[(pooled[:, 0] == kind) & (pooled[:, 1] == l)]
                cover = np.zeros(_rows(shape, kind), dtype=np.int32)
                for t in sel:
                    cover[t[3]:t[3] + t[4]] += 1
                assert (cover == 1).all(), f"kind {kind} layer {l}: rows not covered exactly once"
                assert len(sel) <= n_sms * tps
                # each task notifies the op's event; the event's count is the pool's task count
                if kind != 2:
                    assert counts[sel[0, 9]] == len(sel)
        # static tasks stay on their SMs: embedding, attention and the LM head
        static = tasks[(tasks[:, 2] >= 0) & (tasks[:, 0] != 8)]
        assert set(static[:, 0].tolist()) == {1, 3, 7}
        mk.mk_set_dispatch(ctx, mk.MK_DISPATCH_STATIC)
        assert mk.mk_get_graph_info(ctx)["n_tasks"] == n0
        assert not (mk.mk_export_taskgraph(ctx)[0][:, 0] == 8).any()
    finally:
        mk.mk_destroy(ctx)


@pytest.mark.parametrize("shape", [mi.TINY, mi.LLAMA8B.with_layers(2)])
def test_priority_dispatch_pools_the_attention_chunks(shape):
    # priority claims: every layer's attention chunks form a pool right after its QKV pool
    ctx = mk.mk_build_taskgraph(mk.Config.from_shape(shape, 1, 256).c(), -1)
    try:
        info = mk.mk_get_graph_info(ctx)
        mk.mk_set_dispatch(ctx, mk.MK_DISPATCH_CLAIM_PRIORITY, 2)
        tasks, counts = mk.mk_export_taskgraph(ctx)
        n_sms, L = info["n_sms"], shape.n_layers
        entries = tasks[tasks[:, 0] == 8]
        assert len(entries) == n_sms * 5 * L  # QKV, attention, O, gate/up, down
        pooled = tasks[tasks[:, 2] == -1]
        assert set(pooled[:, 0].tolist()) == {2, 3, 4, 5, 6}
        for l in range(L):
            attn = pooled[(pooled[:, 0] == 3) & (pooled[:, 1] == l)]
            assert len(attn) == shape.n_kv_heads * info["attn_chunks"]
            # every (sequence, KV head) has each chunk once
            seen = {(int(t[3]), int(t[4])) for t in attn}
            assert len(seen) == len(attn)
        static = tasks[(tasks[:, 2] >= 0) & (tasks[:, 0] != 8)]
        assert set(static[:, 0].tolist()) == {1, 7}  # only the embedding and the LM head stay fixed
        # on every SM the layer's attention entry comes right after its QKV entry
        sm0 = tasks[tasks[:, 2] == 0]
        kinds = [int(t[0]) for t in sm0]
        assert kinds.count(8) == 5 * L
    finally:
        mk.mk_destroy(ctx)


def test_claim_dispatch_rejections():
    for shape, b in ((mi.TINY, 4), (mi.TINY, 16), (mi.CHAMELEON7B.with_layers(1), 1)):
        ctx = mk.mk_build_taskgraph(mk.Config.from_shape(shape, b, 64).c(), -1)
        try:
            with pytest.raises(mk.MkError) as e:
                mk.mk_set_dispatch(ctx, mk.MK_DISPATCH_CLAIM, 2)
            assert e.value.code == mk.MK_ERR_UNSUPPORTED
        finally:
            mk.mk_destroy(ctx)
    ctx = mk.mk_build_taskgraph(_cfg().c(), -1)
    try:
        for mode, tps in ((mk.MK_DISPATCH_CLAIM, 0), (mk.MK_DISPATCH_CLAIM, 5), (7, 1), (-1, 1)):
            with pytest.raises(mk.MkError) as e:
                mk.mk_set_dispatch(ctx, mode, tps)
            assert e.value.code == mk.MK_ERR_INVALID_ARG
        n0 = mk.mk_get_graph_info(ctx)["n_tasks"]
        mk.mk_set_dispatch(ctx, mk.MK_DISPATCH_CLAIM, 1)
        assert mk.mk_get_graph_info(ctx)["n_tasks"] > n0
    finally:
        mk.mk_destroy(ctx)


def test_claim_dispatch_survives_repartitioning():
    # per-SM weights re-partition the static tasks; with run-time claims the pools stay whole
    ctx = mk.mk_build_taskgraph(mk.Config.from_shape(mi.TINY, 1, 64).c(), -1)
    try:
        mk.mk_set_dispatch(ctx, mk.MK_DISPATCH_CLAIM, 2)
        n_sms = mk.mk_get_graph_info(ctx)["n_sms"]
        before = mk.mk_export_taskgraph(ctx)[0]
        w = np.linspace(0.5, 1.5, n_sms).astype(np.float32)
        mk.mk_set_sm_weights(ctx, w)
        after, counts = mk.mk_export_taskgraph(ctx)
        pooled_b, pooled_a = before[before[:, 2] == -1], after[after[:, 2] == -1]
        assert np.array_equal(pooled_b, pooled_a)
        assert (after[:, 0] == 8).sum() == (before[:, 0] == 8).sum()
        # the static part (embedding, LM head) follows the weights: more rows on faster SMs
        lm = after[after[:, 0] == 7]
        rows = np.zeros(n_sms)
        np.add.at(rows, lm[:, 2], lm[:, 4])
        assert rows[-1] > rows[0]
    finally:
        mk.mk_destroy(ctx)
