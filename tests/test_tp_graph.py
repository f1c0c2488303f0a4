"""Tensor-parallel lowering on the CPU (no device): every rank's task graph, its remote-signal
edges and the cross-rank validator.  The decoder is split as the MPK summary's compiler splits
a matmul followed by an all-reduce ("Compiler des LLM en MegaKernel ...", Part 1): QKV, gate/up
and the LM head by output rows, O and down by input columns, whose tasks store partial rows
into every rank's receive buffer and raise the op's event on every rank."""
import numpy as np
import pytest

import mk_inputs as mi
import persistent_megakernel_decode_04_b200 as mk

F = {name: i for i, name in enumerate(mk.TP_FIELDS)}
KIND = {"embed": 1, "qkv": 2, "attn": 3, "oproj": 4, "gateup": 5, "down": 6, "lmhead": 7}


def build(shape, ranks, max_seq=64):
    ctx = mk.mk_build_taskgraph_tp(mk.Config.from_shape(shape, 1, max_seq).c(), ranks, -1)
    tasks, counts = mk.mk_export_taskgraph_tp(ctx)
    return ctx, tasks, counts


def rejected(ctx, tasks, counts, text):
    rc = mk.mk_validate_taskgraph_tp(ctx, tasks, counts)
    assert rc == mk.MK_ERR_INVALID_ARG, "the corrupted graph was accepted"
    msg = mk.mk_last_error(ctx)
    assert text in msg, msg
    return msg


@pytest.mark.parametrize("shape,ranks", [(mi.TINY, 2), (mi.LLAMA8B, 2), (mi.LLAMA8B, 4)])
def test_tp_graph_is_valid_and_sharded(shape, ranks):
    ctx, t, c = build(shape, ranks)
    try:
        assert mk.mk_validate_taskgraph_tp(ctx, t, c) == mk.MK_OK
        info = mk.mk_get_graph_info(ctx)
        per = info["n_sms"] // ranks
        assert (t[:, F["sm"]] // per == t[:, F["rank"]]).all()  # every task on an SM of its rank
        nkv_l = shape.n_kv_heads // ranks
        for r in range(ranks):
            mine = t[t[:, F["rank"]] == r]
            attn = mine[mine[:, F["kind"]] == KIND["attn"]]
            # each rank attends over its own KV heads only: row0 = sequence * n_kv_local + head
            assert attn[:, F["row0"]].max() == nkv_l - 1
            assert len(attn) == shape.n_layers * nkv_l * info["attn_chunks"]
            qkv = mine[(mine[:, F["kind"]] == KIND["qkv"]) & (mine[:, F["layer"]] == 0)]
            assert (qkv[:, F["row0"]] + qkv[:, F["nrows"]]).max() == (shape.n_q_heads + 2 * shape.n_kv_heads) // ranks * shape.head_dim
            lm = mine[mine[:, F["kind"]] == KIND["lmhead"]]
            assert (lm[:, F["row0"]] + lm[:, F["nrows"]]).max() == shape.vocab // ranks
        # the row-parallel projections, and only they, carry remote-signal edges
        rp = np.isin(t[:, F["kind"]], [KIND["oproj"], KIND["down"]])
        assert (t[rp, F["remote"]] == 1).all() and (t[~rp, F["remote"]] == 0).all()
        # gate/up tasks of a (rank, layer) write the residual rows [0, hidden) once between them
        gu = t[(t[:, F["kind"]] == KIND["gateup"]) & (t[:, F["rank"]] == 0) & (t[:, F["layer"]] == 0)]
        cover = np.zeros(shape.hidden, dtype=int)
        for lo, hi in gu[:, [F["row_lo"], F["row_hi"]]]:
            cover[lo:hi] += 1
        assert (cover == 1).all()
    finally:
        mk.mk_destroy(ctx)


def test_tp_dropped_remote_signal_is_rejected():
    ctx, t, c = build(mi.TINY, 2)
    try:
        t2 = t.copy()
        i = np.flatnonzero((t2[:, F["kind"]] == KIND["oproj"]) & (t2[:, F["rank"]] == 0))[0]
        t2[i, F["remote"]] = 0  # rank 0's partial rows would never be announced to rank 1
        rejected(ctx, t2, c, "rank 1 event")
    finally:
        mk.mk_destroy(ctx)


def test_tp_missing_wait_is_rejected():
    ctx, t, c = build(mi.TINY, 2)
    try:
        t2 = t.copy()
        i = np.flatnonzero((t2[:, F["kind"]] == KIND["gateup"]) & (t2[:, F["rank"]] == 1) & (t2[:, F["layer"]] == 1))[0]
        t2[i, F["n_wait"]] = 0  # would read the ranks' O rows without waiting for them
        rejected(ctx, t2, c, "may read data before its producers finish")
    finally:
        mk.mk_destroy(ctx)


def test_tp_wrong_threshold_is_rejected():
    ctx, t, c = build(mi.TINY, 2)
    try:
        c2 = c.copy()
        ev = t[(t[:, F["kind"]] == KIND["down"])][0, F["notify0"]]
        c2[ev] -= 1  # one producer short: the next layer could start before every rank's rows landed
        rejected(ctx, t, c2, "threshold")
    finally:
        mk.mk_destroy(ctx)


def test_tp_uncovered_residual_rows_are_rejected():
    ctx, t, c = build(mi.TINY, 2)
    try:
        t2 = t.copy()
        i = np.flatnonzero((t2[:, F["kind"]] == KIND["gateup"]) & (t2[:, F["rank"]] == 1)
                           & (t2[:, F["row_hi"]] > t2[:, F["row_lo"]]))[0]
        t2[i, F["row_hi"]] = t2[i, F["row_lo"]]  # its slice of x_mid would never be written
        rejected(ctx, t2, c, "of x_mid written 0 times")
    finally:
        mk.mk_destroy(ctx)


def test_tp_deadlocking_queue_is_rejected():
    ctx, t, c = build(mi.TINY, 2)
    try:
        # on an SM of rank 1 that runs both an attention chunk and an O task of layer 0, put
        # the O task first: it waits for the attention its own SM has not run yet
        r1 = t[:, F["rank"]] == 1
        for sm in np.unique(t[r1, F["sm"]]):
            idx = np.flatnonzero(t[:, F["sm"]] == sm)
            kinds = t[idx, F["kind"]]
            a = [i for i in idx if t[i, F["kind"]] == KIND["attn"] and t[i, F["layer"]] == 0]
            o = [i for i in idx if t[i, F["kind"]] == KIND["oproj"] and t[i, F["layer"]] == 0]
            if a and o and a[0] < o[0] and len(kinds):
                t2 = t.copy()
                t2[[a[0], o[0]]] = t2[[o[0], a[0]]]
                rejected(ctx, t2, c, "deadlock")
                return
        pytest.fail("no SM with an attention chunk before an O task")
    finally:
        mk.mk_destroy(ctx)


@pytest.mark.parametrize("change,code", [
    (dict(max_batch=2), mk.MK_ERR_UNSUPPORTED),
    (dict(ranks=5), mk.MK_ERR_INVALID_ARG),
    (dict(ranks=1), mk.MK_ERR_INVALID_ARG),
    (dict(vocab=1023), mk.MK_ERR_INVALID_ARG),
])
def test_tp_rejects_configs_it_cannot_split(change, code):
    shape = mi.TINY
    cfg = mk.Config.from_shape(shape, change.get("max_batch", 1), 64)
    if "vocab" in change:
        cfg.vocab = change["vocab"]
    with pytest.raises(mk.MkError) as e:
        mk.mk_build_taskgraph_tp(cfg.c(), change.get("ranks", 2), -1)
    assert e.value.code == code


def test_tp_qknorm_is_unsupported():
    cfg = mk.Config.from_shape(mi.TINY_QK, 1, 64)
    with pytest.raises(mk.MkError) as e:
        mk.mk_build_taskgraph_tp(cfg.c(), 2, -1)
    assert e.value.code == mk.MK_ERR_UNSUPPORTED
