"""Tensor-parallel decode, emulated on one GPU (every rank's shard in one persistent launch,
their partial rows and signals exchanged through device memory), against the CPU oracle of the
whole, unsharded model.  Teacher-forced on the oracle's tokens: per-step logits and argmax, and
each rank's KV cache against the oracle's cache of that rank's KV heads.  The split is the MPK
summary's matmul + all-reduce lowering ("Compiler des LLM en MegaKernel ...", Part 1)."""
import numpy as np
import pytest
import torch

import mk_inputs as mi
import oracle
import persistent_megakernel_decode_04_b200 as mk
from _parity import argmax_agrees, kv_close, logits_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def tp_model(w, ranks, max_seq):
    return mk.Megakernel(mk.Config.from_shape(w.shape, 1, max_seq), w, 0, tp_ranks=ranks)


def fill_cache(m, kv, length, ranks):
    """kv: oracle layout [layer][K|V][1][n_kv][length][head_dim]; rank r holds heads r*n_kv/ranks..."""
    per = kv.shape[3] // ranks
    view = m.kv_view()
    for r in range(ranks):
        view[r, :, :, :, :, :length, :] = torch.from_numpy(kv[:, :, :, r * per:(r + 1) * per].view(np.int16)).to(DEV)


def gather_cache(m, length, ranks):
    """The ranks' caches back in the oracle layout [layer][K|V][1][n_kv][length][head_dim]."""
    v = m.kv_view()[:, :, :, :, :, :length, :].cpu().numpy()
    return np.concatenate([v[r] for r in range(ranks)], axis=3)


def step_both(ref, m, tok, label):
    rl = ref.decode(np.array([tok], dtype=np.int32))[0]
    g, nt = m.decode(torch.tensor([tok], dtype=torch.int32, device=DEV))
    g = g[0].cpu().numpy()
    logits_close(g, rl, label)
    assert argmax_agrees(g, rl, int(nt[0].item())), f"{label}: argmax differs with a clear margin"
    return oracle.argmax(rl)


@pytest.mark.parametrize("shape,ranks,head_keys", [(mi.TINY, 2, 256), (mi.LLAMA8B.with_layers(2), 2, 256),
                                                   (mi.LLAMA8B.with_layers(2), 2, 0),
                                                   (mi.LLAMA8B.with_layers(2), 4, 256)])
def test_tp_decode_over_a_filled_cache(shape, ranks, head_keys):
    # head_keys 256: the attention of every step in head mode; 0: the keys split and merged
    w = mi.make_weights(shape, seed=31)
    L0, steps, max_seq = 100, 4, 128
    kv = mi.kv_cache_values(31, shape, 1, L0, sigma=1.0)
    ref = oracle.Decoder(w, 1, max_seq)
    ref.set_cache(kv, L0)
    m = tp_model(w, ranks, max_seq)
    mk.mk_set_attn_head_keys(m.ctx, head_keys)
    fill_cache(m, kv, L0, ranks)
    m.set_positions([L0])
    tok = int(mi.prompt(31, 0, 1, shape.vocab)[0])
    for i in range(steps):
        tok = step_both(ref, m, tok, f"{shape.name} x{ranks} step {i}")
    assert m.sync_status() == mk.MK_OK
    n = L0 + steps
    kv_close(gather_cache(m, n, ranks)[:, :, :, :, L0:n], ref.get_cache(n)[:, :, :, :, L0:n], "kv cache")
    m.close()


def test_tp_prompt_as_decode_steps_then_greedy_launches():
    """From an empty cache: the prompt is fed one decode step per token (position 0 upwards),
    then greedy steps, one per launch and several per launch (the argmax exchanged on the
    device feeds the next step's embedding)."""
    w = mi.make_weights(mi.TINY, seed=32)
    prompt = mi.prompt(32, 0, 20, w.shape.vocab)
    ref = oracle.Decoder(w, 1, 64)
    m = tp_model(w, 2, 64)
    m.set_positions([0])
    for i, p in enumerate(prompt[:-1]):
        ref.decode(np.array([p], dtype=np.int32))
        m.decode(torch.tensor([int(p)], dtype=torch.int32, device=DEV))
    tok = step_both(ref, m, int(prompt[-1]), "last prompt token")
    for i in range(3):
        tok = step_both(ref, m, tok, f"greedy step {i}")
    n = len(prompt) + 3
    kv_close(gather_cache(m, n, 2), ref.get_cache(n), "kv cache")
    # 6 greedy steps in one launch: tokens and last logits against the oracle's greedy run
    want = []
    t = tok
    for _ in range(6):
        rl = ref.decode(np.array([t], dtype=np.int32))[0]
        t = oracle.argmax(rl)
        want.append(t)
    lg, toks = m.decode_steps(torch.tensor([tok], dtype=torch.int32, device=DEV), 6)
    assert m.sync_status() == mk.MK_OK
    assert [int(x) for x in toks[:, 0].cpu().numpy()] == want
    logits_close(lg[0].cpu().numpy(), rl, "last step of the multi-step launch")
    m.close()


def test_tp_matches_the_single_rank_kernel():
    """The same model, unsharded on the ordinary kernel and split over 2 ranks: logits close."""
    w = mi.make_weights(mi.TINY, seed=33)
    kv = mi.kv_cache_values(33, w.shape, 1, 30, sigma=1.0)
    one = mk.Megakernel(mk.Config.from_shape(w.shape, 1, 48), w, 0)
    one.kv_view()[:, :, :1, :, :30, :] = torch.from_numpy(kv.view(np.int16)).to(DEV)
    one.set_positions([30])
    two = tp_model(w, 2, 48)
    fill_cache(two, kv, 30, 2)
    two.set_positions([30])
    tok = torch.tensor([5], dtype=torch.int32, device=DEV)
    for i in range(4):
        a, na = one.decode(tok)
        b, nb = two.decode(tok)
        a, b = a[0].cpu().numpy(), b[0].cpu().numpy()
        assert np.abs(a - b).max() <= 1e-3, f"step {i}: {np.abs(a - b).max():.3e}"
        tok = na.clone()
    one.close()
    two.close()


def test_tp_dropped_signal_times_out_cleanly():
    """A remote signal that never comes (the test hook drops the notify of layer 0's O tasks on
    every rank) makes the waiting tasks give up after the wait limit: MK_ERR_DEVICE_TIMEOUT,
    nothing faults, and the context decodes correctly afterwards."""
    w = mi.make_weights(mi.TINY, seed=34)
    kv = mi.kv_cache_values(34, w.shape, 1, 12, sigma=1.0)
    m = tp_model(w, 2, 32)
    fill_cache(m, kv, 12, 2)
    m.set_positions([12])
    mk.mk_set_wait_timeout_ns(m.ctx, 100_000_000)
    tasks, _ = mk.mk_export_taskgraph_tp(m.ctx)
    F = {name: i for i, name in enumerate(mk.TP_FIELDS)}
    ev_o0 = int(tasks[(tasks[:, F["kind"]] == 4) & (tasks[:, F["layer"]] == 0)][0, F["notify0"]])
    mk.mk_debug_drop_notify(m.ctx, ev_o0, True)
    m.decode(torch.tensor([3], dtype=torch.int32, device=DEV))
    assert m.sync_status() == mk.MK_ERR_DEVICE_TIMEOUT
    assert "timed out" in mk.mk_last_error(m.ctx)
    mk.mk_debug_drop_notify(m.ctx, ev_o0, False)
    ref = oracle.Decoder(w, 1, 32)
    ref.set_cache(kv, 12)
    fill_cache(m, kv, 12, 2)
    m.set_positions([12])
    step_both(ref, m, 3, "after recovery")
    assert m.sync_status() == mk.MK_OK
    m.close()
