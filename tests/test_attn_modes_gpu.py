"""Decode attention in head mode (short lengths: chunk task c < G computes query head c of its
KV head over every key and stores the output, no partial merged) and in split mode (the keys
split over the chunk tasks, the last to arrive merging the partials), and the switch from one
to the other inside a multi-step launch and across launches, against the CPU oracle
teacher-forced on its tokens.  The split is FlashDecoding's, which the Mirage article's
attention example names; head mode is the same attention with the key split taken away."""
import numpy as np
import pytest
import torch

import mk_inputs as mi
import oracle
import persistent_megakernel_decode_04_b200 as mk
from _parity import argmax_agrees, kv_close, logits_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _filled(w, L0, max_seq, head_keys, seed):
    kv = mi.kv_cache_values(seed, w.shape, 1, L0, sigma=1.0)
    m = mk.Megakernel(mk.Config.from_shape(w.shape, 1, max_seq), w, 0)
    mk.mk_set_attn_head_keys(m.ctx, head_keys)
    m.kv_view()[:, :, :1, :, :L0, :] = torch.from_numpy(kv.view(np.int16)).to(DEV)
    m.set_positions([L0])
    return m, kv


def _step_both(ref, m, tok, label):
    rl = ref.decode(np.array([tok], dtype=np.int32))[0]
    g, nt = m.decode(torch.tensor([tok], dtype=torch.int32, device=DEV))
    g = g[0].cpu().numpy()
    logits_close(g, rl, label)
    assert argmax_agrees(g, rl, int(nt[0].item())), f"{label}: argmax differs with a clear margin"
    return oracle.argmax(rl)


@pytest.mark.parametrize("head_keys", [0, 1 << 20], ids=["split", "head"])
def test_llama8b_two_layers_each_mode_over_a_filled_cache(head_keys):
    shape = mi.LLAMA8B.with_layers(2)
    w = mi.make_weights(shape, seed=41)
    L0, steps, max_seq = 300, 3, 320
    m, kv = _filled(w, L0, max_seq, head_keys, 41)
    ref = oracle.Decoder(w, 1, max_seq)
    ref.set_cache(kv, L0)
    tok = int(mi.prompt(41, 0, 1, shape.vocab)[0])
    for i in range(steps):
        tok = _step_both(ref, m, tok, f"head_keys={head_keys} step {i}")
    assert m.sync_status() == mk.MK_OK
    n = L0 + steps
    got = m.kv_view()[:, :, :1, :, L0:n, :].cpu().numpy()
    kv_close(got, ref.get_cache(n)[:, :, :, :, L0:n], "new cache rows")
    m.close()


def test_llama8b_two_layers_switch_inside_and_across_launches():
    """head_keys = L0 + 3: the first three steps of an 8-step launch run in head mode, the rest
    split; the split steps' arrival counts must go on from where the head-mode steps left them,
    in the same launch and in the next one."""
    shape = mi.LLAMA8B.with_layers(2)
    w = mi.make_weights(shape, seed=42)
    L0, steps, more, max_seq = 120, 8, 4, 160
    tok0 = int(mi.prompt(42, 0, 1, shape.vocab)[0])
    # one step per launch
    a, kv = _filled(w, L0, max_seq, L0 + 3, 42)
    tok = torch.tensor([tok0], dtype=torch.int32, device=DEV)
    picks = []
    for _ in range(steps + more):
        lg_a, nt = a.decode(tok)
        tok = nt.clone()
        picks.append(int(tok.item()))
        if len(picks) == steps:
            lg_a_mid = lg_a[0].cpu().numpy().copy()
    lg_a = lg_a[0].cpu().numpy().copy()
    assert a.sync_status() == mk.MK_OK
    a.close()
    # the same steps as two multi-step launches
    b, _ = _filled(w, L0, max_seq, L0 + 3, 42)
    lg_b, out = b.decode_steps(torch.tensor([tok0], dtype=torch.int32, device=DEV), steps)
    lg_b_mid = lg_b[0].cpu().numpy().copy()
    first = out[-1].clone()
    lg_b2, out2 = b.decode_steps(first, more)
    assert b.sync_status() == mk.MK_OK
    got = np.concatenate([out.cpu().numpy()[:, 0], out2.cpu().numpy()[:, 0]])
    assert np.array_equal(got, np.array(picks)), "multi-step picks differ from one-step launches"
    assert np.abs(lg_b_mid - lg_a_mid).max() <= 1e-3
    assert np.abs(lg_b2[0].cpu().numpy() - lg_a).max() <= 1e-3
    b.close()
    # and the picks against the oracle fed the same tokens
    ref = oracle.Decoder(w, 1, max_seq)
    ref.set_cache(kv, L0)
    toks = [tok0] + picks[:-1]
    for i, t in enumerate(toks):
        rl = ref.decode(np.array([t], dtype=np.int32))[0]
        assert argmax_agrees(rl, rl, picks[i]), f"step {i}: pick is not the oracle's argmax"
    logits_close(lg_a, rl, "last step")


def test_tiny_prompt_crosses_the_head_mode_limit():
    """Tiny model (2 query heads per KV head): head mode up to 20 keys, then split, one step per
    launch, every step against the oracle."""
    w = mi.make_weights(mi.TINY, seed=43)
    prompt = mi.prompt(43, 0, 16, w.shape.vocab)
    m = mk.Megakernel(mk.Config.from_shape(w.shape, 1, 64), w, 0)
    mk.mk_set_attn_head_keys(m.ctx, 20)
    ref = oracle.Decoder(w, 1, 64)
    rl = ref.prefill(prompt)[0]
    lg = m.prefill(torch.from_numpy(prompt[None].astype(np.int32)).to(DEV))
    logits_close(lg[0].cpu().numpy(), rl, "prefill")
    tok = oracle.argmax(rl)
    for i in range(10):  # lengths 17 .. 26
        tok = _step_both(ref, m, tok, f"step {i}")
    assert m.sync_status() == mk.MK_OK
    m.close()


def test_head_keys_argument_checks():
    w = mi.make_weights(mi.TINY, seed=44)
    m = mk.Megakernel(mk.Config.from_shape(w.shape, 1, 16), w, 0)
    with pytest.raises(mk.MkError):
        mk.mk_set_attn_head_keys(m.ctx, -1)
    with pytest.raises(mk.MkError):
        mk.mk_set_attn_head_keys(m.ctx, (1 << 20) + 1)
    mk.mk_set_attn_head_keys(m.ctx, 0)
    m.close()


@pytest.mark.parametrize("head_keys,L0", [(1 << 20, 300), (0, 2400)], ids=["head", "split"])
def test_llama8b_two_layers_whole_stage_chunks_with_fresh_rows(head_keys, L0):
    """Chunks of three or more ring stages (whole stages per warp or warp pair) while a 12-step
    launch writes fresh rows: the fresh rows go to the warps after those of the stages, the
    first two of each such warp fetched with q.  Picks and logits against one-step launches, and
    every step's logits against the oracle fed the same tokens."""
    shape = mi.LLAMA8B.with_layers(2)
    w = mi.make_weights(shape, seed=45)
    steps, max_seq = 12, L0 + 16
    tok0 = int(mi.prompt(45, 0, 1, shape.vocab)[0])
    a, kv = _filled(w, L0, max_seq, head_keys, 45)
    tok = torch.tensor([tok0], dtype=torch.int32, device=DEV)
    picks, logits = [], []
    for _ in range(steps):
        lg, nt = a.decode(tok)
        tok = nt.clone()
        picks.append(int(tok.item()))
        logits.append(lg[0].cpu().numpy().copy())
    assert a.sync_status() == mk.MK_OK
    a.close()
    b, _ = _filled(w, L0, max_seq, head_keys, 45)
    lg_b, out = b.decode_steps(torch.tensor([tok0], dtype=torch.int32, device=DEV), steps)
    assert b.sync_status() == mk.MK_OK
    assert np.array_equal(out.cpu().numpy()[:, 0], np.array(picks)), "multi-step picks differ from one-step launches"
    assert np.abs(lg_b[0].cpu().numpy() - logits[-1]).max() <= 1e-3
    n = L0 + steps
    got_kv = b.kv_view()[:, :, :1, :, L0:n, :].cpu().numpy()
    b.close()
    ref = oracle.Decoder(w, 1, max_seq)
    ref.set_cache(kv, L0)
    for i, t in enumerate([tok0] + picks[:-1]):
        rl = ref.decode(np.array([t], dtype=np.int32))[0]
        logits_close(logits[i], rl, f"head_keys={head_keys} step {i}")
        assert argmax_agrees(logits[i], rl, picks[i]), f"step {i}: pick is not the oracle's argmax with a clear margin"
    kv_close(got_kv, ref.get_cache(n)[:, :, :, :, L0:n], "rows written inside the launch")
