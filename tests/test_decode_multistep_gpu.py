"""Several greedy decode steps in one launch of the persistent kernel (the token picked by a
step feeds the next step's embedding on the device) against the same number of one-step
launches fed with their own picks: identical tokens, last-step logits within rounding
(the attention of later steps reads the rows written inside the launch in another order)."""
import numpy as np
import pytest
import torch

import mk_inputs as mi
import oracle
import persistent_megakernel_decode_04_b200 as mk
from _parity import argmax_agrees, logits_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _model(w, max_batch, max_seq):
    return mk.Megakernel(mk.Config.from_shape(w.shape, max_batch, max_seq), w, 0)


def _prefilled(w, B, max_batch, T, max_seq, seed):
    prompts = np.stack([mi.prompt(seed, b, T, w.shape.vocab) for b in range(B)]).astype(np.int32)
    m = _model(w, max_batch, max_seq)
    lg = m.prefill(torch.from_numpy(prompts).to(DEV))
    first = torch.argmax(lg[:B], dim=1).to(torch.int32)
    return m, prompts, first


def _compare(w, B, max_batch, T, steps, max_seq, seed):
    a, prompts, first = _prefilled(w, B, max_batch, T, max_seq, seed)
    tok = first.clone()
    picks = []
    for _ in range(steps):
        lg_a, nt = a.decode(tok)
        tok = nt.clone()
        picks.append(tok.cpu().numpy().copy())
    lg_a = lg_a.cpu().numpy().copy()
    assert a.sync_status() == mk.MK_OK
    b, _, first_b = _prefilled(w, B, max_batch, T, max_seq, seed)
    lg_b, out = b.decode_steps(first_b, steps)
    assert b.sync_status() == mk.MK_OK
    assert np.array_equal(out.cpu().numpy(), np.stack(picks)), "multi-step picks differ from one-step launches"
    lg_b = lg_b.cpu().numpy()
    assert np.abs(lg_a - lg_b).max() <= 1e-3
    assert b.positions()[:B] == a.positions()[:B]
    a.close()
    b.close()
    return prompts, first.cpu().numpy(), np.stack(picks), lg_b


def test_tiny_single_sequence_8_steps_in_one_launch():
    w = mi.make_weights(mi.TINY, seed=20)
    prompts, first, picks, lg = _compare(w, 1, 1, 16, 8, 64, 20)
    # and the launch against the oracle fed the same tokens
    ref = oracle.Decoder(w, 1, 64)
    ref.prefill(prompts[0])
    toks = [int(first[0])] + [int(p[0]) for p in picks[:-1]]
    for i, t in enumerate(toks):
        rl = ref.decode(np.array([t], dtype=np.int32))[0]
        assert argmax_agrees(rl, rl, int(picks[i][0])), f"step {i}: pick is not the oracle's argmax"
    logits_close(lg[0], rl, "last step")


def test_tiny_batch4_multi_step():
    w = mi.make_weights(mi.TINY, seed=21)
    _compare(w, 3, 4, 10, 6, 32, 21)


def test_tiny_batch16_tensor_core_multi_step():
    w = mi.make_weights(mi.TINY, seed=22)
    _compare(w, 16, 16, 8, 5, 32, 22)


def test_llama8b_two_layers_long_context_multi_step():
    # split-KV over many chunks: rows written by earlier steps of the launch sit in the last one
    shape = mi.LLAMA8B.with_layers(2)
    w = mi.make_weights(shape, seed=23)
    L, steps = 700, 6
    kv = mi.kv_cache_values(23, shape, 1, L, sigma=1.0)
    runs = []
    for multi in (False, True):
        m = _model(w, 1, L + 16)
        m.kv_view()[:, :, :1, :, :L, :] = torch.from_numpy(kv.view(np.int16)).to(DEV)
        m.set_positions([L])
        tok = torch.tensor([int(mi.prompt(23, 0, 1, shape.vocab)[0])], dtype=torch.int32, device=DEV)
        if multi:
            lg, out = m.decode_steps(tok, steps)
            picks = out.cpu().numpy()[:, 0]
        else:
            picks = []
            for _ in range(steps):
                lg, nt = m.decode(tok)
                tok = nt.clone()
                picks.append(int(tok.item()))
            picks = np.array(picks)
        assert m.sync_status() == mk.MK_OK
        runs.append((picks, lg[0].cpu().numpy().copy()))
        m.close()
    assert np.array_equal(runs[0][0], runs[1][0])
    assert np.abs(runs[0][1] - runs[1][1]).max() <= 1e-3


def test_multi_step_argument_checks():
    w = mi.make_weights(mi.TINY, seed=24)
    m, _, first = _prefilled(w, 1, 1, 4, 8, 24)
    with pytest.raises(mk.MkError):
        m.decode_steps(first, 5)  # 4 + 5 > max_seq 8
    with pytest.raises(mk.MkError):
        mk.mk_decode_steps(m.ctx, first, 2, m.kv, m.logits, None)  # tokens_out required
    lg, out = m.decode_steps(first, 4)
    assert m.sync_status() == mk.MK_OK and m.positions()[0] == 8
    m.close()
