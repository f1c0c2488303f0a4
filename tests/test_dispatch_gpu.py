"""Scheduling variant: projection tasks claimed at run time from per-op pools (MK_DISPATCH_CLAIM;
paced; with priority to the attention chunks of the critical path) instead of fixed per-SM queues.  The result must not depend on which SM ran which task: parity
with the oracle, with the static schedule (one-step and multi-step launches, where the claim
counters of a step are recycled two steps later), and clean timeouts."""
import numpy as np
import pytest
import torch

import mk_inputs as mi
import oracle
import persistent_megakernel_decode_04_b200 as mk
from _parity import argmax_agrees, logits_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _model(w, max_seq, tps=None, mode=mk.MK_DISPATCH_CLAIM):
    m = mk.Megakernel(mk.Config.from_shape(w.shape, 1, max_seq), w, 0)
    if tps:
        m.set_dispatch(mode, tps)
    return m


@pytest.mark.parametrize("tps,mode", [(1, mk.MK_DISPATCH_CLAIM), (2, mk.MK_DISPATCH_CLAIM), (4, mk.MK_DISPATCH_CLAIM),
                                      (2, mk.MK_DISPATCH_CLAIM_PACED), (2, mk.MK_DISPATCH_CLAIM_PRIORITY)])
def test_claims_match_the_oracle(tps, mode):
    w = mi.make_weights(mi.TINY, seed=40)
    prompt = mi.prompt(40, 0, 14, w.shape.vocab)
    ref = oracle.Decoder(w, 1, 64)
    m = _model(w, 64, tps, mode)
    rl = ref.prefill(prompt)[0]
    m.prefill(torch.from_numpy(prompt[None].astype(np.int32)).to(DEV))
    tok = oracle.argmax(rl)
    for i in range(12):
        rl = ref.decode(np.array([tok], dtype=np.int32))[0]
        gl, nt = m.decode(torch.tensor([tok], dtype=torch.int32, device=DEV))
        gl = gl[0].cpu().numpy()
        logits_close(gl, rl, f"step {i}")
        assert argmax_agrees(gl, rl, int(nt[0].item())), f"step {i}: argmax differs with a clear margin"
        tok = oracle.argmax(rl)
    assert m.sync_status() == mk.MK_OK
    m.close()


def _run(w, max_seq, tps, prompt_or_cache, steps, multi, mode=mk.MK_DISPATCH_CLAIM):
    m = _model(w, max_seq, tps, mode)
    if isinstance(prompt_or_cache, tuple):
        kv, L = prompt_or_cache
        m.kv_view()[:, :, :1, :, :L, :] = torch.from_numpy(kv.view(np.int16)).to(DEV)
        m.set_positions([L])
        tok = torch.tensor([int(mi.prompt(41, 0, 1, w.shape.vocab)[0])], dtype=torch.int32, device=DEV)
    else:
        lg = m.prefill(torch.from_numpy(prompt_or_cache[None].astype(np.int32)).to(DEV))
        tok = torch.argmax(lg[:1], dim=1).to(torch.int32)
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
    res = picks, lg[0].cpu().numpy().copy()
    m.close()
    return res


@pytest.mark.parametrize("multi", [False, True])
def test_claims_equal_static_schedule_tiny(multi):
    # 9 steps in one launch: the claim counters of each step are zeroed by the token pick of
    # the step two before and reused
    w = mi.make_weights(mi.TINY, seed=42)
    prompt = mi.prompt(42, 0, 10, w.shape.vocab)
    a = _run(w, 32, None, prompt, 9, multi)
    for tps, mode in ((1, mk.MK_DISPATCH_CLAIM), (3, mk.MK_DISPATCH_CLAIM), (2, mk.MK_DISPATCH_CLAIM_PACED),
                      (2, mk.MK_DISPATCH_CLAIM_PRIORITY)):
        b = _run(w, 32, tps, prompt, 9, multi, mode)
        assert np.array_equal(a[0], b[0])
        assert np.abs(a[1] - b[1]).max() <= 1e-3


def test_claims_equal_static_schedule_llama8b_two_layers():
    shape = mi.LLAMA8B.with_layers(2)
    w = mi.make_weights(shape, seed=43)
    L = 600
    kv = mi.kv_cache_values(43, shape, 1, L, sigma=1.0)
    a = _run(w, L + 16, None, (kv, L), 5, True)
    b = _run(w, L + 16, 2, (kv, L), 5, True)
    c = _run(w, L + 16, 2, (kv, L), 5, False)
    d = _run(w, L + 16, 2, (kv, L), 5, True, mk.MK_DISPATCH_CLAIM_PACED)
    e = _run(w, L + 16, 2, (kv, L), 5, True, mk.MK_DISPATCH_CLAIM_PRIORITY)
    for r in (b, c, d, e):
        assert np.array_equal(a[0], r[0])
        assert np.abs(a[1] - r[1]).max() <= 1e-3


def test_claims_switch_back_and_forth_and_time_out_cleanly():
    w = mi.make_weights(mi.TINY, seed=44)
    prompt = mi.prompt(44, 0, 8, w.shape.vocab)
    ref = oracle.Decoder(w, 1, 32)
    rl = ref.prefill(prompt)[0]
    m = _model(w, 32, 2)
    m.prefill(torch.from_numpy(prompt[None].astype(np.int32)).to(DEV))
    mk.mk_set_wait_timeout_ns(m.ctx, 100_000_000)  # 0.1 s
    mk.mk_debug_drop_notify(m.ctx, 4, True)  # layer 0's O-projection event: its pool never completes
    m.decode(torch.tensor([1], dtype=torch.int32, device=DEV))
    assert m.sync_status() == mk.MK_ERR_DEVICE_TIMEOUT
    mk.mk_debug_drop_notify(m.ctx, 4, False)
    # recover, then alternate the dispatch modes step by step against the oracle
    m.prefill(torch.from_numpy(prompt[None].astype(np.int32)).to(DEV))
    tok = oracle.argmax(rl)
    for i in range(6):
        m.set_dispatch(mk.MK_DISPATCH_CLAIM if i % 2 else mk.MK_DISPATCH_STATIC, 2)
        rl = ref.decode(np.array([tok], dtype=np.int32))[0]
        gl, _ = m.decode(torch.tensor([tok], dtype=torch.int32, device=DEV))
        logits_close(gl[0].cpu().numpy(), rl, f"step {i}")
        tok = oracle.argmax(rl)
    assert m.sync_status() == mk.MK_OK
    m.close()
