"""Batched decode against the CPU oracle, teacher-forced per sequence on the oracle's tokens:
2..16 sequences on the tensor-core kernel (the default), and 2..4 also on the CUDA-core
batch-4 kernel (tc_min_batch = 5).  Per-step
logits of every sequence, argmax, the bf16 KV cache, masking of sequences outside the active
batch and per-sequence positions."""
import numpy as np
import pytest
import torch

import mk_inputs as mi
import oracle
import persistent_megakernel_decode_04_b200 as mk
from _parity import argmax_agrees, kv_close, logits_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _model(weights, max_batch, max_seq, tc_min=0):
    cfg = mk.Config.from_shape(weights.shape, max_batch, max_seq)
    cfg.tc_min_batch = tc_min
    return mk.Megakernel(cfg, weights, 0)


def _step_both(ref, m, toks, label):
    """One decode step on both sides with the same per-sequence tokens; returns the oracle's picks."""
    B = len(toks)
    rl = ref.decode(np.array(toks, dtype=np.int32))
    gl, nt = m.decode(torch.tensor(toks, dtype=torch.int32, device=DEV))
    gl, nt = gl[:B].cpu().numpy(), nt[:B].cpu().numpy()
    for b in range(B):
        logits_close(gl[b], rl[b], f"{label} seq {b}")
        assert argmax_agrees(gl[b], rl[b], int(nt[b])), f"{label} seq {b}: argmax differs with a clear margin"
    return [oracle.argmax(rl[b]) for b in range(B)]


def _teacher_forced_batch(w, B, max_batch, T, steps, max_seq, seed, tc_min=0):
    prompts = np.stack([mi.prompt(seed, b, T, w.shape.vocab) for b in range(B)])
    ref = oracle.Decoder(w, B, max_seq)
    m = _model(w, max_batch, max_seq, tc_min)
    rl = ref.prefill(prompts)
    gl = m.prefill(torch.from_numpy(prompts.astype(np.int32)).to(DEV)).cpu().numpy()
    for b in range(B):
        logits_close(gl[b], rl[b], f"prefill seq {b}")
    toks = [oracle.argmax(rl[b]) for b in range(B)]
    for i in range(steps):
        toks = _step_both(ref, m, toks, f"step {i}")
    assert m.sync_status() == mk.MK_OK
    n = T + steps
    kv_close(m.kv_view()[:, :, :B, :, :n, :].cpu().numpy(), ref.get_cache(n), "kv cache")
    m.close()


@pytest.mark.parametrize("tc_min", [0, 5], ids=["tensor-core", "cuda-core"])
def test_tiny_batch4_prefill_and_16_steps(tc_min):
    w = mi.make_weights(mi.TINY, seed=5)
    _teacher_forced_batch(w, B=4, max_batch=4, T=12, steps=16, max_seq=64, seed=5, tc_min=tc_min)


@pytest.mark.parametrize("tc_min", [0, 5], ids=["tensor-core", "cuda-core"])
@pytest.mark.parametrize("B", [1, 2, 3])
def test_tiny_partial_batch_is_masked(B, tc_min):
    # a batched kernel serving fewer sequences: the unused slots compute nothing visible
    w = mi.make_weights(mi.TINY, seed=6)
    _teacher_forced_batch(w, B=B, max_batch=4, T=9, steps=6, max_seq=32, seed=6 + B, tc_min=tc_min)


@pytest.mark.parametrize("tc_min", [0, 5], ids=["tensor-core", "cuda-core"])
def test_tiny_batch4_ragged_positions(tc_min):
    # every sequence at its own position: RoPE angle, cache slot and attention length per sequence
    w = mi.make_weights(mi.TINY, seed=7)
    s = w.shape
    L = 50
    kv = mi.kv_cache_values(7, s, 4, L, sigma=1.0)
    pos = [50, 17, 33, 1]
    ref = oracle.Decoder(w, 4, 64)
    ref.set_cache(kv, L)
    ref.set_positions(pos)
    m = _model(w, 4, 64, tc_min)
    m.kv_view()[:, :, :4, :, :L, :] = torch.from_numpy(kv.view(np.int16)).to(DEV)
    m.set_positions(pos)
    toks = [3, 99, 512, 1000]
    for i in range(6):
        toks = _step_both(ref, m, toks, f"step {i}")
    assert m.sync_status() == mk.MK_OK
    got = m.kv_view()[:, :, :4, :, :57, :].cpu().numpy()
    want = ref.get_cache(57)
    for b in range(4):  # compare each sequence over the positions it has written or read
        n = pos[b] + 6
        kv_close(got[:, :, b : b + 1, :, :n], want[:, :, b : b + 1, :, :n], f"kv cache seq {b}")


def test_tiny_batch16_tensor_core_prefill_and_12_steps():
    # more than 4 sequences: the projections run as tcgen05 tiles (weights in block layout)
    w = mi.make_weights(mi.TINY, seed=8)
    _teacher_forced_batch(w, B=16, max_batch=16, T=10, steps=12, max_seq=32, seed=8)


@pytest.mark.parametrize("B", [5, 8])
def test_tiny_tensor_core_partial_batch(B):
    w = mi.make_weights(mi.TINY, seed=9)
    _teacher_forced_batch(w, B=B, max_batch=16, T=7, steps=5, max_seq=16, seed=9 + B)


def test_tiny_batch16_ragged_positions_and_random_gains():
    # norm gains != 1 and a position per sequence, through the tensor-core path
    w = mi.make_weights(mi.TINY, seed=12, sigma=0.05)
    w.final_norm = mi.normal_bf16(12, 50, (w.shape.hidden,), sigma=0.3, mean=1.0)
    for l in range(w.shape.n_layers):
        w.attn_norm[l] = mi.normal_bf16(12, 51 + 2 * l, (w.shape.hidden,), sigma=0.3, mean=1.0)
        w.mlp_norm[l] = mi.normal_bf16(12, 52 + 2 * l, (w.shape.hidden,), sigma=0.3, mean=1.0)
    s = w.shape
    L = 40
    kv = mi.kv_cache_values(12, s, 16, L, sigma=1.0)
    pos = [int(p) for p in 1 + (np.arange(16) * 7) % L]
    ref = oracle.Decoder(w, 16, 48)
    ref.set_cache(kv, L)
    ref.set_positions(pos)
    m = _model(w, 16, 48)
    m.kv_view()[:, :, :16, :, :L, :] = torch.from_numpy(kv.view(np.int16)).to(DEV)
    m.set_positions(pos)
    toks = [int(t) for t in mi.prompt(12, 1, 16, s.vocab)]
    for i in range(4):
        toks = _step_both(ref, m, toks, f"step {i}")
    assert m.sync_status() == mk.MK_OK
    m.close()


@pytest.fixture(scope="module")
def w_chameleon():
    return mi.make_weights(mi.CHAMELEON7B, seed=0)


@pytest.mark.parametrize("B", [1, 4, 16])
def test_chameleon7b_1024_context(w_chameleon, B):
    """Chameleon-7B-shaped MHA decoder, every sequence at 1024 cached positions (a seeded
    synthetic cache standing in for the 1024-token prompts), 2 decode steps."""
    w = w_chameleon
    s = w.shape
    L, steps, max_seq = 1024, 2, 1040
    kv = mi.kv_cache_values(11, s, B, L, sigma=1.0)
    ref = oracle.Decoder(w, B, max_seq)
    ref.set_cache(kv, L)
    m = _model(w, B, max_seq)
    m.kv_view()[:, :, :B, :, :L, :] = torch.from_numpy(kv.view(np.int16)).to(DEV)
    del kv
    m.set_positions([L] * B)
    toks = [int(t) for t in mi.prompt(11, 0, B, s.vocab)]
    for i in range(steps):
        toks = _step_both(ref, m, toks, f"step {i}")
    assert m.sync_status() == mk.MK_OK
    n = L + steps
    got = m.kv_view()[:, :, :B, :, L:n, :].cpu().numpy()
    kv_close(got, ref.get_cache(n)[:, :, :, :, L:n], "kv cache (appended positions)")
    m.close()


@pytest.mark.parametrize("L0", [400, 1000])
def test_chameleon7b_two_layers_tensor_core_long_chunks_multistep(L0):
    """Tensor-core kernel, 4 sequences, chunks of 7 and 16 stages: the last quarter of each
    chunk's K/V stages is loaded into the idle operand buffers by the last warp pair (at 1000
    positions each buffer is loaded twice), the rest comes through the ring.  A 6-step launch against
    one-step launches (same picks, last logits within 1e-3), every step's logits against the
    oracle fed the same tokens, and the rows written inside the launch."""
    s = mi.CHAMELEON7B.with_layers(2)
    w = mi.make_weights(s, seed=46)
    B, steps, max_seq = 4, 6, L0 + 8
    kv = mi.kv_cache_values(46, s, B, L0, sigma=1.0)
    toks0 = [int(t) for t in mi.prompt(46, 0, B, s.vocab)]

    def filled():
        m = _model(w, B, max_seq)
        m.kv_view()[:, :, :B, :, :L0, :] = torch.from_numpy(kv.view(np.int16)).to(DEV)
        m.set_positions([L0] * B)
        return m

    a = filled()
    tok = torch.tensor(toks0, dtype=torch.int32, device=DEV)
    picks, logits = [], []
    for _ in range(steps):
        lg, nt = a.decode(tok)
        tok = nt.clone()
        picks.append(tok.cpu().numpy().copy())
        logits.append(lg[:B].cpu().numpy().copy())
    assert a.sync_status() == mk.MK_OK
    a.close()
    b = filled()
    lg_b, out = b.decode_steps(torch.tensor(toks0, dtype=torch.int32, device=DEV), steps)
    assert b.sync_status() == mk.MK_OK
    assert np.array_equal(out.cpu().numpy()[:, :B], np.stack(picks)), "multi-step picks differ from one-step launches"
    assert np.abs(lg_b[:B].cpu().numpy() - logits[-1]).max() <= 1e-3
    n = L0 + steps
    got_kv = b.kv_view()[:, :, :B, :, L0:n, :].cpu().numpy()
    b.close()
    ref = oracle.Decoder(w, B, max_seq)
    ref.set_cache(kv, L0)
    feed = [np.array(toks0, dtype=np.int32)] + [p.astype(np.int32) for p in picks[:-1]]
    for i, t in enumerate(feed):
        rl = ref.decode(t)
        for q in range(B):
            logits_close(logits[i][q], rl[q], f"step {i} sequence {q}")
            assert argmax_agrees(logits[i][q], rl[q], int(picks[i][q])), f"step {i} sequence {q}: argmax"
    kv_close(got_kv, ref.get_cache(n)[:, :, :, :, L0:n], "rows written inside the launch")
