"""QK-norm decode (Mirage article, "Case 4.1: Attention with Query-Key Normalization", as in
Chameleon) against the CPU oracle: every query and key head goes through a LayerNorm with its
own gain and bias before RoPE.  On the GPU the QKV epilogue stores the raw projections and the
attention task of each KV head normalises and rotates q and the new key (which it writes to
the cache).  Covered: the batch-1, batch-4 (CUDA-core) and batch-16 (tensor-core) kernels,
prefill, ragged positions, several steps per launch, and the Chameleon-7B shape at 1024
cached positions."""
import numpy as np
import pytest
import torch

import mk_inputs as mi
import oracle
import persistent_megakernel_decode_04_b200 as mk
from _parity import argmax_agrees, kv_close, logits_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _model(w, max_batch, max_seq):
    cfg = mk.Config.from_shape(w.shape, max_batch, max_seq)
    assert cfg.qk_norm
    return mk.Megakernel(cfg, w, 0)


def _step_both(ref, m, toks, label):
    B = len(toks)
    rl = ref.decode(np.array(toks, dtype=np.int32))
    gl, nt = m.decode(torch.tensor(toks, dtype=torch.int32, device=DEV))
    gl, nt = gl[:B].cpu().numpy(), nt[:B].cpu().numpy()
    for b in range(B):
        logits_close(gl[b], rl[b], f"{label} seq {b}")
        assert argmax_agrees(gl[b], rl[b], int(nt[b])), f"{label} seq {b}: argmax differs with a clear margin"
    return [oracle.argmax(rl[b]) for b in range(B)]


def _teacher_forced(w, B, max_batch, T, steps, max_seq, seed):
    prompts = np.stack([mi.prompt(seed, b, T, w.shape.vocab) for b in range(B)])
    ref = oracle.Decoder(w, B, max_seq)
    m = _model(w, max_batch, max_seq)
    rl = ref.prefill(prompts)
    gl = m.prefill(torch.from_numpy(prompts.astype(np.int32)).to(DEV)).cpu().numpy()
    for b in range(B):
        logits_close(gl[b], rl[b], f"prefill seq {b}")
    kv_close(m.kv_view()[:, :, :B, :, :T, :].cpu().numpy(), ref.get_cache(T), "kv cache after prefill")
    toks = [oracle.argmax(rl[b]) for b in range(B)]
    for i in range(steps):
        toks = _step_both(ref, m, toks, f"step {i}")
    assert m.sync_status() == mk.MK_OK
    n = T + steps
    kv_close(m.kv_view()[:, :, :B, :, :n, :].cpu().numpy(), ref.get_cache(n), "kv cache")
    m.close()


@pytest.fixture(scope="module")
def w_tiny():
    w = mi.make_weights(mi.TINY_QK, seed=30, sigma=0.05)
    return w


def test_qk_norm_single_sequence(w_tiny):
    _teacher_forced(w_tiny, B=1, max_batch=1, T=12, steps=16, max_seq=64, seed=30)


def test_qk_norm_batch4(w_tiny):
    _teacher_forced(w_tiny, B=4, max_batch=4, T=9, steps=10, max_seq=32, seed=31)


def test_qk_norm_batch16_tensor_core(w_tiny):
    _teacher_forced(w_tiny, B=16, max_batch=16, T=10, steps=8, max_seq=32, seed=32)


def test_qk_norm_long_prompt_crossing_chunks(w_tiny):
    # 200 positions: several split-KV chunks; the new key sits in the last one
    _teacher_forced(w_tiny, B=1, max_batch=1, T=200, steps=4, max_seq=256, seed=33)


@pytest.mark.parametrize("max_batch", [4, 16])
def test_qk_norm_ragged_positions(w_tiny, max_batch):
    w = w_tiny
    s = w.shape
    L = 50
    B = 4
    kv = mi.kv_cache_values(34, s, B, L, sigma=1.0)
    pos = [50, 17, 33, 1]
    ref = oracle.Decoder(w, B, 64)
    ref.set_cache(kv, L)
    ref.set_positions(pos)
    m = _model(w, max_batch, 64)
    m.kv_view()[:, :, :B, :, :L, :] = torch.from_numpy(kv.view(np.int16)).to(DEV)
    m.set_positions(pos)
    toks = [3, 99, 512, 1000]
    for i in range(5):
        toks = _step_both(ref, m, toks, f"step {i}")
    assert m.sync_status() == mk.MK_OK
    got = m.kv_view()[:, :, :B, :, :56, :].cpu().numpy()
    want = ref.get_cache(56)
    for b in range(B):
        n = pos[b] + 5
        kv_close(got[:, :, b:b + 1, :, :n], want[:, :, b:b + 1, :, :n], f"kv cache seq {b}")
    m.close()


@pytest.mark.parametrize("B,max_batch", [(1, 1), (3, 4), (16, 16)])
def test_qk_norm_multi_step_launch(w_tiny, B, max_batch):
    # n greedy steps in one launch: the key of each step is normalised by that step's attention
    # task and read from the cache by the later steps of the same launch
    w = w_tiny
    T, steps, max_seq = 11, 7, 32
    prompts = np.stack([mi.prompt(35, b, T, w.shape.vocab) for b in range(B)]).astype(np.int32)
    m = _model(w, max_batch, max_seq)
    lg = m.prefill(torch.from_numpy(prompts).to(DEV))
    first = torch.argmax(lg[:B], dim=1).to(torch.int32)
    lg_m, out = m.decode_steps(first, steps)
    assert m.sync_status() == mk.MK_OK
    picks = out.cpu().numpy()[:, :B]
    lg_m = lg_m[:B].cpu().numpy()
    ref = oracle.Decoder(w, B, max_seq)
    ref.prefill(prompts)
    toks = first.cpu().numpy()
    for i in range(steps):
        rl = ref.decode(np.asarray(toks, dtype=np.int32))
        for b in range(B):
            assert argmax_agrees(rl[b], rl[b], int(picks[i][b])), f"step {i} seq {b}: pick is not the oracle's argmax"
        toks = picks[i]
    for b in range(B):
        logits_close(lg_m[b], rl[b], f"last step seq {b}")
    n = T + steps
    kv_close(m.kv_view()[:, :, :B, :, :n, :].cpu().numpy(), ref.get_cache(n), "kv cache")
    m.close()


@pytest.fixture(scope="module")
def w_chameleon_qk():
    return mi.make_weights(mi.CHAMELEON7B_QK, seed=0)


@pytest.mark.parametrize("B", [1, 4, 16])
def test_chameleon7b_qk_norm_1024_context(w_chameleon_qk, B):
    """Chameleon-7B shape with QK-norm, every sequence at 1024 cached positions (a seeded
    synthetic cache of unit-variance keys standing in for the normalised keys of 1024-token
    prompts), 2 decode steps."""
    w = w_chameleon_qk
    s = w.shape
    L, steps, max_seq = 1024, 2, 1040
    kv = mi.kv_cache_values(36, s, B, L, sigma=1.0)
    ref = oracle.Decoder(w, B, max_seq)
    ref.set_cache(kv, L)
    m = _model(w, B, max_seq)
    m.kv_view()[:, :, :B, :, :L, :] = torch.from_numpy(kv.view(np.int16)).to(DEV)
    del kv
    m.set_positions([L] * B)
    toks = [int(t) for t in mi.prompt(36, 0, B, s.vocab)]
    for i in range(steps):
        toks = _step_both(ref, m, toks, f"step {i}")
    assert m.sync_status() == mk.MK_OK
    n = L + steps
    got = m.kv_view()[:, :, :B, :, L:n, :].cpu().numpy()
    kv_close(got, ref.get_cache(n)[:, :, :, :, L:n], "kv cache (appended positions)")
    m.close()
