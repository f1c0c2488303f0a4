"""Full-size parity: Llama-3-8B-shaped decoder, batch 1, in the launch configuration the
bench times (one persistent grid, 1 CTA per SM).  Teacher-forced on the oracle's tokens.
Weights are 16 GB of seeded bf16; the oracle runs row-parallel on the host cores."""
import numpy as np
import pytest
import torch

import mk_inputs as mi
import oracle
import persistent_megakernel_decode_04_b200 as mk
from _parity import argmax_agrees, kv_close, logits_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module")
def w8b():
    return mi.make_weights(mi.LLAMA8B, seed=0)


def test_llama8b_prompt39_decode(w8b):
    w = w8b
    prompt = mi.prompt(0, 0, 39, w.shape.vocab)
    steps, max_seq = 3, 64
    ref = oracle.Decoder(w, 1, max_seq)
    m = mk.Megakernel(mk.Config.from_shape(w.shape, 1, max_seq), w, 0)
    rl = ref.prefill(prompt)[0]
    gl = m.prefill(torch.from_numpy(prompt[None].astype(np.int32)).to(DEV))[0].cpu().numpy()
    logits_close(gl, rl, "prefill")
    tok = oracle.argmax(rl)
    for i in range(steps):
        rl = ref.decode(np.array([tok], dtype=np.int32))[0]
        g, nt = m.decode(torch.tensor([tok], dtype=torch.int32, device=DEV))
        g = g[0].cpu().numpy()
        logits_close(g, rl, f"step {i}")
        assert argmax_agrees(g, rl, int(nt[0].item()))
        tok = oracle.argmax(rl)
    assert m.sync_status() == mk.MK_OK
    n = 39 + steps
    kv_close(m.kv_view()[:, :, :1, :, :n, :].cpu().numpy(), ref.get_cache(n), "kv cache")
    m.close()


def test_llama8b_4096_context(w8b):
    """Long context: 4096 cached positions (a seeded synthetic cache standing in for the
    4096-token prompt), 2 decode steps; split-KV attention spans every chunk."""
    w = w8b
    s = w.shape
    L, steps, max_seq = 4096, 2, 4112
    kv = mi.kv_cache_values(4, s, 1, L, sigma=1.0)
    ref = oracle.Decoder(w, 1, max_seq)
    ref.set_cache(kv, L)
    m = mk.Megakernel(mk.Config.from_shape(s, 1, max_seq), w, 0)
    m.kv_view()[:, :, :1, :, :L, :] = torch.from_numpy(kv.view(np.int16)).to(DEV)
    del kv
    m.set_positions([L])
    tok = int(mi.prompt(4, 0, 1, s.vocab)[0])
    for i in range(steps):
        rl = ref.decode(np.array([tok], dtype=np.int32))[0]
        g, nt = m.decode(torch.tensor([tok], dtype=torch.int32, device=DEV))
        g = g[0].cpu().numpy()
        logits_close(g, rl, f"step {i}")
        assert argmax_agrees(g, rl, int(nt[0].item()))
        tok = oracle.argmax(rl)
    assert m.sync_status() == mk.MK_OK
    n = L + steps
    got = m.kv_view()[:, :, :1, :, L:n, :].cpu().numpy()
    kv_close(got, ref.get_cache(n)[:, :, :, :, L:n], "kv cache (appended positions)")
    m.close()
