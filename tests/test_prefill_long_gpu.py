"""Long prompts through mk_prefill against the CPU oracle, then decode on the megakernel.

Prefill runs (sequence, position) rows in chunks of at most 1024; a prompt longer than one
chunk makes the second chunk's attention read cache rows the first chunk wrote.  Two cases
cross that boundary:
  * the Llama-3-8B shape cut to 2 layers (full 128256-row LM head) with an 1100-token prompt
    (chunks of 1024 and 76 positions), then 3 decode steps on the batch-1 kernel;
  * the Chameleon-7B shape (MHA) cut to 2 layers with 16 prompts of 80 tokens (1280 rows:
    chunks of 64 and 16 positions per sequence), then 3 decode steps on the tensor-core kernel.
Compared: the last prompt token's logits of every sequence, every cache row the prompt wrote,
the decode logits and argmax (teacher-forced on the oracle's picks), and the rows decode
appended.  The prompts are seeded uniform token ids, standing in for the long prompts of the
8B 4K-context and Chameleon-7B workloads."""
import numpy as np
import pytest
import torch

import mk_inputs as mi
import oracle
import persistent_megakernel_decode_04_b200 as mk
from _parity import argmax_agrees, kv_close, logits_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _prefill_then_decode(w, B, T, steps, seed):
    max_seq = T + steps + 8
    prompts = np.stack([mi.prompt(seed, b, T, w.shape.vocab) for b in range(B)]).astype(np.int32)
    ref = oracle.Decoder(w, B, max_seq)
    m = mk.Megakernel(mk.Config.from_shape(w.shape, B, max_seq), w, 0)
    rl = ref.prefill(prompts)
    gl = m.prefill(torch.from_numpy(prompts).to(DEV)).cpu().numpy()
    for b in range(B):
        logits_close(gl[b], rl[b], f"prefill seq {b}")
        assert argmax_agrees(gl[b], rl[b]), f"prefill seq {b}: argmax differs with a clear margin"
    assert m.positions() == [T] * B
    kv_close(m.kv_view()[:, :, :B, :, :T, :].cpu().numpy(), ref.get_cache(T), "kv cache after prefill")
    toks = [oracle.argmax(rl[b]) for b in range(B)]
    for i in range(steps):
        rl = ref.decode(np.array(toks, dtype=np.int32))
        g, nt = m.decode(torch.tensor(toks, dtype=torch.int32, device=DEV))
        g, nt = g[:B].cpu().numpy(), nt[:B].cpu().numpy()
        for b in range(B):
            logits_close(g[b], rl[b], f"step {i} seq {b}")
            assert argmax_agrees(g[b], rl[b], int(nt[b])), f"step {i} seq {b}: argmax differs with a clear margin"
        toks = [oracle.argmax(rl[b]) for b in range(B)]
    assert m.sync_status() == mk.MK_OK
    n = T + steps
    kv_close(m.kv_view()[:, :, :B, :, :n, :].cpu().numpy(), ref.get_cache(n), "kv cache after decode")
    m.close()


def test_llama8b_2layer_prompt_1100():
    w = mi.make_weights(mi.LLAMA8B.with_layers(2), seed=21)
    _prefill_then_decode(w, B=1, T=1100, steps=3, seed=21)


def test_chameleon7b_2layer_16_prompts_of_80():
    w = mi.make_weights(mi.CHAMELEON7B.with_layers(2), seed=22)
    _prefill_then_decode(w, B=16, T=80, steps=3, seed=22)
