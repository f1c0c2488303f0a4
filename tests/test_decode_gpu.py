"""The persistent decode megakernel against the CPU oracle, teacher-forced on the
oracle's tokens: per-step logits, argmax, and the bf16 KV cache."""
import numpy as np
import pytest
import torch

import mk_inputs as mi
import oracle
import persistent_megakernel_decode_04_b200 as mk
from _parity import argmax_agrees, kv_close, logits_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def gpu_model(weights, max_seq, max_batch=1):
    cfg = mk.Config.from_shape(weights.shape, max_batch, max_seq)
    return mk.Megakernel(cfg, weights, 0)


def teacher_forced(weights, prompt, steps, max_seq, check_kv=True):
    """Prefill + `steps` greedy decode steps on both sides; the GPU gets the oracle's tokens."""
    ref = oracle.Decoder(weights, 1, max_seq)
    m = gpu_model(weights, max_seq)
    ref_logits = ref.prefill(prompt)[0]
    tok_dev = torch.from_numpy(prompt[None].astype(np.int32)).to(DEV)
    got = m.prefill(tok_dev)[0].cpu().numpy()
    logits_close(got, ref_logits, "prefill")
    tok = oracle.argmax(ref_logits)
    worst = (0.0, 0.0)
    for i in range(steps):
        rl = ref.decode(np.array([tok], dtype=np.int32))[0]
        gl, nt = m.decode(torch.tensor([tok], dtype=torch.int32, device=DEV))
        gl, nt = gl[0].cpu().numpy(), int(nt[0].item())
        d, r = logits_close(gl, rl, f"step {i}")
        worst = (max(worst[0], d), max(worst[1], r))
        assert argmax_agrees(gl, rl, nt), f"step {i}: argmax differs with a clear margin"
        assert nt == int(np.argmax(gl)) or gl[nt] == gl.max()
        tok = oracle.argmax(rl)
    assert m.sync_status() == mk.MK_OK
    if check_kv:
        n = len(prompt) + steps
        got_kv = m.kv_view()[:, :, :1, :, :n, :].cpu().numpy()
        kv_close(got_kv, ref.get_cache(n), "kv cache")
    return m, worst


def test_tiny_prefill_and_32_steps():
    w = mi.make_weights(mi.TINY, seed=0)
    prompt = mi.prompt(0, 0, 16, w.shape.vocab)
    teacher_forced(w, prompt, 32, 64)


def test_tiny_random_gains_and_long_prompt():
    # gains != 1 so a dropped norm gain would show; a prompt crossing several split-KV chunks
    w = mi.make_weights(mi.TINY, seed=3, sigma=0.05)
    w.final_norm = mi.normal_bf16(3, 50, (w.shape.hidden,), sigma=0.3, mean=1.0)
    for l in range(w.shape.n_layers):
        w.attn_norm[l] = mi.normal_bf16(3, 51 + 2 * l, (w.shape.hidden,), sigma=0.3, mean=1.0)
        w.mlp_norm[l] = mi.normal_bf16(3, 52 + 2 * l, (w.shape.hidden,), sigma=0.3, mean=1.0)
    prompt = mi.prompt(3, 0, 200, w.shape.vocab)
    teacher_forced(w, prompt, 8, 256)


def test_decode_is_deterministic():
    w = mi.make_weights(mi.TINY, seed=1)
    prompt = mi.prompt(1, 0, 10, w.shape.vocab)
    outs = []
    for _ in range(2):
        m = gpu_model(w, 32)
        m.prefill(torch.from_numpy(prompt[None].astype(np.int32)).to(DEV))
        seq = []
        tok = torch.tensor([5], dtype=torch.int32, device=DEV)
        for _ in range(6):
            lg, nt = m.decode(tok)
            seq.append(lg[0].cpu().numpy().copy())
            tok = nt.clone()
        outs.append(np.stack(seq))
        m.close()
    assert np.array_equal(outs[0], outs[1])


def test_synthetic_cache_decode_matches_oracle():
    # the caller fills the cache (no prefill); decode continues from position 40
    w = mi.make_weights(mi.TINY, seed=2)
    s = w.shape
    kv = mi.kv_cache_values(2, s, 1, 40, sigma=1.0)
    ref = oracle.Decoder(w, 1, 64)
    ref.set_cache(kv, 40)
    m = gpu_model(w, 64)
    m.kv_view()[:, :, :1, :, :40, :] = torch.from_numpy(kv.view(np.int16)).to(DEV)
    m.set_positions([40])
    tok = 7
    for i in range(4):
        rl = ref.decode(np.array([tok], dtype=np.int32))[0]
        gl, _ = m.decode(torch.tensor([tok], dtype=torch.int32, device=DEV))
        logits_close(gl[0].cpu().numpy(), rl, f"step {i}")
        tok = oracle.argmax(rl)


def test_dependency_wait_times_out_cleanly():
    """A notify that never comes (test hook) makes the waiting tasks give up after the limit;
    the step reports MK_ERR_DEVICE_TIMEOUT and the context works again afterwards."""
    w = mi.make_weights(mi.TINY, seed=0)
    prompt = mi.prompt(0, 0, 8, w.shape.vocab)
    m = gpu_model(w, 32)
    m.prefill(torch.from_numpy(prompt[None].astype(np.int32)).to(DEV))
    mk.mk_set_wait_timeout_ns(m.ctx, 100_000_000)  # 0.1 s
    info = m.info()
    mk.mk_debug_drop_notify(m.ctx, 3, True)  # an event in layer 0
    m.decode(torch.tensor([1], dtype=torch.int32, device=DEV))
    assert m.sync_status() == mk.MK_ERR_DEVICE_TIMEOUT
    assert "timed out" in mk.mk_last_error(m.ctx)
    mk.mk_debug_drop_notify(m.ctx, 3, False)
    # recover: re-prefill and decode normally, matching the oracle
    ref = oracle.Decoder(w, 1, 32)
    ref.prefill(prompt)
    m.prefill(torch.from_numpy(prompt[None].astype(np.int32)).to(DEV))
    rl = ref.decode(np.array([1], dtype=np.int32))[0]
    gl, _ = m.decode(torch.tensor([1], dtype=torch.int32, device=DEV))
    assert m.sync_status() == mk.MK_OK
    logits_close(gl[0].cpu().numpy(), rl, "after recovery")
    assert info["n_sms"] > 0


def test_calibrated_schedule_keeps_parity():
    # re-partitioned rows (per-SM weights measured from traced steps) must not change results
    w = mi.make_weights(mi.TINY, seed=4)
    prompt = mi.prompt(4, 0, 12, w.shape.vocab)
    ref = oracle.Decoder(w, 1, 64)
    m = gpu_model(w, 64)
    ref.prefill(prompt)
    m.prefill(torch.from_numpy(prompt[None].astype(np.int32)).to(DEV))
    tok = 3
    # calibration decodes real steps: mirror them on the oracle
    weights = m.calibrate(torch.tensor([tok], dtype=torch.int32, device=DEV), steps=1, rounds=2)
    for _ in range(2):
        ref.decode(np.array([tok], dtype=np.int32))
    assert weights.shape == (5, m.info()["n_sms"])  # one row per projection kind
    for i in range(4):
        rl = ref.decode(np.array([tok], dtype=np.int32))[0]
        gl, _ = m.decode(torch.tensor([tok], dtype=torch.int32, device=DEV))
        logits_close(gl[0].cpu().numpy(), rl, f"step {i}")
        tok = oracle.argmax(rl)
    assert m.sync_status() == mk.MK_OK
