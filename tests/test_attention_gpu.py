"""Standalone decode attention (the Mirage article's attention example) on the GPU vs the
fp64 oracle: O = softmax(scale * Q K) V, fp16 inputs, K given transposed [BH, d, L]."""
import numpy as np
import pytest
import torch

import mk_inputs as mi
import oracle
import persistent_megakernel_decode_04_b200 as mk

pytestmark = pytest.mark.gpu
MAX_ABS, REL_L2 = 1e-3, 1e-4  # fp32 accumulation against fp64


def run(BH, d, L, scale=1.0, seed=0, calls=1):
    q = mi.normal_f16(seed, 1, (BH, d))
    kt = mi.normal_f16(seed, 2, (BH, d, L))
    v = mi.normal_f16(seed, 3, (BH, L, d))
    dev = torch.device("cuda", 0)
    tq, tk, tv = (torch.from_numpy(a.view(np.int16)).to(dev) for a in (q, kt, v))
    o = torch.empty((BH, d), dtype=torch.float32, device=dev)
    ws = torch.zeros(max(mk.mk_attention_workspace_bytes(BH, d, L), 256), dtype=torch.uint8, device=dev)
    outs = []
    for _ in range(calls):
        o.fill_(float("nan"))
        mk.mk_attention_decode(tq, tk, tv, o, BH, d, L, scale, ws)
        assert mk.mk_attention_status(ws, BH, d, L) == mk.MK_OK
        outs.append(o.cpu().numpy().copy())
    ref = oracle.attention_decode_f16(q, kt, v, scale)
    return outs, ref


def check(got, ref):
    d = np.abs(got.astype(np.float64) - ref)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert np.isfinite(got).all()
    assert d.max() <= MAX_ABS and rel <= REL_L2, (d.max(), rel)


def test_mirage_example_full_size():
    # Q [64,1,128], K [64,128,4096], V [64,4096,128], no scaling
    outs, ref = run(64, 128, 4096, 1.0, calls=2)
    check(outs[0], ref)
    assert np.array_equal(outs[0], outs[1])  # deterministic, counters self-clean between calls


@pytest.mark.parametrize("BH,d,L,scale", [
    (1, 128, 64, 1.0),      # one unit, one CTA
    (3, 128, 1000, 0.125),  # ragged last unit (1000 = 15*64 + 40)
    (5, 64, 4104, 1.0),     # head_dim 64, ragged tail
    (200, 128, 128, 1.0),   # more heads than SMs
    (2, 128, 8, 1.0),       # shortest TMA-eligible length
    (4, 128, 1, 1.0),       # single key: plain path, output equals V
    (3, 64, 301, 0.5),      # L % 8 != 0: plain path
])
def test_edge_shapes(BH, d, L, scale):
    outs, ref = run(BH, d, L, scale, seed=L)
    check(outs[0], ref)


def test_single_key_returns_v():
    BH, d = 4, 128
    q = mi.normal_f16(9, 1, (BH, d))
    kt = mi.normal_f16(9, 2, (BH, d, 1))
    v = mi.normal_f16(9, 3, (BH, 1, d))
    outs, _ = run(BH, d, 1, seed=9)
    assert np.allclose(outs[0], mi.f16_to_f32(v)[:, 0, :], atol=1e-6)


def test_wait_that_runs_out_is_reported_and_the_workspace_recovers():
    """A tile the producer never loads (test hook) makes its compute warp give up after the wait
    limit: the status reports MK_ERR_DEVICE_TIMEOUT (and re-zeroes the workspace), nothing faults,
    and the next call with the same workspace is correct."""
    BH, d, L = 6, 128, 2048
    q = mi.normal_f16(4, 1, (BH, d))
    kt = mi.normal_f16(4, 2, (BH, d, L))
    v = mi.normal_f16(4, 3, (BH, L, d))
    dev = torch.device("cuda", 0)
    tq, tk, tv = (torch.from_numpy(a.view(np.int16)).to(dev) for a in (q, kt, v))
    o = torch.zeros((BH, d), dtype=torch.float32, device=dev)
    ws = torch.zeros(mk.mk_attention_workspace_bytes(BH, d, L), dtype=torch.uint8, device=dev)
    mk.mk_attention_set_wait_timeout_ns(50_000_000)
    try:
        mk.mk_attention_debug_drop_unit(70)  # head 4, keys 768..895 (units of 128 keys)
        mk.mk_attention_decode(tq, tk, tv, o, BH, d, L, 1.0, ws)
        assert mk.mk_attention_status(ws, BH, d, L) == mk.MK_ERR_DEVICE_TIMEOUT
    finally:
        mk.mk_attention_debug_drop_unit(-1)
        mk.mk_attention_set_wait_timeout_ns(2_000_000_000)
    o.fill_(float("nan"))
    mk.mk_attention_decode(tq, tk, tv, o, BH, d, L, 1.0, ws)
    assert mk.mk_attention_status(ws, BH, d, L) == mk.MK_OK
    check(o.cpu().numpy(), oracle.attention_decode_f16(q, kt, v, 1.0))
