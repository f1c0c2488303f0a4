"""mk_attention_decode_noalloc: the decode-attention entry point for callers that may not
allocate device memory (for example a serving process whose allocator reserved the GPU's
memory up front, or a latency-critical loop where cudaMalloc would block and synchronise the
device).  Its scratch is a fixed 4 MiB array inside libmk.so instead of a caller workspace.

Checked against the workspace entry point mk_attention_decode on the same inputs, on two
calls in a row (the fixed array keeps the previous call's contents between calls), on both
kernels (split-KV with TMA tiles when L % 8 == 0, the plain-load kernel otherwise), for the size
limit, and for the status of a call whose device wait ran out.  The file name makes pytest
collect it last: a run that stops at the first failure (-x) has then run every other test
before anything here can stop it."""
import numpy as np
import pytest
import torch

import mk_inputs as mi
import persistent_megakernel_decode_04_b200 as mk

pytestmark = pytest.mark.gpu
MAX_ABS, REL_L2 = 1e-3, 1e-4  # the tolerance of the attention parity tests
DEV = torch.device("cuda", 0)


def inputs(BH, d, L, seed):
    q = mi.normal_f16(seed, 1, (BH, d))
    kt = mi.normal_f16(seed, 2, (BH, d, L))
    v = mi.normal_f16(seed, 3, (BH, L, d))
    return tuple(torch.from_numpy(a.view(np.int16)).to(DEV) for a in (q, kt, v))


@pytest.mark.parametrize("BH,d,L,scale", [(64, 128, 4096, 1.0), (5, 64, 1000, 0.125), (3, 64, 1001, 0.125)])
def test_noalloc_matches_the_workspace_entry_point_on_two_calls(BH, d, L, scale):
    ws = torch.zeros(mk.mk_attention_workspace_bytes(BH, d, L), dtype=torch.uint8, device=DEV)
    for call in range(2):
        q, kt, v = inputs(BH, d, L, seed=call)
        want = torch.empty((BH, d), dtype=torch.float32, device=DEV)
        got = torch.full((BH, d), float("nan"), dtype=torch.float32, device=DEV)
        mk.mk_attention_decode(q, kt, v, want, BH, d, L, scale, ws)
        mk.mk_attention_decode_noalloc(q, kt, v, got, BH, d, L, scale)
        assert mk.mk_attention_noalloc_status() == mk.MK_OK
        g, w = got.cpu().numpy().astype(np.float64), want.cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all(), f"call {call}: non-finite output"
        d_abs = np.abs(g - w).max()
        rel = np.linalg.norm(g - w) / np.linalg.norm(w)
        assert d_abs <= MAX_ABS and rel <= REL_L2, f"call {call}: {d_abs:.3e} {rel:.3e}"


def test_noalloc_rejects_sizes_beyond_its_fixed_array():
    # 8192 heads of 8 keys need about 4.3 MB of partials: more than the 4 MiB array.  The
    # inputs are real so that nothing could be read out of bounds even if the check failed.
    BH, d, L = 8192, 128, 8
    assert mk.mk_attention_workspace_bytes(BH, d, L) > 4 << 20
    q, kt, v = inputs(BH, d, L, seed=7)
    o = torch.zeros((BH, d), dtype=torch.float32, device=DEV)
    with pytest.raises(mk.MkError) as e:
        mk.mk_attention_decode_noalloc(q, kt, v, o, BH, d, L, 1.0)
    assert e.value.code == mk.MK_ERR_INVALID_ARG
    assert "fixed array" in str(e.value)


def test_noalloc_status_reports_a_wait_that_ran_out():
    """A tile that is never loaded (test hook) makes the compute warp waiting for it give up
    after the wait limit; the status call reports it once, and the next call is clean."""
    BH, d, L = 8, 128, 1024
    q, kt, v = inputs(BH, d, L, seed=3)
    o = torch.zeros((BH, d), dtype=torch.float32, device=DEV)
    assert mk.mk_attention_noalloc_status() == mk.MK_OK  # nothing pending from earlier calls
    mk.mk_attention_set_wait_timeout_ns(50_000_000)
    try:
        mk.mk_attention_debug_drop_unit(5)
        mk.mk_attention_decode_noalloc(q, kt, v, o, BH, d, L, 1.0)
        assert mk.mk_attention_noalloc_status() == mk.MK_ERR_DEVICE_TIMEOUT
        assert "timed out" in mk.mk_last_error()
    finally:
        mk.mk_attention_debug_drop_unit(-1)
        mk.mk_attention_set_wait_timeout_ns(2_000_000_000)
    assert mk.mk_attention_noalloc_status() == mk.MK_OK  # reported once, then cleared
    ws = torch.zeros(mk.mk_attention_workspace_bytes(BH, d, L), dtype=torch.uint8, device=DEV)
    want = torch.empty((BH, d), dtype=torch.float32, device=DEV)
    mk.mk_attention_decode(q, kt, v, want, BH, d, L, 1.0, ws)
    mk.mk_attention_decode_noalloc(q, kt, v, o, BH, d, L, 1.0)
    assert mk.mk_attention_noalloc_status() == mk.MK_OK
    g, w = o.cpu().numpy().astype(np.float64), want.cpu().numpy().astype(np.float64)
    assert np.abs(g - w).max() <= MAX_ABS and np.linalg.norm(g - w) / np.linalg.norm(w) <= REL_L2
