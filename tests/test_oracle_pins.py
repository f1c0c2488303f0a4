"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each check comes from the mathematics, a library routine the oracle does not call
(numpy, torch, transformers' Llama), a closed form, or a worked example in
tests/golden.  They are chosen so that a dropped term, a wrong sign or index, a
transposed operand or a wrong head grouping in the oracle fails at least one.
"""
import math
import os

import numpy as np
import pytest
import torch

import mk_inputs as mi
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_splitmix64_matches_published_values():
    import ctypes
    want = [int(l, 16) for l in open(os.path.join(GOLDEN, "splitmix64_state0.txt")) if l.startswith("0x")]
    st = ctypes.c_uint64(0)
    got = [mi.lib().mki_splitmix64_next(st) for _ in want]
    assert got == want


def test_generator_is_counter_based_and_normal():
    a = mi.normal_bf16(0, 77, (3_000_001,), sigma=0.02)
    b = mi.normal_bf16(0, 77, (1000,), sigma=0.02)
    assert np.array_equal(a[:1000], b)  # prefix property: element i depends only on i
    f = mi.bf16_to_f32(a).astype(np.float64)
    assert abs(f.mean()) < 1e-4 and abs(f.std() - 0.02) < 1e-4
    t = mi.tokens(0, 5, 10000, 1000)
    assert t.min() >= 0 and t.max() < 1000 and len(np.unique(t)) > 990


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_constant_vector_closed_form():
    # RMSNorm(c * 1) = c / sqrt(c^2 + eps) * g
    for c, eps in [(3.0, 1e-6), (-0.5, 1e-5), (1e-3, 1e-5)]:
        g = np.linspace(0.5, 2.0, 64)
        y = oracle.rmsnorm(np.full(64, c), g, eps)
        assert np.allclose(y, c / math.sqrt(c * c + eps) * g, rtol=1e-14, atol=0)


def test_rmsnorm_matches_torch_and_is_scale_invariant():
    rng = np.random.default_rng(1)
    x, g = rng.normal(size=300), rng.normal(size=300)
    y = oracle.rmsnorm(x, g, 1e-5)
    ref = torch.nn.functional.rms_norm(torch.tensor(x), (300,), torch.tensor(g), eps=1e-5).numpy()
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)
    # RMSNorm(a x) = RMSNorm(x) up to the eps term: relative change <= eps / (2 mean(x^2))
    assert np.allclose(oracle.rmsnorm(1000 * x, g, 1e-5), y, rtol=1e-5 / np.mean(x * x))


# ---------------------------------------------------------------- matvec

def test_matvec_matches_numpy_on_non_square_shapes():
    w = mi.normal_bf16(3, 9, (37, 53), sigma=0.5)
    x = np.random.default_rng(2).normal(size=53)
    ref = mi.bf16_to_f32(w).astype(np.float64) @ x
    assert np.allclose(oracle.matvec_bf16(w, x), ref, rtol=1e-12, atol=1e-13)


def test_norm_then_linear_equals_linear_then_divide():
    # Mirage article, "Case 1: Normalization + Linear": RMSNorm(x) W = ((x * g) W) / rms(x).
    rng = np.random.default_rng(3)
    H, N, eps = 128, 40, 1e-5
    x, g = rng.normal(size=H), rng.normal(size=H)
    w = mi.normal_bf16(0, 11, (N, H), sigma=0.1)
    lhs = oracle.matvec_bf16(w, oracle.rmsnorm(x, g, eps))
    rms = math.sqrt(np.mean(x * x) + eps)
    rhs = oracle.matvec_bf16(w, x * g) / rms
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- RoPE

def test_rope_position_zero_is_identity():
    v = np.random.default_rng(4).normal(size=128)
    assert np.array_equal(oracle.rope(v, 0, 5e5), v)


def test_rope_two_dims_is_plane_rotation():
    # d = 2: one pair with inverse frequency theta^0 = 1, so position p rotates by p radians.
    for p in (1, 2, 7):
        out = oracle.rope(np.array([1.0, 0.0]), p, 1e4)
        assert np.allclose(out, [math.cos(p), math.sin(p)], atol=1e-15)


def test_rope_pairs_i_with_i_plus_half():
    # a one-hot at index 1 of a 8-dim head must rotate into index 1 + 4 (rotate-half pairing),
    # with the angle of pair 1: p * theta^(-2/8).
    d, p, theta = 8, 3, 100.0
    e = np.zeros(d)
    e[1] = 1.0
    out = oracle.rope(e, p, theta)
    ang = p * theta ** (-2.0 / d)
    want = np.zeros(d)
    want[1], want[5] = math.cos(ang), math.sin(ang)
    assert np.allclose(out, want, atol=1e-15)


def test_rope_preserves_pair_norms_and_is_relative():
    rng = np.random.default_rng(5)
    d = 64
    q, k = rng.normal(size=d), rng.normal(size=d)
    rq = oracle.rope(q, 11, 1e4)
    half = d // 2
    assert np.allclose(rq[:half] ** 2 + rq[half:] ** 2, q[:half] ** 2 + q[half:] ** 2, rtol=1e-12)
    # <R_m q, R_n k> depends on m - n only
    a = oracle.rope(q, 17, 1e4) @ oracle.rope(k, 5, 1e4)
    b = oracle.rope(q, 112, 1e4) @ oracle.rope(k, 100, 1e4)
    assert abs(a - b) < 1e-10


# ---------------------------------------------------------------- attention

def _golden_attention():
    rows = {}
    for line in open(os.path.join(GOLDEN, "attention_two_keys.txt")):
        if line.startswith("#") or not line.strip():
            continue
        key, *vals = line.split()
        rows.setdefault(key, []).append([float(v) for v in vals])
    return rows


def test_attention_worked_example():
    g = _golden_attention()
    o, p = oracle.attention_head(np.array(g["q"][0]), np.array(g["k"]), np.array(g["v"]), 1.0)
    assert np.allclose(p, g["probs"][0], atol=1e-15)
    assert np.allclose(o, g["o"][0], atol=1e-14)


def test_attention_single_key_returns_v_and_equal_keys_return_mean():
    rng = np.random.default_rng(6)
    q, v = rng.normal(size=16), rng.normal(size=(5, 16))
    o, p = oracle.attention_head(q, rng.normal(size=(1, 16)), v[:1], 0.25)
    assert np.allclose(o, v[0], atol=1e-15) and p[0] == 1.0
    k = np.repeat(rng.normal(size=(1, 16)), 5, axis=0)
    o, p = oracle.attention_head(q, k, v, 0.25)
    assert np.allclose(o, v.mean(axis=0), atol=1e-14)
    assert np.allclose(p, 0.2, atol=1e-15)


def test_attention_matches_torch_sdpa_and_probs_sum_to_one():
    rng = np.random.default_rng(7)
    for L, d, scale in [(1, 8, 1.0), (37, 64, 0.125), (300, 128, 1 / math.sqrt(128))]:
        q, k, v = rng.normal(size=d), rng.normal(size=(L, d)), rng.normal(size=(L, d))
        o, p = oracle.attention_head(q, k, v, scale)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.tensor(q)[None, None, None], torch.tensor(k)[None, None], torch.tensor(v)[None, None],
            scale=scale)[0, 0, 0].numpy()
        assert np.allclose(o, ref, rtol=1e-12, atol=1e-13)
        assert abs(p.sum() - 1.0) < 1e-12


def test_standalone_attention_f16_matches_torch_sdpa():
    # The Mirage example's form: fp16 inputs, K given transposed [BH, d, L], no scaling.
    BH, d, L = 3, 128, 200
    q = mi.normal_f16(0, 1, (BH, d))
    kt = mi.normal_f16(0, 2, (BH, d, L))
    v = mi.normal_f16(0, 3, (BH, L, d))
    o = oracle.attention_decode_f16(q, kt, v, 1.0)
    qt = torch.tensor(mi.f16_to_f32(q), dtype=torch.float64)
    kk = torch.tensor(mi.f16_to_f32(kt), dtype=torch.float64).transpose(1, 2)
    vv = torch.tensor(mi.f16_to_f32(v), dtype=torch.float64)
    ref = torch.nn.functional.scaled_dot_product_attention(qt[:, None], kk, vv, scale=1.0)[:, 0].numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- SiLU

def test_silu_special_values_and_torch():
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(40.0) - 40.0) < 1e-12
    assert abs(oracle.silu(-40.0)) < 1e-15
    z = np.linspace(-8, 8, 33)
    ref = torch.nn.functional.silu(torch.tensor(z)).numpy()
    assert np.allclose([oracle.silu(t) for t in z], ref, rtol=1e-14, atol=1e-15)


def test_argmax_ties_take_lowest_index():
    x = np.array([0.0, 3.0, -1.0, 3.0, 2.0], dtype=np.float32)
    assert oracle.argmax(x) == 1


# ---------------------------------------------------------------- whole decoder

def _hf_llama(w):
    """transformers' Llama (an independent implementation), float64, same weights."""
    from transformers import LlamaConfig, LlamaForCausalLM
    s = w.shape
    cfg = LlamaConfig(vocab_size=s.vocab, hidden_size=s.hidden, intermediate_size=s.ffn,
                      num_hidden_layers=s.n_layers, num_attention_heads=s.n_q_heads,
                      num_key_value_heads=s.n_kv_heads, head_dim=s.head_dim, rms_norm_eps=s.rms_eps,
                      rope_theta=s.rope_theta, max_position_embeddings=4096, tie_word_embeddings=False,
                      attention_bias=False, mlp_bias=False)
    cfg._attn_implementation = "eager"
    m = LlamaForCausalLM(cfg).to(torch.float64).eval()

    def t(a):
        return torch.tensor(mi.bf16_to_f32(a), dtype=torch.float64)

    with torch.no_grad():
        m.model.embed_tokens.weight.copy_(t(w.embed))
        m.lm_head.weight.copy_(t(w.lm_head))
        m.model.norm.weight.copy_(t(w.final_norm))
        for l, layer in enumerate(m.model.layers):
            layer.input_layernorm.weight.copy_(t(w.attn_norm[l]))
            layer.post_attention_layernorm.weight.copy_(t(w.mlp_norm[l]))
            layer.self_attn.q_proj.weight.copy_(t(w.wq[l]))
            layer.self_attn.k_proj.weight.copy_(t(w.wk[l]))
            layer.self_attn.v_proj.weight.copy_(t(w.wv[l]))
            layer.self_attn.o_proj.weight.copy_(t(w.wo[l]))
            layer.mlp.gate_proj.weight.copy_(t(w.wg[l]))
            layer.mlp.up_proj.weight.copy_(t(w.wu[l]))
            layer.mlp.down_proj.weight.copy_(t(w.wd[l]))
    return m


def _random_gains(w, seed=9):
    # gains are 1 in every config; random gains here make a dropped gain visible
    H = w.shape.hidden
    w.final_norm = mi.normal_bf16(seed, 50, (H,), sigma=0.3, mean=1.0)
    for l in range(w.shape.n_layers):
        w.attn_norm[l] = mi.normal_bf16(seed, 51 + 2 * l, (H,), sigma=0.3, mean=1.0)
        w.mlp_norm[l] = mi.normal_bf16(seed, 52 + 2 * l, (H,), sigma=0.3, mean=1.0)
    return w


@pytest.fixture(scope="module")
def tiny_weights():
    return _random_gains(mi.make_weights(mi.TINY, seed=0, sigma=0.05))


def test_decoder_matches_transformers_llama(tiny_weights):
    w = tiny_weights
    T = 12
    toks = mi.prompt(0, 0, T + 3, w.shape.vocab)
    m = _hf_llama(w)
    with torch.no_grad():
        ref = m(torch.tensor(toks[None].astype(np.int64)), use_cache=False).logits[0].numpy()
    d = oracle.Decoder(w, 1, 64, f64=True, kv_round=False)
    got = [d.prefill(toks[:T])[0]]
    for t in range(T, T + 3):
        got.append(d.decode_f64(toks[t:t + 1])[0])
    got = np.stack(got)
    want = ref[T - 1:]
    # transformers computes RoPE angles, the norm and the softmax in fp32
    assert np.max(np.abs(got - want)) < 2e-5 * np.max(np.abs(want))


def test_gqa_equals_mha_with_replicated_kv_heads(tiny_weights):
    # GQA with kv head floor(h*nkv/nq) == MHA whose K/V weight rows repeat each kv head nq/nkv times.
    w = tiny_weights
    s = w.shape
    rep = s.n_q_heads // s.n_kv_heads
    import copy
    w2 = copy.copy(w)
    w2.shape = mi.Shape("tiny-mha", s.n_layers, s.hidden, s.n_q_heads, s.n_q_heads, s.head_dim, s.ffn, s.vocab,
                        s.rms_eps, s.rope_theta)
    D = s.head_dim
    w2.wk = [np.ascontiguousarray(np.repeat(a.reshape(s.n_kv_heads, D, s.hidden), rep, axis=0).reshape(-1, s.hidden))
             for a in w.wk]
    w2.wv = [np.ascontiguousarray(np.repeat(a.reshape(s.n_kv_heads, D, s.hidden), rep, axis=0).reshape(-1, s.hidden))
             for a in w.wv]
    toks = mi.prompt(0, 1, 9, s.vocab)
    a = oracle.Decoder(w, 1, 32, f64=True, kv_round=False).prefill(toks)
    b = oracle.Decoder(w2, 1, 32, f64=True, kv_round=False).prefill(toks)
    assert np.allclose(a, b, rtol=1e-13, atol=1e-13)


def test_prefill_equals_token_by_token_decode(tiny_weights):
    w = tiny_weights
    toks = mi.prompt(0, 2, 10, w.shape.vocab)
    a = oracle.Decoder(w, 1, 32, f64=True).prefill(toks)
    d = oracle.Decoder(w, 1, 32, f64=True)
    d.prefill(toks[:1])
    for t in range(1, 10):
        b = d.decode_f64(toks[t:t + 1])
    # prefill hands back fp32 logits; the decode path keeps fp64
    assert np.allclose(a, b, rtol=1e-6, atol=1e-7)


def test_fp32_mode_tracks_fp64_mode(tiny_weights):
    w = tiny_weights
    toks = mi.prompt(0, 3, 16, w.shape.vocab)
    a = oracle.Decoder(w, 1, 64, f64=False, kv_round=False)
    b = oracle.Decoder(w, 1, 64, f64=True, kv_round=False)
    la, lb = a.prefill(toks), b.prefill(toks)
    for t in range(4):
        tok = np.array([oracle.argmax(lb[0])], dtype=np.int32)
        la, lb = a.decode(tok), b.decode_f64(tok)
        assert np.max(np.abs(la - lb)) < 1e-5 * max(1.0, np.max(np.abs(lb)))


def test_kv_cache_holds_bf16_rounded_keys_and_values(tiny_weights):
    w = tiny_weights
    toks = mi.prompt(0, 4, 8, w.shape.vocab)
    a = oracle.Decoder(w, 1, 16, f64=True, kv_round=True)
    b = oracle.Decoder(w, 1, 16, f64=True, kv_round=False)
    a.prefill(toks)
    b.prefill(toks)
    ca, cb = mi.bf16_to_f32(a.get_cache(8)), mi.bf16_to_f32(b.get_cache(8))
    # the first layer sees identical inputs, so its K/V differ only by the storage rounding
    assert np.array_equal(ca[0], cb[0])
    assert not np.all(ca == 0)


def test_batch_rows_are_independent(tiny_weights):
    w = tiny_weights
    p0, p1 = mi.prompt(0, 5, 6, w.shape.vocab), mi.prompt(0, 6, 6, w.shape.vocab)
    both = oracle.Decoder(w, 2, 16).prefill(np.stack([p0, p1]))
    one = oracle.Decoder(w, 1, 16).prefill(p1)
    assert np.array_equal(both[1], one[0])


def test_set_cache_then_decode_equals_prefill_then_decode(tiny_weights):
    w = tiny_weights
    toks = mi.prompt(0, 7, 9, w.shape.vocab)
    a = oracle.Decoder(w, 1, 16)
    a.prefill(toks[:8])
    kv = a.get_cache(8)
    want = a.decode(toks[8:9])
    b = oracle.Decoder(w, 1, 16)
    b.set_cache(kv, 8)
    assert b.position(0) == 8
    assert np.array_equal(b.decode(toks[8:9]), want)


def test_per_sequence_positions_equal_separate_decoders(tiny_weights):
    # two sequences at different positions in one batch: each row equals a one-sequence
    # decoder whose prompt ends at that position (entries past a position are ignored)
    w = tiny_weights
    pa, pb = mi.prompt(0, 9, 10, w.shape.vocab), mi.prompt(0, 10, 4, w.shape.vocab)
    ra, rb = oracle.Decoder(w, 1, 16), oracle.Decoder(w, 1, 16)
    ra.prefill(pa[:-1])
    rb.prefill(pb[:-1])
    kva, kvb = ra.get_cache(9), rb.get_cache(9)  # rb's entries 3..8 are zero padding
    both = oracle.Decoder(w, 2, 16)
    both.set_cache(np.concatenate([kva, kvb], axis=2), 9)
    both.set_positions([9, 3])
    assert (both.position(0), both.position(1)) == (9, 3)
    got = both.decode(np.array([pa[-1], pb[-1]], dtype=np.int32))
    assert np.array_equal(got[0], ra.decode(pa[-1:])[0])
    assert np.array_equal(got[1], rb.decode(pb[-1:])[0])
    with pytest.raises(ValueError):
        both.set_positions([17, 0])  # beyond max_seq


def test_thread_count_does_not_change_results(tiny_weights):
    w = mi.make_weights(mi.TINY.with_layers(1), seed=1)
    toks = mi.prompt(0, 8, 5, w.shape.vocab)
    oracle.set_threads(1)
    a = oracle.Decoder(w, 1, 8).prefill(toks)
    oracle.set_threads(7)
    b = oracle.Decoder(w, 1, 8).prefill(toks)
    oracle.set_threads(0)
    assert np.array_equal(a, b)


# ---------------------------------------------------------------- QK-norm (Chameleon)
# Mirage article, "Case 4.1: Attention with Query-Key Normalization": a LayerNorm on the
# query and key vectors before attention.

def test_layernorm_closed_form_and_torch():
    # [1, 2, 3, 4]: mean 2.5, mean squared deviation 1.25 -> (x - 2.5) / sqrt(1.25) = (2x - 5) / sqrt(5)
    x = np.array([1.0, 2.0, 3.0, 4.0])
    y = oracle.layernorm(x, np.ones(4), np.zeros(4), 0.0)
    assert np.allclose(y, (2 * x - 5) / math.sqrt(5), rtol=1e-15, atol=1e-15)
    g, b = np.array([2.0, -1.0, 0.5, 3.0]), np.array([0.25, 0.0, -1.0, 4.0])
    assert np.allclose(oracle.layernorm(x, g, b, 0.0), (2 * x - 5) / math.sqrt(5) * g + b, rtol=1e-15, atol=1e-15)
    # eps enters next to the variance: constant input -> b exactly; eps shrinks the spread
    assert np.array_equal(oracle.layernorm(np.full(8, 7.0), np.full(8, 3.0), np.arange(8.0), 1e-5), np.arange(8.0))
    assert np.allclose(oracle.layernorm(x, np.ones(4), np.zeros(4), 1.25), (x - 2.5) / math.sqrt(2.5), rtol=1e-15)
    rng = np.random.default_rng(7)
    x, g, b = rng.normal(size=128) * 3 + 1, rng.normal(size=128), rng.normal(size=128)
    ref = torch.nn.functional.layer_norm(torch.tensor(x), (128,), torch.tensor(g), torch.tensor(b), eps=1e-5).numpy()
    assert np.allclose(oracle.layernorm(x, g, b, 1e-5), ref, rtol=1e-12, atol=1e-13)


@pytest.fixture(scope="module")
def tiny_qk_weights():
    return _random_gains(mi.make_weights(mi.TINY_QK, seed=3, sigma=0.05))


def _hf_chameleon(w):
    """transformers' Chameleon text decoder (independent implementation; LayerNorm over each
    query / key head with per-head gain and bias, eps 1e-5, before RoPE), float64."""
    from transformers import ChameleonConfig, ChameleonForConditionalGeneration
    s = w.shape
    assert s.rms_eps == 1e-5  # the transformers model fixes the QK LayerNorm eps at 1e-5
    vq = dict(embed_dim=32, num_embeddings=16, double_latent=False, latent_channels=32, resolution=16,
              in_channels=3, base_channels=32, channel_multiplier=[1], num_res_blocks=1, attn_resolutions=[],
              attn_type="vanilla", dropout=0.0)  # unused image tokenizer, kept small
    cfg = ChameleonConfig(vocab_size=s.vocab, hidden_size=s.hidden, intermediate_size=s.ffn,
                          num_hidden_layers=s.n_layers, num_attention_heads=s.n_q_heads,
                          num_key_value_heads=s.n_kv_heads, rms_norm_eps=s.rms_eps, rope_theta=s.rope_theta,
                          max_position_embeddings=4096, tie_word_embeddings=False, attention_bias=False,
                          vq_config=vq, vocabulary_map={"<image>": s.vocab + 5})
    cfg._attn_implementation = "eager"
    m = ChameleonForConditionalGeneration(cfg).to(torch.float64).eval()
    assert not cfg.swin_norm

    def t(a):
        return torch.tensor(mi.bf16_to_f32(a), dtype=torch.float64)

    D = s.head_dim
    with torch.no_grad():
        m.model.embed_tokens.weight.copy_(t(w.embed))
        m.lm_head.weight.copy_(t(w.lm_head))
        m.model.norm.weight.copy_(t(w.final_norm))
        for l, layer in enumerate(m.model.layers):
            layer.input_layernorm.weight.copy_(t(w.attn_norm[l]))
            layer.post_attention_layernorm.weight.copy_(t(w.mlp_norm[l]))
            a = layer.self_attn
            a.q_proj.weight.copy_(t(w.wq[l]))
            a.k_proj.weight.copy_(t(w.wk[l]))
            a.v_proj.weight.copy_(t(w.wv[l]))
            a.o_proj.weight.copy_(t(w.wo[l]))
            a.q_norm.weight.copy_(t(w.q_norm_w[l]).reshape(s.n_q_heads, D))
            a.q_norm.bias.copy_(t(w.q_norm_b[l]).reshape(s.n_q_heads, D))
            a.k_norm.weight.copy_(t(w.k_norm_w[l]).reshape(s.n_kv_heads, D))
            a.k_norm.bias.copy_(t(w.k_norm_b[l]).reshape(s.n_kv_heads, D))
            layer.mlp.gate_proj.weight.copy_(t(w.wg[l]))
            layer.mlp.up_proj.weight.copy_(t(w.wu[l]))
            layer.mlp.down_proj.weight.copy_(t(w.wd[l]))
    return m


def test_qk_norm_decoder_matches_transformers_chameleon(tiny_qk_weights):
    w = tiny_qk_weights
    T = 11
    toks = mi.prompt(3, 0, T + 3, w.shape.vocab)
    m = _hf_chameleon(w)
    with torch.no_grad():
        ref = m(input_ids=torch.tensor(toks[None].astype(np.int64)), use_cache=False).logits[0].numpy()
    d = oracle.Decoder(w, 1, 64, f64=True, kv_round=False)
    got = [d.prefill(toks[:T])[0]]
    for t in range(T, T + 3):
        got.append(d.decode_f64(toks[t:t + 1])[0])
    got, want = np.stack(got), ref[T - 1:]
    assert np.max(np.abs(got - want)) < 2e-5 * np.max(np.abs(want))
    # and the norm matters: the same weights without QK-norm give other logits
    import copy
    w0 = copy.copy(w)
    w0.q_norm_w = []
    plain = oracle.Decoder(w0, 1, 64, f64=True, kv_round=False).prefill(toks[:T])[0]
    assert np.max(np.abs(plain - want[0])) > 1e-2 * np.max(np.abs(want[0]))


def _unrotate(v, pos, theta, D):
    # inverse RoPE of every head: rotation by -pos (RoPE pinned above as a plane rotation per pair)
    return np.concatenate([oracle.rope(h, -pos, theta) for h in v.reshape(-1, D)])


@pytest.mark.parametrize("T", [1, 6])
def test_qk_norm_heads_are_layer_normed_before_rope(tiny_qk_weights, T):
    # Every query and key head of the last token, rotated back, is g * z + b with z of mean 0
    # and mean square var/(var+eps) ~ 1: a dropped mean, a gain or bias of another head, or
    # RoPE applied before the norm all break it (T = 1: position 0, no rotation at all).
    w = tiny_qk_weights
    s = w.shape
    D = s.head_dim
    d = oracle.Decoder(w, 2, 16, f64=True)
    d.prefill(np.stack([mi.prompt(3, 1, T, s.vocab), mi.prompt(3, 2, T, s.vocab)]))
    for l in range(s.n_layers):
        q, k = d.get_qk(l)
        for vec, gw, gb in ((q, w.q_norm_w[l], w.q_norm_b[l]), (k, w.k_norm_w[l], w.k_norm_b[l])):
            g = mi.bf16_to_f32(gw).astype(np.float64)
            b = mi.bf16_to_f32(gb).astype(np.float64)
            for row in vec:
                z = ((_unrotate(row, T - 1, s.rope_theta, D) - b) / g).reshape(-1, D)
                assert np.max(np.abs(z.mean(axis=1))) < 1e-10
                assert np.max(np.abs((z * z).mean(axis=1) - 1.0)) < 1e-3
    # the cache holds the normalised, rotated keys (bf16-rounded)
    kv = d.get_cache(T)
    _, k = d.get_qk(s.n_layers - 1)
    got = mi.bf16_to_f32(kv[s.n_layers - 1, 0, :, :, T - 1, :]).reshape(2, -1)
    assert np.allclose(got, k, rtol=2 ** -8, atol=1e-6)


def test_qk_norm_absorbs_a_per_head_scale(tiny_qk_weights):
    # LayerNorm(a x) = LayerNorm(x) up to eps: scaling the W_q rows of one query head by 4 and
    # the W_k rows of one key head by 2 (exact in bf16) leaves the logits unchanged with
    # QK-norm and changes them without.
    w = tiny_qk_weights
    s = w.shape
    D = s.head_dim
    import copy

    def scaled(src):
        w2 = copy.copy(src)
        w2.wq, w2.wk = list(src.wq), list(src.wk)
        for l in range(s.n_layers):
            q = mi.bf16_to_f32(src.wq[l]).copy()
            q[D:2 * D] *= 4.0
            k = mi.bf16_to_f32(src.wk[l]).copy()
            k[:D] *= 2.0
            w2.wq[l] = (q.view(np.uint32) >> 16).astype(np.uint16)
            w2.wk[l] = (k.view(np.uint32) >> 16).astype(np.uint16)
        return w2

    toks = mi.prompt(3, 3, 9, s.vocab)
    a = oracle.Decoder(w, 1, 16, f64=True, kv_round=False).prefill(toks)[0]
    b = oracle.Decoder(scaled(w), 1, 16, f64=True, kv_round=False).prefill(toks)[0]
    assert np.max(np.abs(a - b)) < 1e-4 * np.max(np.abs(a))
    w0 = copy.copy(w)
    w0.q_norm_w = []
    a0 = oracle.Decoder(w0, 1, 16, f64=True, kv_round=False).prefill(toks)[0]
    b0 = oracle.Decoder(scaled(w0), 1, 16, f64=True, kv_round=False).prefill(toks)[0]
    assert np.max(np.abs(a0 - b0)) > 1e-2 * np.max(np.abs(a0))
