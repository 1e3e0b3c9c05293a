"""Pins of the fp64 oracle against things other than itself.

Each test fixes one step of the round against a hand-worked value, a closed
form, an invariant, brute force on a tiny case, or an independent library
routine (NumPy / torch fp64, and the HF ``transformers`` Gemma4 modules that
the drafter page says its RMSNorm, RoPE and scaled embedding were checked
against). No test here needs a GPU or the CUDA library.
"""
import math

import numpy as np
import pytest
import torch

from oracle import dspark as O
from synthetic import ModelShape, make_weights, quantize_affine4, small_model

RNG = np.random.default_rng(1234)


def tiny_model(**kw):
    base = dict(hidden_size=32, num_hidden_layers=1, num_attention_heads=4, global_head_dim=16,
                num_global_key_value_heads=2, intermediate_size=48, vocab_size=64, block_size=3,
                mask_token_id=63, markov_rank=4, rope_theta=10000.0, partial_rotary_factor=0.5,
                final_logit_softcapping=None, dtype="fp32")
    base.update(kw)
    return ModelShape(**base)


def f64w(m, seed=0, **kw):
    return O.OracleWeights(make_weights(m, seed, **kw), m)


# --------------------------------------------------------------------------- RoPE

def test_rope_wavelengths_hand_values():
    wl = O.rope_wavelengths(64, 10000.0, 0.25)        # rotated = 16 -> 8 finite entries
    assert np.isfinite(wl[:8]).all() and np.isinf(wl[8:]).all()
    assert wl[0] == 1.0
    assert wl[1] == pytest.approx(10000.0 ** (2 / 64), rel=1e-15)
    assert wl[7] == pytest.approx(10000.0 ** (14 / 64), rel=1e-15)
    # odd rotated count: k < rotated/2 keeps k = floor(rotated/2) too
    wl = O.rope_wavelengths(8, 100.0, 5 / 8)          # rotated = 5 -> k in {0, 1, 2}
    assert np.isfinite(wl[:3]).all() and np.isinf(wl[3:]).all()


def test_rope_wavelengths_vs_hf_proportional():
    from transformers.modeling_rope_utils import _compute_proportional_rope_parameters
    from transformers.models.gemma4.configuration_gemma4 import Gemma4TextConfig
    for hd, theta, partial in [(64, 10000.0, 0.25), (256, 1e6, 1.0), (256, 1e6, 0.25), (128, 1e6, 0.5)]:
        cfg = Gemma4TextConfig(vocab_size=64, hidden_size=32, intermediate_size=48, num_hidden_layers=1,
                               num_attention_heads=4, num_key_value_heads=4, head_dim=8, global_head_dim=hd,
                               num_global_key_value_heads=1, attention_k_eq_v=True,
                               layer_types=["full_attention"], hidden_size_per_layer_input=0,
                               rope_parameters={"full_attention": {"rope_type": "proportional",
                                                                   "rope_theta": theta,
                                                                   "partial_rotary_factor": partial}})
        inv, _ = _compute_proportional_rope_parameters(cfg, layer_type="full_attention",
                                                      head_dim_key="global_head_dim")
        ours = 1.0 / O.rope_wavelengths(hd, theta, partial)         # 1/inf = 0
        np.testing.assert_allclose(ours, inv.double().numpy(), rtol=2e-7, atol=0)


def _rope_brute(x, pos, wl):
    """Per-lane scalar loop: pair (i, i + hd/2) rotated by pos / wl[i]."""
    hd = x.shape[-1]
    out = np.array(x, dtype=np.float64)
    for t in range(x.shape[0]):
        for i in range(hd // 2):
            a = pos[t] / wl[i] if np.isfinite(wl[i]) else 0.0
            c, s = math.cos(a), math.sin(a)
            u, v = x[t, i], x[t, i + hd // 2]
            out[t, i] = u * c - v * s
            out[t, i + hd // 2] = v * c + u * s
    return out


def test_rope_hand_worked_example():
    # hd = 4, theta 100, full rotation -> wavelengths [1, 10]; pos 1, x = e0.
    wl = O.rope_wavelengths(4, 100.0, 1.0)
    np.testing.assert_allclose(wl, [1.0, 10.0], rtol=1e-15)
    y = O.apply_rope(np.array([[1.0, 0.0, 0.0, 0.0]]), np.array([1.0]), wl)
    np.testing.assert_allclose(y, [[math.cos(1.0), 0.0, math.sin(1.0), 0.0]], atol=1e-15)
    y = O.apply_rope(np.array([[0.0, 1.0, 0.0, 0.0]]), np.array([5.0]), wl)
    np.testing.assert_allclose(y, [[0.0, math.cos(0.5), 0.0, math.sin(0.5)]], atol=1e-15)


def test_rope_vs_brute_force_and_invariants():
    hd = 16
    wl = O.rope_wavelengths(hd, 1e4, 0.5)              # lanes 0..3 and 8..11 rotate
    x = RNG.standard_normal((7, hd))
    pos = np.array([0, 1, 2, 17, 1000, 40000, 123457], dtype=np.float64)
    y = O.apply_rope(x, pos, wl)
    np.testing.assert_allclose(y, _rope_brute(x, pos, wl), rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(y[0], x[0])                      # p = 0: identity
    np.testing.assert_array_equal(y[:, 4:8], x[:, 4:8])            # inf wavelengths: identity
    np.testing.assert_array_equal(y[:, 12:16], x[:, 12:16])
    half = hd // 2
    np.testing.assert_allclose(y[:, :half] ** 2 + y[:, half:] ** 2,
                               x[:, :half] ** 2 + x[:, half:] ** 2, rtol=1e-12)


def test_rope_relative_position_identity():
    hd = 32
    wl = O.rope_wavelengths(hd, 1e4, 1.0)
    q, k = RNG.standard_normal(hd), RNG.standard_normal(hd)
    for p, pp, d in [(3, 11, 5), (100, 7, 1000), (0, 0, 12345)]:
        lhs = O.apply_rope(q[None], np.array([p + d]), wl)[0] @ O.apply_rope(k[None], np.array([pp + d]), wl)[0]
        rhs = O.apply_rope(q[None], np.array([p]), wl)[0] @ O.apply_rope(k[None], np.array([pp]), wl)[0]
        assert lhs == pytest.approx(rhs, rel=1e-9, abs=1e-9)


def test_rope_vs_hf_apply_rotary():
    from transformers.models.gemma4 import modeling_gemma4 as mg
    hd = 16
    wl = O.rope_wavelengths(hd, 1e4, 0.5)
    x = RNG.standard_normal((5, hd))
    pos = np.arange(5, dtype=np.float64) * 3
    inv = 1.0 / wl
    freqs = pos[:, None] * inv[None, :]
    emb = np.concatenate([freqs, freqs], axis=-1)
    cos, sin = torch.from_numpy(np.cos(emb)), torch.from_numpy(np.sin(emb))
    hf = mg.apply_rotary_pos_emb(torch.from_numpy(x)[None], cos, sin, unsqueeze_dim=0)[0].numpy()
    np.testing.assert_allclose(O.apply_rope(x, pos, wl), hf, rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------- RMSNorm, gelu

def test_rms_norm_closed_form_and_hf():
    from transformers.models.gemma4 import modeling_gemma4 as mg
    x = RNG.standard_normal((6, 40)) * np.array([[1e-4], [1e-2], [1.0], [3.0], [100.0], [0.0]])
    eps = 1e-6
    y = O.rms_norm(x, None, eps)
    ms = np.mean(x * x, axis=-1)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), ms / (ms + eps), rtol=1e-12, atol=1e-300)
    w = 1 + 0.02 * RNG.standard_normal(40)
    hf = mg.Gemma4RMSNorm(40, eps=eps).double()
    with torch.no_grad():
        hf.weight.copy_(torch.from_numpy(w))
        ref = hf(torch.from_numpy(x)).numpy()
        ref0 = mg.Gemma4RMSNorm(40, eps=eps, with_scale=False).double()(torch.from_numpy(x)).numpy()
    # Gemma4RMSNorm casts its input to fp32 before normalising
    np.testing.assert_allclose(O.rms_norm(x, w, eps), ref, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(y, ref0, rtol=1e-6, atol=1e-7)
    tw = torch.nn.functional.rms_norm(torch.from_numpy(x), (40,), torch.from_numpy(w), eps).numpy()
    np.testing.assert_allclose(O.rms_norm(x, w, eps), tw, rtol=1e-12, atol=1e-14)


def test_gelu_tanh_vs_torch():
    x = np.linspace(-8, 8, 1001)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    np.testing.assert_allclose(O.gelu_tanh(x), ref, rtol=1e-13, atol=1e-15)
    from transformers.activations import ACT2FN
    np.testing.assert_allclose(O.gelu_tanh(x), ACT2FN["gelu_pytorch_tanh"](torch.from_numpy(x)).numpy(),
                               rtol=1e-13, atol=1e-15)


# --------------------------------------------------------------------------- attention

def _attn_case(L=9, G=3, nH=4, nKv=2, hd=8):
    q = RNG.standard_normal((G, nH, hd))
    kc, vc = RNG.standard_normal((L, nKv, hd)), RNG.standard_normal((L, nKv, hd))
    kb, vb = RNG.standard_normal((G, nKv, hd)), RNG.standard_normal((G, nKv, hd))
    return q, kc, vc, kb, vb


def _torch_sdpa(q, k, v):
    """torch fp64 SDPA, scale 1, no mask, GQA expanded by head // group."""
    nH, nKv = q.shape[1], k.shape[1]
    grp = nH // nKv
    Q = torch.from_numpy(q).permute(1, 0, 2)[None]
    K = torch.from_numpy(np.repeat(k, grp, axis=1)).permute(1, 0, 2)[None]
    V = torch.from_numpy(np.repeat(v, grp, axis=1)).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=1.0, is_causal=False)
    return o[0].permute(1, 0, 2).numpy()


def test_attention_rows_sum_to_one():
    q, kc, vc, kb, vb = _attn_case()
    P = O.attention_weights(q, kc, kb)
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=1e-14)
    assert (P >= 0).all()


def test_attention_vs_torch_sdpa_concat():
    q, kc, vc, kb, vb = _attn_case(L=13)
    ref = _torch_sdpa(q, np.concatenate([kc, kb]), np.concatenate([vc, vb]))
    np.testing.assert_allclose(O.attend_concat(q, kc, vc, kb, vb), ref, rtol=1e-12, atol=1e-13)


def test_attention_empty_context_is_block_self_attention():
    q, kc, vc, kb, vb = _attn_case(L=0)
    ref = _torch_sdpa(q, kb, vb)
    np.testing.assert_allclose(O.attend_concat(q, kc, vc, kb, vb), ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(O.attend_split(q, kc, vc, kb, vb), ref, rtol=1e-12, atol=1e-13)


def test_attention_split_equals_concat():
    for L, splits in [(1, 1), (9, 3), (50, 7), (128, 4)]:
        q, kc, vc, kb, vb = _attn_case(L=L)
        q = q * 4.0    # larger logits: exercises the max-shift of the merge
        np.testing.assert_allclose(O.attend_split(q, kc, vc, kb, vb, splits), O.attend_concat(q, kc, vc, kb, vb),
                                   rtol=1e-12, atol=1e-13)


def test_attention_special_cases():
    q, kc, vc, kb, vb = _attn_case(L=6, G=1)
    # a single key (no context, block of one) returns its value for every head of the group
    out = O.attend_concat(q, kc[:0], vc[:0], kb, vb)
    np.testing.assert_allclose(out[0, 0], vb[0, 0], rtol=1e-15)
    np.testing.assert_allclose(out[0, 3], vb[0, 1], rtol=1e-15)    # head 3 -> kv head 1 (group 2)
    # q = 0: uniform weights -> mean of all values of the head's kv head
    out = O.attend_concat(np.zeros_like(q), kc, vc, kb, vb)
    allv = np.concatenate([vc, vb])
    np.testing.assert_allclose(out[0, 1], allv[:, 0].mean(0), rtol=1e-13)
    np.testing.assert_allclose(out[0, 2], allv[:, 1].mean(0), rtol=1e-13)


# --------------------------------------------------------------------------- context K/V

def test_context_kv_identities_and_append_equals_recompute():
    m = tiny_model(num_hidden_layers=2)
    W = f64w(m)
    hidden = torch.randn(2, 11, m.hidden_size, generator=torch.Generator().manual_seed(3))
    pos0 = [5, 100]
    full = O.project_context_kv(W, hidden, pos0)
    wl = O.rope_wavelengths(m.global_head_dim, m.rope_theta, m.partial_rotary_factor)
    for b in range(2):
        for li in range(2):
            k, v = full[b][li]
            # k_eq_v: K = rope(V * k_norm) at pos0 + t, exactly
            kn = W.vector(f"layers.{li}.k_norm")
            pos = pos0[b] + np.arange(11)
            kk = O.apply_rope((v * kn).transpose(1, 0, 2), pos[None, :], wl).transpose(1, 0, 2)
            np.testing.assert_allclose(k, kk, rtol=1e-13, atol=1e-14)
            # v is the scale-less norm of k_proj's output (unit mean square up to eps)
            ms = np.mean(v * v, axis=-1)
            assert np.all(np.abs(ms - 1) < 1e-3)
    # appends: rows [0,4) then [4,9) then [9,11), each at its own first position
    pieces = [(0, 4), (4, 9), (9, 11)]
    for b in range(2):
        got = [O.project_context_kv(W, hidden[b:b + 1, lo:hi], [pos0[b] + lo]) for lo, hi in pieces]
        for li in range(2):
            k = np.concatenate([g[0][li][0] for g in got])
            v = np.concatenate([g[0][li][1] for g in got])
            np.testing.assert_allclose(k, full[b][li][0], rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(v, full[b][li][1], rtol=1e-13, atol=1e-14)


# --------------------------------------------------------------------------- the decoder layer vs HF

def _hf_layer(m, W, li):
    from transformers.models.gemma4 import modeling_gemma4 as mg
    from transformers.models.gemma4.configuration_gemma4 import Gemma4TextConfig
    cfg = Gemma4TextConfig(
        vocab_size=m.vocab_size, hidden_size=m.hidden_size, intermediate_size=m.intermediate_size,
        num_hidden_layers=1, num_attention_heads=m.num_attention_heads, num_key_value_heads=m.num_attention_heads,
        head_dim=8, global_head_dim=m.global_head_dim, num_global_key_value_heads=m.num_global_key_value_heads,
        attention_k_eq_v=True, layer_types=["full_attention"], use_bidirectional_attention="all",
        rope_parameters={"full_attention": {"rope_type": "proportional", "rope_theta": m.rope_theta,
                                            "partial_rotary_factor": m.partial_rotary_factor}},
        hidden_size_per_layer_input=0, rms_norm_eps=m.rms_norm_eps)
    cfg._attn_implementation = "eager"
    layer = mg.Gemma4TextDecoderLayer(cfg, 0).double().eval()
    p = f"layers.{li}."
    t = lambda n: torch.from_numpy(W.matrix(p + n) if W.t[p + n].dim() == 2 else W.vector(p + n))
    with torch.no_grad():
        a = layer.self_attn
        a.q_proj.weight.copy_(t("q_proj")); a.k_proj.weight.copy_(t("k_proj")); a.o_proj.weight.copy_(t("o_proj"))
        a.q_norm.weight.copy_(t("q_norm")); a.k_norm.weight.copy_(t("k_norm"))
        layer.mlp.gate_proj.weight.copy_(t("gate_proj")); layer.mlp.up_proj.weight.copy_(t("up_proj"))
        layer.mlp.down_proj.weight.copy_(t("down_proj"))
        layer.input_layernorm.weight.copy_(t("input_layernorm"))
        layer.post_attention_layernorm.weight.copy_(t("post_attention_layernorm"))
        layer.pre_feedforward_layernorm.weight.copy_(t("pre_feedforward_layernorm"))
        layer.post_feedforward_layernorm.weight.copy_(t("post_feedforward_layernorm"))
        layer.layer_scalar.copy_(t("layer_scalar"))
    return cfg, layer, mg.Gemma4TextRotaryEmbedding(cfg)


@pytest.mark.parametrize("partial,scalar", [(0.5, 1.0), (1.0, 0.75), (0.25, 1.3)])
def test_decoder_layer_vs_hf_gemma4(partial, scalar):
    """One oracle layer over [context ++ block] equals HF's Gemma4 decoder layer fed the
    same context through its K/V cache (k_eq_v, full attention, bidirectional, scale 1)."""
    from transformers.cache_utils import DynamicCache
    m = tiny_model(partial_rotary_factor=partial, block_size=4)
    tens = make_weights(m, 7)
    tens["layers.0.layer_scalar"] = torch.tensor([scalar])
    W = O.OracleWeights(tens, m)
    cfg, layer, rot = _hf_layer(m, W, 0)
    L, pos0 = 6, 9
    ctx = torch.randn(1, L, m.hidden_size, generator=torch.Generator().manual_seed(5), dtype=torch.float64)
    h = torch.randn(1, m.block_size, m.hidden_size, generator=torch.Generator().manual_seed(6), dtype=torch.float64)
    cache = DynamicCache(config=cfg)
    with torch.no_grad():
        cs = rot(ctx, torch.arange(pos0, pos0 + L)[None], layer_type="full_attention")
        layer.self_attn(ctx, cs, None, past_key_values=cache)           # fills the cache with context K/V
        bs = rot(h, torch.arange(pos0 + L, pos0 + L + m.block_size)[None], layer_type="full_attention")
        ref = layer(h, position_embeddings=bs, attention_mask=None, past_key_values=cache).numpy()
    kv = O.project_context_kv(W, ctx, [pos0])
    ours, _ = O.decoder_layer(W, 0, h.numpy(), [kv[0][0]], [pos0 + L])
    # HF computes rotary angles and the softmax in fp32 internally
    np.testing.assert_allclose(ours, ref, rtol=2e-5, atol=2e-5)


def test_layer_scalar_scales_whole_output():
    """Zero o_proj and down_proj: the attention and MLP branches vanish (rms of 0 is 0),
    so the layer is h -> h * layer_scalar (the scalar includes the residual)."""
    m = tiny_model()
    tens = make_weights(m, 1)
    tens["layers.0.o_proj"].zero_()
    tens["layers.0.down_proj"].zero_()
    tens["layers.0.layer_scalar"] = torch.tensor([0.37])
    W = O.OracleWeights(tens, m)
    h = RNG.standard_normal((1, m.block_size, m.hidden_size))
    kv = O.project_context_kv(W, torch.randn(1, 5, m.hidden_size), [0])
    out, _ = O.decoder_layer(W, 0, h, [kv[0][0]], [5])
    np.testing.assert_allclose(out, h * float(np.float32(0.37)), rtol=1e-14)


def test_scaled_embedding_vs_hf():
    from transformers.models.gemma4 import modeling_gemma4 as mg
    m = tiny_model()
    W = f64w(m)
    anchors = [5, 17]
    emb = mg.Gemma4TextScaledWordEmbedding(m.vocab_size, m.hidden_size, 0, embed_scale=m.hidden_size ** 0.5).double()
    with torch.no_grad():
        emb.weight.copy_(torch.from_numpy(W.matrix("embed_tokens")))
        ref = emb(torch.from_numpy(O.block_ids(anchors, m.block_size, m.mask_token_id))).numpy()
    # the HF module keeps its sqrt(hidden) scale as an fp32 buffer
    np.testing.assert_allclose(O.embed_block(W, anchors), ref, rtol=1e-7)
    assert (O.block_ids(anchors, 3, 63) == np.array([[5, 63, 63], [17, 63, 63]])).all()


# --------------------------------------------------------------------------- logits, walk, confidence

def test_softcap_bounds_and_monotone_argmax():
    m = tiny_model(final_logit_softcapping=2.0, markov_rank=0)
    W = f64w(m)
    h = RNG.standard_normal((2, m.block_size, m.hidden_size)) * 30
    U = O.compute_logits(W, h)
    raw = W.linear(h, "lm_head")
    assert np.abs(U).max() < 2.0
    assert (np.argmax(U, -1) == np.argmax(raw, -1)).all()
    np.testing.assert_allclose(U, 2.0 * np.tanh(raw / 2.0), rtol=1e-14)


def test_walk_without_transition_is_stepwise_argmax():
    m = tiny_model()
    tens = make_weights(m, 2)
    tens["markov_w2"].zero_()
    W = O.OracleWeights(tens, m)
    U = RNG.standard_normal((3, m.block_size, m.vocab_size))
    np.testing.assert_array_equal(O.markov_walk(W, U, [1, 2, 3]), np.argmax(U, -1))
    m0 = tiny_model(markov_rank=0)
    W0 = f64w(m0)
    np.testing.assert_array_equal(O.markov_walk(W0, U, [1, 2, 3]), np.argmax(U, -1))


def test_walk_chain_brute_force():
    """U = 0: each step is argmax_v sum_j w1[prev, j] * W2[v, j], computed here by explicit loops."""
    m = tiny_model(vocab_size=24, mask_token_id=23, markov_rank=3, block_size=5)
    W = f64w(m, seed=4, markov_scale=50.0)
    w1, w2 = W.matrix("markov_w1"), W.matrix("markov_w2")
    U = np.zeros((1, m.block_size, m.vocab_size))
    got = O.markov_walk(W, U, [7])[0]
    prev, want = 7, []
    for _ in range(m.block_size):
        best, arg = -math.inf, -1
        for v in range(m.vocab_size):
            s = 0.0
            for j in range(m.markov_rank):
                s += w1[prev, j] * w2[v, j]
            if s > best:
                best, arg = s, v
        want.append(arg)
        prev = arg
    assert list(got) == want


def test_walk_ties_take_lowest_index_and_teacher_forcing():
    m = tiny_model(markov_rank=0, vocab_size=8, mask_token_id=7, block_size=2)
    W = f64w(m)
    U = np.zeros((1, 2, 8))
    U[0, 0, [3, 5]] = 1.0
    U[0, 1, [6, 2]] = 2.0
    toks, margins = O.teacher_forced_walk(W, U, [0], None)
    assert toks.tolist() == [[3, 2]] and margins.tolist() == [[0.0, 0.0]]


def test_teacher_forced_walk_uses_given_prev():
    m = tiny_model(vocab_size=16, mask_token_id=15, markov_rank=2, block_size=3)
    W = f64w(m, seed=9, markov_scale=40.0)
    U = RNG.standard_normal((1, 3, 16)) * 0.01
    forced = np.array([[4, 9, 1]])
    toks, _ = O.teacher_forced_walk(W, U, [2], forced)
    for k, prev in enumerate([2, 4, 9]):
        assert toks[0, k] == int(np.argmax(U[0, k] + O.markov_bias(W, [prev])[0]))


def test_confidence_zero_projection_and_threshold_rule():
    m = tiny_model()
    tens = make_weights(m, 3)
    tens["confidence_proj"].zero_()
    tens["confidence_bias"] = torch.tensor([0.4])
    W = O.OracleWeights(tens, m)
    h = RNG.standard_normal((2, m.block_size, m.hidden_size))
    c = O.confidence(W, h, [1, 2], np.zeros((2, m.block_size), dtype=np.int64))
    np.testing.assert_allclose(c, 1 / (1 + math.exp(-float(np.float32(0.4)))), rtol=1e-15)
    assert O.prefix_length([0.1, 0.2], 0.0, 2) == 2
    assert O.prefix_length([0.1, 0.9], 0.5, 2) == 0            # empty proposal
    assert O.prefix_length([0.9, 0.6, 0.4, 0.9], 0.5, 4) == 2
    assert O.prefix_length([0.9, 0.6], 0.5, 2) == 2


def test_confidence_feature_order_is_hidden_then_markov():
    m = tiny_model()
    tens = make_weights(m, 3)
    H, r = m.hidden_size, m.markov_rank
    tens["confidence_proj"].zero_()
    tens["confidence_proj"][0, H + 1] = 1.0                   # picks w1[prev][1]
    tens["confidence_bias"] = torch.tensor([0.0])
    W = O.OracleWeights(tens, m)
    h = np.zeros((1, m.block_size, H))
    toks = np.array([[10, 11, 12]])
    c = O.confidence(W, h, [9], toks)
    w1 = W.matrix("markov_w1")
    np.testing.assert_allclose(np.log(c / (1 - c))[0], [w1[9, 1], w1[10, 1], w1[11, 1]], rtol=1e-12)


# --------------------------------------------------------------------------- quantization

def test_dequantize_hand_packed_word():
    words = torch.tensor([[int("0x76543210", 16), int("0xFEDCBA98", 16) - 2 ** 32]], dtype=torch.int32)
    scales = torch.tensor([[0.5]], dtype=torch.bfloat16)
    biases = torch.tensor([[-1.0]], dtype=torch.bfloat16)
    w = O.dequantize_affine4(words, scales, biases, 16)
    np.testing.assert_array_equal(w[0], 0.5 * np.arange(16) - 1.0)


def test_quantize_dequantize_round_trip_within_half_step():
    w = torch.randn(8, 128, generator=torch.Generator().manual_seed(0)) * 0.02
    q, s, b = quantize_affine4(w, 64)
    d = O.dequantize_affine4(q, s, b, 64)
    step = np.repeat(s.double().numpy(), 64, axis=1)
    err = np.abs(d - w.double().numpy())
    # half a step, plus the bf16 rounding of the group's bias and range
    assert np.all(err <= 0.5 * step + 2 ** -8 * (np.abs(w.double().numpy()) + step * 16) + 1e-7)


def test_quantized_oracle_weights_match_dense_dequant():
    m = small_model(quant_bits=4, hidden_size=128, intermediate_size=128, vocab_size=256, mask_token_id=255,
                    num_hidden_layers=1, num_attention_heads=2, global_head_dim=64, num_global_key_value_heads=1,
                    markov_rank=64)
    tens = make_weights(m, 0)
    W = O.OracleWeights(tens, m)
    assert W.is_quantized("lm_head") and W.is_quantized("embed_tokens") and not W.is_quantized("markov_w1")
    x = RNG.standard_normal((3, 128))
    dense = O.dequantize_affine4(tens["lm_head.q"], tens["lm_head.scales"], tens["lm_head.biases"], 64)
    np.testing.assert_allclose(W.linear(x, "lm_head", chunk=100), x @ dense.T, rtol=1e-13)
    np.testing.assert_allclose(W.gather("embed_tokens", np.array([3, 200]))[1],
                               O.dequantize_affine4(tens["embed_tokens.q"][200:201], tens["embed_tokens.scales"][200:201],
                                                    tens["embed_tokens.biases"][200:201], 64)[0])


# --------------------------------------------------------------------------- whole round

def test_full_round_shapes_and_consistency():
    m = tiny_model(num_hidden_layers=2, final_logit_softcapping=5.0, confidence_threshold=0.5)
    W = f64w(m, seed=11, markov_scale=20.0)
    hid = torch.randn(2, 7, m.hidden_size, generator=torch.Generator().manual_seed(2))
    kv = O.project_context_kv(W, hid, [0, 3], lengths=[7, 4])
    out = O.draft_rows(W, kv, [1, 2], [7, 7], keep_attention=True)
    A, G = 2, m.block_size
    assert out["tokens"].shape == (A, G) and out["conf"].shape == (A, G) and out["base_logits"].shape == (A, G, 64)
    toks2, _ = O.teacher_forced_walk(W, out["base_logits"], [1, 2], out["tokens"])
    np.testing.assert_array_equal(toks2, out["tokens"])           # self-consistent when fed its own tokens
    for b in range(A):
        assert out["lengths"][b] == O.prefix_length(out["conf"][b], 0.5, G)
    assert len(out["attention"]) == 2


def test_store_rounded_is_round_to_nearest_even_bf16():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -3.14159, 1e-3, 0.0])
    got = O.store_rounded(x, "bf16")
    # bf16 keeps 8 significant bits: 1 + 2^-8 is a tie -> even (1.0); 1 + 3*2^-9 rounds up to 1 + 2^-7
    assert got[0] == 1.0 and got[1] == 1.0 and got[2] == 1.0 + 2 ** -7
    assert abs(got[3] + 3.140625) < 1e-12
    np.testing.assert_array_equal(O.store_rounded(x, None), x)


def test_store_rounded_is_round_to_nearest_even_fp16():
    """fp16 keeps 11 significant bits: hand-worked ties and the subnormal spacing 2^-24."""
    x = np.array([1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11, 2049.0, 2051.0, -3.14159, 2 ** -24 * 1.5, 70000.0])
    got = O.store_rounded(x, "fp16")
    assert got[0] == 1.0                          # a tie -> even
    assert got[1] == 1.0 + 2 ** -9                # 1 + 3 * 2^-11 -> up to 1 + 4 * 2^-11
    assert got[2] == 2048.0 and got[3] == 2052.0  # spacing 2 above 2048: ties to even
    assert got[4] == -3.140625                    # -3.14159 -> nearest multiple of 2^-9
    assert got[5] == 2 ** -23                     # subnormals: a multiple of 2^-24, tie -> even
    assert np.isinf(got[6])                       # past 65504


# --------------------------------------------------------------------------- context feature projection

def _ctx_case(taps=3, H=24, rows=5, seed=0):
    g = np.random.default_rng(seed)
    x = g.standard_normal((rows, taps * H))
    fc = g.standard_normal((H, taps * H)) * 0.1
    w = 1.0 + 0.05 * g.standard_normal(H)
    return x, fc, w


def test_context_projection_identity_fc_is_rms_norm():
    """taps = 1 and fc = I: the projection reduces to Gemma4RMSNorm of the tap (torch's rms_norm)."""
    x, _, w = _ctx_case(taps=1)
    H = x.shape[-1]
    got = O.project_context(np.eye(H), w, x, 1e-6)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (H,), torch.from_numpy(w), 1e-6).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_context_projection_vs_torch_linear_then_rms_norm():
    """A non-symmetric fc: x @ fc^T (torch's linear, [out, in] storage) then the norm; a transposed
    operand would fail here."""
    x, fc, w = _ctx_case(taps=1, H=16, seed=3)
    fc = fc + np.triu(np.ones_like(fc))               # clearly not symmetric
    t = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(fc))
    ref = torch.nn.functional.rms_norm(t, (16,), torch.from_numpy(w), 1e-6).numpy()
    np.testing.assert_allclose(O.project_context(fc, w, x, 1e-6), ref, rtol=1e-12, atol=1e-12)


def test_context_projection_tap_order_and_zero_tap():
    """Permuting the taps together with fc's column blocks changes nothing; a tap of zeros
    drops out (the projection over the remaining taps alone)."""
    x, fc, w = _ctx_case(taps=3, H=24, seed=5)
    H = 24
    blocks = lambda a: [a[..., i * H:(i + 1) * H] for i in range(3)]
    xb, fb = blocks(x), blocks(fc)
    perm = [2, 0, 1]
    xp = np.concatenate([xb[i] for i in perm], -1)
    fp = np.concatenate([fb[i] for i in perm], -1)
    base = O.project_context(fc, w, x, 1e-6)
    np.testing.assert_allclose(O.project_context(fp, w, xp, 1e-6), base, rtol=1e-12, atol=1e-12)
    xz = np.concatenate([xb[0], np.zeros_like(xb[1]), xb[2]], -1)
    two = O.project_context(np.concatenate([fb[0], fb[2]], -1), w, np.concatenate([xb[0], xb[2]], -1), 1e-6)
    np.testing.assert_allclose(O.project_context(fc, w, xz, 1e-6), two, rtol=1e-12, atol=1e-12)


def test_context_projection_scale_invariance_and_unit_rms():
    """Scaling fc by c scales each output row by sqrt((ms + eps) / (ms + eps / c^2)) exactly (ms:
    the projection's mean square; RMSNorm removes the scale but for eps), and with unit gain each
    output row has RMS sqrt(ms / (ms + eps))."""
    x, fc, w = _ctx_case(taps=2, H=20, seed=7)
    eps, c = 1e-3, 7.5                                   # an eps large enough to show its term
    base = O.project_context(fc, w, x, eps)
    ms = np.mean((x @ fc.T) ** 2, axis=-1)
    factor = np.sqrt((ms + eps) / (ms + eps / c ** 2))[:, None]
    np.testing.assert_allclose(O.project_context(c * fc, w, x, eps), base * factor, rtol=1e-12, atol=1e-14)
    out = O.project_context(fc, np.ones(20), x, 1e-6)
    np.testing.assert_allclose(np.sqrt(np.mean(out ** 2, axis=-1)), np.sqrt(ms / (ms + 1e-6)), rtol=1e-12)


# --------------------------------------------------------------------------- Alg 1 draft-length pruning

def test_prune_lengths_hand_worked_and_special_cases():
    """Hand-worked rows, then the rule's closed forms: position 0 survives even below its
    threshold; a value equal to the threshold is not below it; zero thresholds never prune
    (confidences are >= 0); thresholds above 1 prune at position 1; gamma = 1 keeps 1."""
    conf = np.array([[0.10, 0.90, 0.20, 0.95],     # 0 below, kept; first k >= 1 below: 2
                     [0.90, 0.80, 0.70, 0.60],     # nothing below 0.5: gamma
                     [0.90, 0.49, 0.99, 0.10],     # 1
                     [0.90, 0.50, 0.50, 0.50]])    # equal is not below: gamma
    np.testing.assert_array_equal(O.prune_lengths(conf, [0.5] * 4), [2, 4, 1, 4])
    # per-position thresholds: row 0 stops at 2 (0.20 < 0.3); rows 1-3 at 3 (0.60, 0.10, 0.50 < 0.65)
    np.testing.assert_array_equal(O.prune_lengths(conf, [0.0, 0.3, 0.3, 0.65]), [2, 3, 3, 3])
    g = np.random.default_rng(5).random((7, 6))
    np.testing.assert_array_equal(O.prune_lengths(g, [0.0] * 6), [6] * 7)
    np.testing.assert_array_equal(O.prune_lengths(g, [2.0] * 6), [1] * 7)
    np.testing.assert_array_equal(O.prune_lengths(g[:, :1], [2.0]), [1] * 7)
    nan = np.array([[0.9, np.nan, 0.1]])
    np.testing.assert_array_equal(O.prune_lengths(nan, [0.5] * 3), [2])
