"""Pins for the CPU oracle: each check ties it to something other than itself
(closed forms, invariants, independent formulations, brute force, library
routines and the ``transformers`` Qwen3 implementation)."""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from conftest import oracle_weights
from dense_token_decode_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- number formats

def test_bf16_rounding_matches_torch_rne():
    x = RNG.standard_normal(20000) * 10.0 ** RNG.uniform(-6, 4, 20000)
    # exact halfway cases between neighbouring bf16 values, both parities
    base = np.array([1.0, 1.0078125, 3.0, 0.015625, -2.0, -5.0078125])
    ulp = np.array([2.0 ** -7, 2.0 ** -7, 2.0 ** -6, 2.0 ** -13, 2.0 ** -6, 2.0 ** -5])
    ties = base + np.sign(base) * ulp / 2
    x = np.concatenate([x, ties, -ties]).astype(np.float32).astype(np.float64)
    want = torch.from_numpy(x).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_to_bf16(x), want)


def test_bf16_widening_matches_torch():
    t = (torch.randn(4096, dtype=torch.float32) * 3).to(torch.bfloat16)
    bits = t.view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.bf16_bits_to_f64(bits), t.to(torch.float64).numpy())


def _fp16_exact(bits: int) -> Fraction:
    """Decode an IEEE half from its bit fields into an exact rational."""
    s, e, m = bits >> 15, (bits >> 10) & 0x1F, bits & 0x3FF
    if e == 0:
        v = Fraction(m, 1024) * Fraction(1, 2 ** 14)
    else:
        v = (1 + Fraction(m, 1024)) * (Fraction(2) ** (e - 15))
    return -v if s else v


def test_q8_0_dequant_bit_exact_against_integer_times_fp16():
    codes, scales = synth.q8_0_blocks(8, 128, seed=5)
    codes, scales = codes.numpy(), scales.numpy()
    # plant extremes: the largest code and the smallest/largest normal and a subnormal scale
    codes[0, :4] = [-127, 127, 0, -1]
    scales[0, 0] = np.float16(6.1035e-05)
    scales[1, 0] = np.float16(65504.0)
    scales[2, 0] = np.float16(5.96e-08)
    w = oracle.q8_0_dequant(codes, scales)
    sbits = scales.view(np.uint16)
    for n in range(codes.shape[0]):
        for k in range(codes.shape[1]):
            want = int(codes[n, k]) * _fp16_exact(int(sbits[n, k // 32]))
            assert Fraction(float(w[n, k])) == want
            assert float(np.float32(w[n, k])) == float(w[n, k])  # exact in fp32 too


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_constant_vector_closed_form():
    for c in (3.0, -0.25, 1e-4, 7e2):
        g = RNG.standard_normal(64)
        y = oracle.rms_norm(np.full(64, c), g, 1e-6)
        np.testing.assert_allclose(y, g * c / math.sqrt(c * c + 1e-6), rtol=1e-14)


def test_rmsnorm_matches_torch():
    x = RNG.standard_normal((5, 96)) * 3
    g = RNG.standard_normal(96)
    want = torch.nn.functional.rms_norm(torch.from_numpy(x), (96,), torch.from_numpy(g), 1e-6)
    np.testing.assert_allclose(oracle.rms_norm(x, g, 1e-6), want.numpy(), rtol=1e-13)


# ---------------------------------------------------------------- RoPE

def test_rope_preserves_norm():
    x = RNG.standard_normal((7, 3, 128))
    cos, sin = oracle.rope_cos_sin(np.arange(100, 107) * 97, 128, 1e6)
    y = oracle.apply_rope(x, cos, sin)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


def test_rope_relative_position_identity():
    d = 64
    q = RNG.standard_normal((1, 1, d))
    k = RNG.standard_normal((1, 1, d))
    for m, n in ((5, 2), (900, 13), (8191, 8000), (3, 3)):
        cm, sm = oracle.rope_cos_sin(np.array([m]), d, 1e6)
        cn, sn = oracle.rope_cos_sin(np.array([n]), d, 1e6)
        cr, sr = oracle.rope_cos_sin(np.array([m - n]), d, 1e6)
        lhs = np.sum(oracle.apply_rope(q, cm, sm) * oracle.apply_rope(k, cn, sn))
        rhs = np.sum(oracle.apply_rope(q, cr, sr) * k)
        assert abs(lhs - rhs) <= 1e-10 * (1 + abs(rhs))


def test_rope_equals_complex_rotation():
    """Pair (i, i+d/2) as the complex number x_i + j x_{i+d/2}, rotated by
    position * theta^(-2i/d)."""
    d, theta = 128, 1e6
    pos = np.array([0, 1, 17, 4099])
    x = RNG.standard_normal((4, 2, d))
    cos, sin = oracle.rope_cos_sin(pos, d, theta)
    y = oracle.apply_rope(x, cos, sin)
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    freq = np.array([theta ** (-(2 * i) / d) for i in range(d // 2)])
    zr = z * np.exp(1j * pos[:, None, None] * freq[None, None, :])
    np.testing.assert_allclose(y[..., : d // 2], zr.real, atol=1e-12)
    np.testing.assert_allclose(y[..., d // 2:], zr.imag, atol=1e-12)
    # position 0 is the identity; the first pair turns by exactly 1 radian per position
    np.testing.assert_array_equal(y[0], x[0])
    e0 = np.zeros((1, 1, d)); e0[0, 0, 0] = 1.0
    c1, s1 = oracle.rope_cos_sin(np.array([1]), d, theta)
    r = oracle.apply_rope(e0, c1, s1)
    assert r[0, 0, 0] == math.cos(1.0) and r[0, 0, d // 2] == math.sin(1.0)


# ---------------------------------------------------------------- attention

def test_softmax_rows_sum_to_one_and_masked_entries_are_zero():
    q = RNG.standard_normal((6, 32))
    k = RNG.standard_normal((10, 32)) * 4
    q_pos = np.arange(4, 10)
    p = oracle.attention_probs(q, k, q_pos, np.arange(10))
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=1e-14)
    for i, qp in enumerate(q_pos):
        assert np.all(p[i, qp + 1:] == 0.0)
        assert np.all(p[i, : qp + 1] > 0.0)


def test_gqa_equals_mha_with_repeated_kv_heads():
    S, C, nq, nkv, d = 5, 9, 8, 2, 16
    q = RNG.standard_normal((S, nq, d))
    k = RNG.standard_normal((C, nkv, d))
    v = RNG.standard_normal((C, nkv, d))
    q_pos, k_pos = np.arange(4, 9), np.arange(C)
    gqa = oracle.causal_gqa_attention(q, k, v, q_pos, k_pos)
    mha = oracle.causal_gqa_attention(q, np.repeat(k, nq // nkv, axis=1),
                                      np.repeat(v, nq // nkv, axis=1), q_pos, k_pos)
    np.testing.assert_array_equal(gqa, mha)
    # and heads 0,1,2,3 read kv head 0 (contiguous groups), not 0,2,4,6
    one = oracle.causal_gqa_attention(q[:, :4], k[:, :1], v[:, :1], q_pos, k_pos)
    np.testing.assert_array_equal(gqa[:, :4], one)


def test_attention_matches_torch_sdpa():
    S, nq, nkv, d = 12, 4, 2, 64
    q = RNG.standard_normal((S, nq, d))
    k = RNG.standard_normal((S, nkv, d))
    v = RNG.standard_normal((S, nkv, d))
    ours = oracle.causal_gqa_attention(q, k, v, np.arange(S), np.arange(S))
    t = lambda a: torch.from_numpy(a).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), is_causal=True, enable_gqa=True)[0].permute(1, 0, 2).numpy()
    np.testing.assert_allclose(ours, ref, rtol=1e-12, atol=1e-13)


def test_attention_single_key_returns_v_exactly():
    q = RNG.standard_normal((1, 4, 16))
    k = RNG.standard_normal((1, 2, 16))
    v = RNG.standard_normal((1, 2, 16))
    o = oracle.causal_gqa_attention(q, k, v, np.array([0]), np.array([0]))
    np.testing.assert_array_equal(o, np.repeat(v, 2, axis=1))


def test_attention_equal_keys_gives_mean_of_v():
    C = 7
    q = RNG.standard_normal((1, 2, 8))
    k = np.repeat(RNG.standard_normal((1, 1, 8)), C, axis=0)
    v = RNG.standard_normal((C, 1, 8))
    o = oracle.causal_gqa_attention(q, k, v, np.array([C - 1]), np.arange(C))
    np.testing.assert_allclose(o[0, 0], v[:, 0].mean(axis=0), rtol=1e-13)
    np.testing.assert_allclose(o[0, 1], v[:, 0].mean(axis=0), rtol=1e-13)


def test_silu_matches_torch():
    z = RNG.standard_normal(1000) * 6
    np.testing.assert_allclose(oracle.silu(z), torch.nn.functional.silu(torch.from_numpy(z)).numpy(),
                               rtol=1e-14, atol=1e-300)


# ---------------------------------------------------------------- greedy selection

def test_greedy_select_lowest_id_wins_tie_and_skips_nonfinite():
    l = np.array([0.5, 2.0, -1.0, 2.0, 1.0])
    assert oracle.greedy_select(l) == 1
    l = np.array([np.nan, 1.0, np.inf, 3.0, 3.0, -np.inf])
    assert oracle.greedy_select(l) == 3
    with pytest.raises(ValueError):
        oracle.greedy_select(np.array([np.nan, np.inf]))


# ---------------------------------------------------------------- whole model

def _micro_shape():
    return synth.ModelShape(n_layers=2, hidden=16, n_q_heads=4, n_kv_heads=2, head_dim=4,
                            ffn=32, vocab=50, max_pos=64)


def _oracle(shape, seed, fmt="bf16", kv_bf16=True):
    return oracle.Qwen3Oracle(shape, oracle_weights(synth.model_weights(shape, seed, fmt)), kv_bf16)


def test_parameter_count_matches_published_qwen3_0p6b():
    g = json.load(open(os.path.join(GOLDEN, "qwen3_0p6b_shape.json")))
    shape = synth.ModelShape(**{k: g[k] for k in ("n_layers", "hidden", "n_q_heads", "n_kv_heads",
                                                    "head_dim", "ffn", "vocab")})
    assert shape.n_q_heads * shape.head_dim == g["q_width"]
    n = oracle.parameter_count(shape)
    assert round(n / 1e6) == g["logical_params_millions"]
    assert n == 596_049_920


def test_causal_brute_force_future_token_does_not_leak():
    orc = _oracle(_micro_shape(), seed=3)
    toks = [3, 17, 42, 8, 0, 49, 21, 5]
    _, h0, _ = orc.forward(toks)
    for j in range(1, len(toks)):
        alt = list(toks)
        alt[j] = (alt[j] + 11) % 50
        _, h1, _ = orc.forward(alt)
        np.testing.assert_array_equal(h1[:, :j], h0[:, :j])
        assert not np.array_equal(h1[:, j], h0[:, j])


def test_cached_decode_equals_uncached_recompute():
    orc = _oracle(synth.TINY, seed=0)
    prompt = synth.token_ids(16, synth.TINY.vocab, seed=0).tolist()
    ids_c, why_c, lg_c = oracle.generate_greedy(orc, prompt, 12, cached=True)
    ids_u, why_u, lg_u = oracle.generate_greedy(orc, prompt, 12, cached=False)
    assert ids_c == ids_u and why_c == why_u == oracle.STOP_BUDGET
    for a, b in zip(lg_c, lg_u):
        np.testing.assert_allclose(a, b, rtol=1e-5, atol=1e-9)


def test_chunked_prefill_equals_one_shot():
    orc = _oracle(synth.TINY, seed=0)
    toks = synth.token_ids(20, synth.TINY.vocab, seed=9).tolist()
    l1, h1, c1 = orc.forward(toks)
    _, _, c2 = orc.forward(toks[:7])
    l2, h2, c2 = orc.forward(toks[7:], c2)
    np.testing.assert_allclose(l2, l1, rtol=1e-11, atol=1e-12)
    for l in range(synth.TINY.n_layers):
        np.testing.assert_array_equal(c1.k[l], c2.k[l])


def test_kv_cache_holds_bf16_values():
    orc = _oracle(synth.TINY, seed=0)
    _, _, cache = orc.forward([1, 2, 3])
    for l in range(synth.TINY.n_layers):
        np.testing.assert_array_equal(cache.k[l], oracle.round_to_bf16(cache.k[l]))
        np.testing.assert_array_equal(cache.v[l], oracle.round_to_bf16(cache.v[l]))


def test_generation_stop_rules():
    orc = _oracle(synth.TINY, seed=0)
    prompt = synth.token_ids(5, synth.TINY.vocab, seed=4).tolist()
    assert oracle.generate_greedy(orc, prompt, 0)[:2] == ([], oracle.STOP_BUDGET)
    with pytest.raises(ValueError):
        oracle.generate_greedy(orc, [], 3)
    first = oracle.generate_greedy(orc, prompt, 1)[0]
    ids, why, _ = oracle.generate_greedy(orc, prompt, 5, eos_ids=[first[0]])
    assert ids == first and why == oracle.STOP_EOS
    # context of 7 positions: forwards at prefix lengths 5, 6, 7 -> three ids
    ids, why, _ = oracle.generate_greedy(orc, prompt, 4, max_context=7)
    assert len(ids) == 3 and why == oracle.STOP_CONTEXT
    ids, why, _ = oracle.generate_greedy(orc, prompt, 3, max_context=7)
    assert len(ids) == 3 and why == oracle.STOP_BUDGET
    ids, why, _ = oracle.generate_greedy(orc, prompt, 3, max_context=5)
    assert len(ids) == 1 and why == oracle.STOP_CONTEXT
    with pytest.raises(ValueError):
        oracle.generate_greedy(orc, prompt, 3, max_context=4)


def test_q8_0_model_runs_on_dequantised_weights():
    shape = synth.TINY
    wq = synth.model_weights(shape, 2, "q8_0")
    orc = oracle.Qwen3Oracle(shape, oracle_weights(wq))
    codes, scales = wq["layers"][1]["wd"]
    np.testing.assert_array_equal(orc.layers[1]["wd"],
                                  codes.double().numpy() * np.repeat(scales.double().numpy(), 32, 1))
    logits, _, _ = orc.forward([1, 2, 3])
    assert np.all(np.isfinite(logits))


def _transformers_run(shape, w, toks):
    """Logits [S, V] and hidden states of the ``transformers`` Qwen3 model in
    fp64 over the same bf16 weights (gains included)."""
    transformers = pytest.importorskip("transformers")
    cfg = transformers.Qwen3Config(
        vocab_size=shape.vocab, hidden_size=shape.hidden, intermediate_size=shape.ffn,
        num_hidden_layers=shape.n_layers, num_attention_heads=shape.n_q_heads,
        num_key_value_heads=shape.n_kv_heads, head_dim=shape.head_dim,
        rms_norm_eps=shape.rms_eps, rope_theta=shape.rope_theta, tie_word_embeddings=True,
        max_position_embeddings=shape.max_pos, attention_bias=False)
    cfg._attn_implementation = "eager"
    m = transformers.Qwen3ForCausalLM(cfg).double().eval()
    names = {"wq": "self_attn.q_proj", "wk": "self_attn.k_proj", "wv": "self_attn.v_proj",
             "wo": "self_attn.o_proj", "wg": "mlp.gate_proj", "wu": "mlp.up_proj",
             "wd": "mlp.down_proj", "q_norm": "self_attn.q_norm", "k_norm": "self_attn.k_norm",
             "attn_norm": "input_layernorm", "ffn_norm": "post_attention_layernorm"}
    sd = {"model.embed_tokens.weight": w["embed"], "model.norm.weight": w["final_norm"],
          "lm_head.weight": w["embed"]}
    for l, lw in enumerate(w["layers"]):
        for k, v in lw.items():
            sd[f"model.layers.{l}.{names[k]}.weight"] = v
    m.load_state_dict({k: v.double() for k, v in sd.items()}, strict=True)
    with torch.no_grad():
        out = m(toks[None].long(), output_hidden_states=True)
    return out.logits[0].numpy(), [h[0].numpy() for h in out.hidden_states]


def _transformers_gap(orc, ref, toks):
    """Worst relative difference of the oracle against the transformers run:
    the hidden states before each block and the logits of every row."""
    ref_logits, ref_hidden = ref
    ours, hidden, _ = orc.forward(toks.tolist(), all_logits=True)
    gaps = [np.linalg.norm(hidden[l] - ref_hidden[l]) / np.linalg.norm(ref_hidden[l])
            for l in range(orc.cfg.n_layers)]
    gaps.append(np.max(np.abs(ours - ref_logits)) / np.max(np.abs(ref_logits)))
    return max(gaps), ours


@pytest.mark.parametrize("gains", ["ones", "random"])
@pytest.mark.parametrize("kv_bf16", [False, True])
def test_forward_matches_transformers_qwen3(kv_bf16, gains):
    """The whole block structure (norm forms and order, q/k-norm before RoPE,
    rotate-half pairs, GQA grouping, scale, SwiGLU, tied head) against the
    Qwen3 implementation in ``transformers`` in fp64. With ``gains="random"``
    every RMSNorm gain vector is its own draw, which pins which gain each norm
    applies (attention vs MLP norm, q vs k norm, final norm). The library's
    RoPE tables are built in fp32, which bounds the agreement near 1e-6; the
    bf16 K/V rounding of the cache bounds it near 1e-3."""
    shape = synth.TINY
    w = synth.model_weights(shape, 0, gains=gains)
    toks = synth.token_ids(16, shape.vocab, seed=0)
    ref = _transformers_run(shape, w, toks)
    orc = oracle.Qwen3Oracle(shape, oracle_weights(w), kv_bf16=kv_bf16)
    gap, ours = _transformers_gap(orc, ref, toks)
    # transformers keeps K/V unrounded; the bf16 cache rounds each stored
    # element by up to 2^-9 relative, so that mode agrees to about 2^-8
    tol = 2.0 ** -8 if kv_bf16 else 2e-6
    assert gap < tol, gap
    if not kv_bf16:
        assert [oracle.greedy_select(r) for r in ours] == ref[0].argmax(-1).tolist()


@pytest.mark.parametrize("swap", [("q_norm", "k_norm"), ("attn_norm", "ffn_norm"), "final"])
def test_transformers_pin_catches_misplaced_gains(swap):
    """The random-gain comparison above fails for an oracle that applies one
    gain in place of another: the mistake is planted in a copy of the oracle
    (CPU only) and the gap must exceed the tolerance by orders of magnitude."""
    shape = synth.TINY
    w = synth.model_weights(shape, 0, gains="random")
    toks = synth.token_ids(16, shape.vocab, seed=0)
    ref = _transformers_run(shape, w, toks)
    orc = oracle.Qwen3Oracle(shape, oracle_weights(w), kv_bf16=False)
    if swap == "final":
        orc.final_norm = orc.layers[0]["attn_norm"].copy()
    else:
        a, b = swap
        for layer in orc.layers:
            layer[a], layer[b] = layer[b], layer[a]
    gap, _ = _transformers_gap(orc, ref, toks)
    assert gap > 1e-2, gap
