"""The seeded input recipe (weights, ids, pre-filled cache): reproducible,
and with the distributions the workloads call for — bf16 N(0, 0.02) weights
with unit norm gains, Q8_0 codes in [-127, 127] with fp16 block scales around
0.02·√3/127 (so the weights keep σ ≈ 0.02), uniform token ids, N(0, 1) K/V."""

from __future__ import annotations

import math

import torch

from dense_token_decode_b200 import synth


def test_weights_are_reproducible_and_distinct_per_tensor():
    a = synth.model_weights(synth.TINY, 0)
    b = synth.model_weights(synth.TINY, 0)
    c = synth.model_weights(synth.TINY, 1)
    assert torch.equal(a["embed"], b["embed"])
    assert torch.equal(a["layers"][1]["wq"], b["layers"][1]["wq"])
    assert not torch.equal(a["embed"], c["embed"])
    # different tensors of one model draw different values
    assert not torch.equal(a["layers"][0]["wk"], a["layers"][1]["wk"])


def test_bf16_weights_are_n_0_002_and_gains_are_one():
    w = synth.model_weights(synth.TINY, 0)
    e = w["embed"].float()
    assert w["embed"].dtype == torch.bfloat16
    assert abs(e.mean().item()) < 1e-3
    assert abs(e.std().item() - 0.02) < 5e-4
    for name in synth.NORM_NAMES:
        assert torch.all(w["layers"][0][name] == 1)
    assert torch.all(w["final_norm"] == 1)


def test_q8_0_codes_and_scales():
    codes, scales = synth.q8_0_blocks(64, 256, seed=5)
    assert codes.dtype == torch.int8 and codes.shape == (64, 256)
    assert scales.dtype == torch.float16 and scales.shape == (64, 8)
    assert int(codes.min()) >= -127 and int(codes.max()) <= 127
    s = scales.float() / (0.02 * math.sqrt(3) / 127)
    assert float(s.min()) >= 0.5 - 1e-3 and float(s.max()) <= 1.5 + 1e-3
    w = codes.float() * scales.float().repeat_interleave(32, dim=1)
    assert abs(w.std().item() - 0.02) < 2e-3


def test_token_ids_are_uniform_in_range():
    ids = synth.token_ids(20000, 4096, seed=3)
    assert ids.dtype == torch.int32
    assert int(ids.min()) >= 0 and int(ids.max()) < 4096
    assert abs(ids.float().mean().item() - 4095 / 2) < 40
    assert torch.equal(ids, synth.token_ids(20000, 4096, seed=3))


def test_prefilled_kv_is_bf16_standard_normal():
    k, v = synth.prefilled_kv(synth.TINY, 512, seed=3, seq=1, layer=0)
    assert k.shape == (512, synth.TINY.n_kv_heads, synth.TINY.head_dim)
    assert k.dtype == v.dtype == torch.bfloat16
    assert abs(k.float().std().item() - 1) < 0.02 and abs(v.float().mean().item()) < 0.02
    k2, _ = synth.prefilled_kv(synth.TINY, 512, seed=3, seq=2, layer=0)
    assert not torch.equal(k, k2)
