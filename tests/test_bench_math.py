"""The algorithmic work bench.py divides by, checked against independent
counts: the parameter count of the oracle's shape table and the FLOPs of the
plain definition (2 per multiply-add; causal attention over S(S+1)/2 visible
query-key pairs)."""

from __future__ import annotations

import bench
import oracle
from dense_token_decode_b200 import synth


def test_decode_bytes_are_every_weight_once_plus_kv():
    s = synth.QWEN3_0P6B
    per_step, weights = bench.decode_bytes(s, [1, 100])
    # bf16: 2 bytes per parameter; the tied head is the embedding (counted once)
    assert weights == 2 * oracle.parameter_count(s) == 1_192_099_840
    kv_tok = s.n_layers * 2 * s.n_kv_heads * s.head_dim * 2
    assert kv_tok == 114_688
    assert per_step[0] == weights + kv_tok * 1 + kv_tok
    assert per_step[1] - per_step[0] == 99 * kv_tok


def test_prefill_flops_2048():
    s, S = synth.QWEN3_0P6B, 2048
    lin = 2 * S * s.n_layers * (s.hidden * (s.n_q_heads + 2 * s.n_kv_heads) * s.head_dim
                                + s.n_q_heads * s.head_dim * s.hidden + 3 * s.hidden * s.ffn)
    attn = s.n_layers * s.n_q_heads * 4 * s.head_dim * S * (S + 1) // 2
    head = 2 * s.hidden * s.vocab
    assert bench.prefill_flops(s, S) == lin + attn + head == 2_285_468_647_424


def test_q8_0_decode_bytes():
    s = synth.QWEN3_0P6B
    _, weights = bench.decode_bytes(s, [1], q8=True)
    n_lin = s.n_layers * 15_728_640
    # 32 int8 codes + one fp16 scale per 32 weights; the tied embedding stays bf16
    assert weights == n_lin * 34 // 32 + s.vocab * s.hidden * 2 + (s.n_layers * 2304 + s.hidden) * 2
    assert weights == 779_223_040
