"""CPU oracle — TEST INFRASTRUCTURE ONLY.

A plain fp64 numpy restatement of the dense Qwen3-class forward pass, used to
check the CUDA library. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arm may import it; the library
(``dense_token_decode_b200``) never does, and this package imports nothing
from the library.
"""

from .qwen3 import (  # noqa: F401
    KVCache,
    Qwen3Oracle,
    STOP_BUDGET,
    STOP_CONTEXT,
    STOP_EOS,
    apply_rope,
    attention_probs,
    bf16_bits_to_f64,
    causal_gqa_attention,
    expected_shapes,
    generate_greedy,
    greedy_select,
    parameter_count,
    q8_0_dequant,
    rms_norm,
    rope_cos_sin,
    round_to_bf16,
    silu,
)
from .sampling import (  # noqa: F401
    filtered_distribution,
    philox4x32_10,
    ranking,
    sample,
    uniform,
)
