"""Seeded synthetic inputs for the Qwen3-class forward pass.

This module holds random draws and nothing else: no step of the forward pass
(no norm, projection, rotation, attention or dequantisation) is computed here.
The CUDA path's harness and the tests both take their inputs from it, so the
two sides see the same bytes.

Recipes (all draws on a CPU ``torch.Generator`` unless ``device`` says
otherwise; every tensor has its own sub-seed so any one tensor can be
regenerated alone):

* linear weights and the (tied) embedding: fp32 N(0, 0.02) draws rounded to
  bf16 with round-to-nearest-even (torch's ``.to(torch.bfloat16)``);
* RMSNorm gains: exactly 1.0 (bf16) for the benchmark configurations; with
  ``gains="random"`` every gain vector (each layer's attn/ffn/q/k norm and the
  final norm) is its own fp32 N(1, 0.3) draw rounded to bf16, so a kernel that
  reads one gain in place of another gives a different result;
* Q8_0 linear weights: blocks of 32 consecutive weights along the input
  (dot-product) axis; int8 codes uniform in [-127, 127]; one fp16 scale per
  block, ``0.02 * sqrt(3) / 127 * u`` with ``u ~ U[0.5, 1.5]`` (weight standard
  deviation close to 0.02). Stored struct-of-arrays: codes ``[N, K]`` int8,
  scales ``[N, K/32]`` fp16;
* token ids: uniform integers in ``[0, V)``;
* pre-filled KV cache: N(0, 1) rounded to bf16, logical layout
  ``[layer][k|v][position][kv_head][head_dim]`` per sequence.
"""

from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class ModelShape:
    """Shape of a dense Qwen3-class decoder with a tied LM head."""

    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rms_eps: float = 1e-6
    rope_theta: float = 1e6
    max_pos: int = 40960

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim


# "Coming back to Failed Star", shape legend under "Second sitting": S, V=151936,
# H=1024, L=28, 16 query heads, 8 KV heads, d=128, I=3072.
QWEN3_0P6B = ModelShape(n_layers=28, hidden=1024, n_q_heads=16, n_kv_heads=8,
                        head_dim=128, ffn=3072, vocab=151936)

# The small seeded model used for exhaustive parity: 2 layers, hidden 256,
# 4 q heads / 2 kv heads, head_dim 64, ffn 768, vocab 4096.
TINY = ModelShape(n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2,
                  head_dim=64, ffn=768, vocab=4096, max_pos=4096)

LINEAR_NAMES = ("wq", "wk", "wv", "wo", "wg", "wu", "wd")
NORM_NAMES = ("attn_norm", "ffn_norm", "q_norm", "k_norm")


def linear_shape(shape: ModelShape, name: str) -> tuple[int, int]:
    """[out, in] of one linear weight (row-major, input axis contiguous)."""
    H, I = shape.hidden, shape.ffn
    return {
        "wq": (shape.q_dim, H), "wk": (shape.kv_dim, H), "wv": (shape.kv_dim, H),
        "wo": (H, shape.q_dim), "wg": (I, H), "wu": (I, H), "wd": (H, I),
    }[name]


def norm_len(shape: ModelShape, name: str) -> int:
    return shape.head_dim if name in ("q_norm", "k_norm") else shape.hidden


def _sub_seed(seed: int, *keys: int) -> int:
    s = seed & 0xFFFFFFFF
    for k in keys:
        s = (s * 1000003 + k + 1) & 0x7FFFFFFFFFFF
    return s


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_bf16(rows: int, cols: int, std: float, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    t = torch.randn((rows, cols), generator=g, dtype=torch.float32, device=device)
    return (t * std).to(torch.bfloat16)


def q8_0_blocks(rows: int, cols: int, seed: int) -> tuple[torch.Tensor, torch.Tensor]:
    """int8 codes [rows, cols] uniform in [-127, 127] and fp16 scales [rows, cols/32]."""
    if cols % 32:
        raise ValueError("Q8_0 needs the input dimension to be a multiple of 32")
    g = _gen(seed)
    codes = torch.randint(-127, 128, (rows, cols), generator=g, dtype=torch.int16).to(torch.int8)
    u = torch.rand((rows, cols // 32), generator=g, dtype=torch.float64) + 0.5
    scales = (0.02 * math.sqrt(3.0) / 127.0 * u).to(torch.float16)
    return codes, scales


def _gain(n: int, gains: str, seed: int) -> torch.Tensor:
    if gains == "ones":
        return torch.ones(n, dtype=torch.bfloat16)
    g = _gen(seed)
    return (1.0 + 0.3 * torch.randn(n, generator=g, dtype=torch.float32)).to(torch.bfloat16)


def model_weights(shape: ModelShape, seed: int, weight_format: str = "bf16",
                  layers: range | None = None, gains: str = "ones") -> dict:
    """Random-init weights as CPU tensors.

    Returns ``{"embed": bf16 [V,H], "final_norm": bf16 [H], "layers": [...]}``
    where each layer maps the linear names to a bf16 ``[N,K]`` tensor (or, for
    ``weight_format="q8_0"``, to a ``(codes, scales)`` pair) and the norm names
    to bf16 gains. ``layers`` restricts which layers are drawn (the others are
    ``None``); the draws of a layer do not depend on which others are drawn.
    ``gains`` is ``"ones"`` (every RMSNorm gain 1.0) or ``"random"`` (each gain
    vector an independent N(1, 0.3) draw); the linear weights do not depend on it.
    """
    if weight_format not in ("bf16", "q8_0"):
        raise ValueError(weight_format)
    if gains not in ("ones", "random"):
        raise ValueError(gains)
    out = {
        "embed": normal_bf16(shape.vocab, shape.hidden, 0.02, _sub_seed(seed, 0)),
        "final_norm": _gain(shape.hidden, gains, _sub_seed(seed, 4999)),
        "layers": [],
    }
    want = set(range(shape.n_layers) if layers is None else layers)
    for l in range(shape.n_layers):
        if l not in want:
            out["layers"].append(None)
            continue
        lw = {}
        for j, name in enumerate(LINEAR_NAMES):
            n, k = linear_shape(shape, name)
            s = _sub_seed(seed, 1 + l, j)
            if weight_format == "bf16":
                lw[name] = normal_bf16(n, k, 0.02, s)
            else:
                lw[name] = q8_0_blocks(n, k, s)
        for j, name in enumerate(NORM_NAMES):
            lw[name] = _gain(norm_len(shape, name), gains, _sub_seed(seed, 5000 + l, j))
        out["layers"].append(lw)
    return out


def token_ids(n: int, vocab: int, seed: int) -> torch.Tensor:
    g = _gen(_sub_seed(seed, 7777))
    return torch.randint(0, vocab, (n,), generator=g, dtype=torch.int64).to(torch.int32)


def prefilled_kv(shape: ModelShape, n_tokens: int, seed: int, seq: int, layer: int,
                 device="cpu") -> tuple[torch.Tensor, torch.Tensor]:
    """N(0,1) bf16 K and V for one (sequence, layer): each ``[n_tokens, n_kv_heads, head_dim]``.

    On a CUDA ``device`` the draws come from torch's CUDA generator (a different
    stream from the CPU one, but equally seeded and reproducible); callers that
    need the values on the host copy the generated tensor back.
    """
    g = _gen(_sub_seed(seed, 9001, seq, layer), device)
    kv = torch.randn((2, n_tokens, shape.n_kv_heads, shape.head_dim), generator=g,
                     dtype=torch.float32, device=device).to(torch.bfloat16)
    return kv[0], kv[1]
