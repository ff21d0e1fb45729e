"""fs_lm_head_argmax_noalloc, the LM-head entry point for callers that may not
allocate device memory (for instance a latency-bound host thread where
cudaMalloc could stall on a device-wide sync, or a process whose memory is all
held by another framework's pool). Its scratch is a fixed array inside the
library, so the check here is that two calls in a row through the C ABI give
what the model's own LM-head entry point gives, and that a call too big for
the array is refused up front. This file is collected last on purpose."""

import ctypes as C

import numpy as np
import pytest
import torch

from dense_token_decode_b200 import abi, synth
from dense_token_decode_b200.engine import Model
from parity_util import LOGIT_ABS

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _call(model, x, logits, am):
    s = model.shape
    return abi.fs_lm_head_argmax_noalloc(model.embed.data_ptr(), model.final_norm.data_ptr(),
                                         s.hidden, s.vocab, C.c_float(s.rms_eps), x.data_ptr(),
                                         x.shape[0], logits.data_ptr() if logits is not None else None,
                                         am.data_ptr() if am is not None else None,
                                         torch.cuda.current_stream().cuda_stream)


def test_no_alloc_lm_head_matches_model_entry_point():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # Qwen3-0.6B hidden size and vocabulary, one block (the LM head only uses the embedding).
    shape = synth.ModelShape(n_layers=1, hidden=1024, n_q_heads=16, n_kv_heads=8, head_dim=128,
                             ffn=3072, vocab=151936, max_pos=128)
    m = Model(shape, synth.model_weights(shape, 5), DEV)
    g = torch.Generator(device="cpu").manual_seed(11)
    for rows in (3, 16):  # two calls in a row; the second reuses the array the first wrote
        x = torch.randn((rows, shape.hidden), generator=g).to(DEV)
        ref_l = torch.empty((rows, shape.vocab), device=DEV)
        ref_a = torch.empty(rows, dtype=torch.int32, device=DEV)
        m.lm_head(x, ref_l, ref_a)
        got_l = torch.full((rows, shape.vocab), float("nan"), device=DEV)
        got_a = torch.full((rows,), -1, dtype=torch.int32, device=DEV)
        abi.check(_call(m, x, got_l, got_a), "fs_lm_head_argmax_noalloc")
        torch.cuda.synchronize()
        assert float((got_l - ref_l).abs().max()) <= LOGIT_ABS
        assert got_a.tolist() == ref_a.tolist()
    # 64 rows of hidden 1024 need more than the fixed array: refused, nothing runs
    x = torch.zeros((64, shape.hidden), device=DEV)
    am = torch.empty(64, dtype=torch.int32, device=DEV)
    assert _call(m, x, None, am) == abi.FS_ERR_INVALID
    assert b"512 KiB" in abi.fs_last_error_string()
    m.close()
