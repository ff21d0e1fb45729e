"""GPU parity of both persistent decode kernels against the oracle.

A decode step of one row runs on the row-split persistent kernel by default,
steps of 2..4 rows on the cluster kernel (clusters of 16 or 8 CTAs per kv
head), and the cooperative kernel serves what neither covers;
fs_debug_decode_path selects one. Each test here runs on every kernel that
serves its batch, so no path goes unchecked while another is the default: teacher-forced decode against the oracle's logits and greedy
ids, each block alone at a decode position (per-block relative L2 <= 1e-3),
batches of 2 to 4 in one launch, random RMSNorm gains, Q8_0 weights and the
bounded-wait error path.
"""

from __future__ import annotations

import pytest
import torch

import oracle
from dense_token_decode_b200 import abi, synth
from parity_util import (BLOCK_REL_L2, GREEDY_STEPS, REPORT, assert_logits_close,
                         check_greedy_step, oracle_tensor)

from test_gpu_parity import (DEV, QWEN_SEED, Pair, _dev_i32, blocks_local_decode,  # noqa: F401
                             decode_teacher_forced)

pytestmark = pytest.mark.gpu

PATHS = {"cluster": 4, "cooperative": 1, "row-split": 3}
KIND = {"cluster": 2, "cooperative": 1, "row-split": 3}
BATCH_PATHS = ["cluster", "cooperative"]  # the row-split kernel serves batch 1


def _use(pair, path):
    pair.model.decode_path(PATHS[path])
    assert pair.model.decode_kernel(1) == KIND[path], "the decode path did not take its kernel"


@pytest.fixture(scope="module")
def tiny_pair():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return Pair(synth.TINY, 0, gains="random")


@pytest.fixture(scope="module")
def qwen_pair():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return Pair(synth.QWEN3_0P6B, QWEN_SEED, max_pos=2048)


@pytest.mark.parametrize("path", list(PATHS))
def test_tiny_decode_both_kernels(tiny_pair, path):
    """Tiny shape, random gains: 16 teacher-forced steps from a 16-token prompt
    (contexts 16..31 split over the 16 CTAs of a cluster: some ranks get no
    key), then each block alone at context 70 (two pages)."""
    _use(tiny_pair, path)
    s = tiny_pair.shape
    toks = synth.token_ids(16, s.vocab, seed=3).tolist()
    ids, _, ref_logits = oracle.generate_greedy(tiny_pair.oracle, toks, 17)
    kv = tiny_pair.model.kv(1, 64)
    tiny_pair.model.prefill(kv, 0, _dev_i32(toks))
    amb, _ = decode_teacher_forced(tiny_pair, kv, 0, ids[0], ids[1:], ref_logits[1:])
    REPORT.append((f"tiny random gains, {path} kernel: ambiguous steps", amb, 1))
    assert amb <= 1
    blocks_local_decode(tiny_pair, synth.token_ids(70, s.vocab, seed=4).tolist(), 11)
    tiny_pair.model.decode_path(0)


@pytest.mark.parametrize("path", list(PATHS))
def test_qwen_decode_both_kernels(qwen_pair, path):
    """Qwen3-0.6B shape: 8 teacher-forced steps from an 8-token prompt, and
    each block alone at contexts 1 (rank 0 alone has keys), 300 and 700
    (ranks whose key range crosses a page boundary)."""
    _use(qwen_pair, path)
    s = qwen_pair.shape
    toks = synth.token_ids(8, s.vocab, seed=1).tolist()
    ids, _, ref_logits = oracle.generate_greedy(qwen_pair.oracle, toks, 9)
    kv = qwen_pair.model.kv(1, 64)
    qwen_pair.model.prefill(kv, 0, _dev_i32(toks))
    amb, _ = decode_teacher_forced(qwen_pair, kv, 0, ids[0], ids[1:], ref_logits[1:])
    assert amb <= 1
    for n, seed in ((1, 8), (300, 9), (700, 10)):
        errs = blocks_local_decode(qwen_pair, synth.token_ids(n, s.vocab, seed=seed).tolist(), 77)
        assert max(errs) <= BLOCK_REL_L2
    qwen_pair.model.decode_path(0)


@pytest.mark.parametrize("path", BATCH_PATHS)
@pytest.mark.parametrize("B", [2, 3, 4])
def test_qwen_batches_both_kernels(qwen_pair, path, B):
    """Batches of 2..4 sequences of different lengths in one launch, rows in
    reverse sequence order; each row against the oracle."""
    _use(qwen_pair, path)
    s = qwen_pair.shape
    lens = [5, 64, 130, 17][:B]
    prompts = [synth.token_ids(n, s.vocab, seed=80 + i).tolist() for i, n in enumerate(lens)]
    kv = qwen_pair.model.kv(B, 160)
    caches = []
    for i, p in enumerate(prompts):
        qwen_pair.model.prefill(kv, i, _dev_i32(p))
        caches.append(qwen_pair.oracle.forward(p)[2])
    nxt = synth.token_ids(B, s.vocab, seed=90).tolist()
    order = list(range(B - 1, -1, -1))
    logits = torch.empty((B, s.vocab), device=DEV)
    am = torch.empty(B, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    n0 = abi.fs_debug_kernel_launches()
    qwen_pair.model.decode_step(kv, order, _dev_i32([nxt[q] for q in order]), logits, am)
    torch.cuda.synchronize()
    assert abi.fs_debug_kernel_launches() - n0 == 1
    assert qwen_pair.model.device_error() == 0
    for b, q in enumerate(order):
        rl = qwen_pair.oracle.forward([nxt[q]], caches[q])[0]
        assert_logits_close(oracle_tensor(logits[b]), rl, what=f"{path} batch {B} row {b}")
        check_greedy_step(int(am[b]), oracle_tensor(logits[b]), rl)
    kv.close()
    qwen_pair.model.decode_path(0)


@pytest.mark.parametrize("path", list(PATHS))
def test_wait_timeout_both_kernels(tiny_pair, path):
    """A 100 us wait limit with one hand-off of block 1 withheld: the step
    returns, the device error word reads 3, and the next step matches the
    oracle. The waits end by themselves; no GPU fault is involved."""
    _use(tiny_pair, path)
    m, s = tiny_pair.model, tiny_pair.shape
    toks = synth.token_ids(16, s.vocab, seed=0).tolist()
    kv = m.kv(1, 64)
    m.prefill(kv, 0, _dev_i32(toks))
    cache = tiny_pair.oracle.forward(toks)[2]
    logits = torch.empty(s.vocab, device=DEV)
    am = torch.empty(1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    assert m.device_error() == 0
    m.wait_limit(100_000, withhold_layer=1)
    m.decode_step(kv, [0], _dev_i32([5]), logits, am)
    torch.cuda.synchronize()
    assert m.device_error() == 3
    assert m.device_error() == 0
    m.wait_limit(1_000_000_000)
    kv.set_length(0, 16)
    m.decode_step(kv, [0], _dev_i32([5]), logits, am)
    torch.cuda.synchronize()
    assert m.device_error() == 0
    rl = tiny_pair.oracle.forward([5], cache)[0]
    assert_logits_close(oracle_tensor(logits), rl, what=f"{path}: step after a timeout")
    check_greedy_step(int(am.item()), oracle_tensor(logits), rl)
    m.decode_path(0)


@pytest.mark.parametrize("path", list(PATHS))
def test_q8_0_decode_both_kernels(path):
    """Q8_0 weights (codes dequantised exactly in the kernels): 8 teacher-forced
    steps on the tiny shape and each block alone at context 90."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pair = Pair(synth.TINY, 4, "q8_0")
    _use(pair, path)
    s = pair.shape
    toks = synth.token_ids(12, s.vocab, seed=12).tolist()
    ids, _, ref_logits = oracle.generate_greedy(pair.oracle, toks, 9)
    kv = pair.model.kv(1, 64)
    pair.model.prefill(kv, 0, _dev_i32(toks))
    amb, _ = decode_teacher_forced(pair, kv, 0, ids[0], ids[1:], ref_logits[1:])
    assert amb <= 1
    blocks_local_decode(pair, synth.token_ids(90, s.vocab, seed=13).tolist(), 21)
    pair.model.close()


def test_greedy_32_steps_cluster_kernel(qwen_pair):
    """fs_greedy free-running on the cluster kernel: the 32 ids of the prompt
    whose oracle top-2 gaps stay above twice the logit bound."""
    _use(qwen_pair, "cluster")
    toks = synth.token_ids(8, qwen_pair.shape.vocab, seed=6).tolist()
    ref, _, _ = oracle.generate_greedy(qwen_pair.oracle, toks, GREEDY_STEPS)
    ids, why = qwen_pair.model.greedy(qwen_pair.model.kv(1, 64), 0, toks, GREEDY_STEPS)
    assert why == abi.FS_STOP_BUDGET and ids == ref
