"""GPU parity: the CUDA path, called through the C ABI, against the fp64
oracle on the same seeded inputs.

Bars (written in parity_util): per-block hidden-state relative L2 <= 1e-3,
max |delta logit| <= 2e-2, greedy ids identical for 32 steps (a step whose
oracle top-2 gap is below twice the measured logit error is "ambiguous": it
passes if the GPU picked either candidate, and both sides continue on the
oracle's id), Q8_0 dequantisation bit-exact.
"""

from __future__ import annotations

import ctypes as C

import numpy as np
import pytest
import torch

import oracle
from conftest import oracle_weights
from dense_token_decode_b200 import abi, synth
from dense_token_decode_b200.engine import Model
from parity_util import (BLOCK_REL_L2, E2E_BLOCK_REL_L2, GREEDY_STEPS, LOGIT_ABS, REPORT,
                         assert_blocks_close, assert_logits_close, check_greedy_step,
                         oracle_tensor, rel_l2, to_dev)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
QWEN_SEED = 1     # decode / prefill / batched-decode configs share these bf16 weights
Q8_SEED = 4


# --------------------------------------------------------------------------- fixtures

class Pair:
    """A GPU model and the oracle over the same weights."""

    def __init__(self, shape, seed, fmt="bf16", max_pos=None, gains="ones"):
        self.shape = shape
        w = synth.model_weights(shape, seed, fmt, gains=gains)
        self.model = Model(shape, w, DEV, max_pos=max_pos)
        self._w = w
        self._oracle = None

    @property
    def oracle(self):
        if self._oracle is None:
            self._oracle = oracle.Qwen3Oracle(self.shape, oracle_weights(self._w))
        return self._oracle


@pytest.fixture(scope="module")
def tiny():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return Pair(synth.TINY, 0)


@pytest.fixture(scope="module")
def tiny_gains():
    """The tiny model with every RMSNorm gain vector drawn on its own."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return Pair(synth.TINY, 0, gains="random")


@pytest.fixture(scope="module")
def qwen():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return Pair(synth.QWEN3_0P6B, QWEN_SEED, max_pos=8192 + 256)


def _dev_i32(xs):
    return torch.tensor(list(xs), dtype=torch.int32, device=DEV)


def prefill_with_capture(pair, kv, seq, toks):
    m, s = pair.model, pair.shape
    n = len(toks)
    hidden = torch.zeros((s.n_layers + 1, n, s.hidden), dtype=torch.float32, device=DEV)
    logits = torch.empty(s.vocab, dtype=torch.float32, device=DEV)
    am = torch.empty(1, dtype=torch.int32, device=DEV)
    m.capture(hidden, n)
    m.prefill(kv, seq, _dev_i32(toks), logits, am)
    torch.cuda.synchronize()
    return oracle_tensor(logits), oracle_tensor(hidden), int(am.item())


def blocks_local_prefill(pair, toks, oracle_run=None):
    """Each block alone on the oracle's input (a prefill of len(toks) rows at
    positions 0..): its output and the K/V it stores, against the oracle."""
    s = pair.shape
    rl, rh, cache = oracle_run if oracle_run is not None else pair.oracle.forward(toks)
    kv = pair.model.kv(1, len(toks))
    errs, kv_errs = [], []
    for l in range(s.n_layers):
        out = pair.model.block(kv, 0, l, to_dev(rh[l]))
        torch.cuda.synchronize()
        errs.append(rel_l2(oracle_tensor(out), rh[l + 1]))
        k, v = kv.export(0, l, 0, len(toks))
        kv_errs.append(max(rel_l2(oracle_tensor(k), cache.k[l]),
                           rel_l2(oracle_tensor(v), cache.v[l])))
    REPORT.append((f"{s.n_layers}-block {len(toks)}-row block-local rel-L2", max(errs),
                   BLOCK_REL_L2))
    assert max(errs) <= BLOCK_REL_L2, f"block-local rel-L2 {max(errs):.3e}: {errs}"
    assert max(kv_errs) <= BLOCK_REL_L2, f"block-local KV rel-L2 {max(kv_errs):.3e}: {kv_errs}"
    return errs


def blocks_local_decode(pair, toks, next_tok):
    """Each block alone at one decode position: the GPU cache holds the
    oracle's K/V of the earlier positions and the block gets the oracle's input."""
    s = pair.shape
    _, _, cache = pair.oracle.forward(toks)
    ref = oracle.KVCache(k=list(cache.k), v=list(cache.v))
    _, rh, _ = pair.oracle.forward([next_tok], ref)
    P = len(toks)
    kv = pair.model.kv(1, P + 8)
    for l in range(s.n_layers):
        kv.import_(0, l, 0, to_dev(cache.k[l], dtype=torch.bfloat16),
                   to_dev(cache.v[l], dtype=torch.bfloat16))
    kv.set_length(0, P)
    errs = []
    for l in range(s.n_layers):
        out = pair.model.block(kv, 0, l, to_dev(rh[l]))
        torch.cuda.synchronize()
        errs.append(rel_l2(oracle_tensor(out), rh[l + 1]))
    REPORT.append((f"{s.n_layers}-block decode block-local rel-L2 (context {P})", max(errs),
                   BLOCK_REL_L2))
    assert max(errs) <= BLOCK_REL_L2, f"decode block-local rel-L2 {max(errs):.3e}: {errs}"
    return errs


def decode_teacher_forced(pair, kv, seq, first_tok, ref_ids, ref_logits, capture_steps=()):
    """GPU decode fed the oracle's ids; checks every step. Returns ambiguous count."""
    m, s = pair.model, pair.shape
    logits = torch.empty(s.vocab, dtype=torch.float32, device=DEV)
    am = torch.empty(1, dtype=torch.int32, device=DEV)
    ambiguous = 0
    inputs = [first_tok] + list(ref_ids[:-1])
    hiddens = {}
    for i, tok in enumerate(inputs):
        hid = None
        if i in capture_steps:
            hid = torch.zeros((s.n_layers + 1, 1, s.hidden), dtype=torch.float32, device=DEV)
            m.capture(hid, 1)
        m.decode_step(kv, [seq], _dev_i32([tok]), logits, am)
        torch.cuda.synchronize()
        gl = oracle_tensor(logits)
        assert_logits_close(gl, ref_logits[i], what=f"decode step {i}")
        if not check_greedy_step(int(am.item()), gl, ref_logits[i]):
            ambiguous += 1
        if hid is not None:
            hiddens[i] = oracle_tensor(hid)
    return ambiguous, hiddens


# --------------------------------------------------------------------------- tiny config

def test_tiny_prefill_logits_blocks_and_cache(tiny):
    toks = synth.token_ids(16, tiny.shape.vocab, seed=0).tolist()
    kv = tiny.model.kv(2, 64)
    gl, gh, am = prefill_with_capture(tiny, kv, 0, toks)
    rl, rh, cache = tiny.oracle.forward(toks)
    assert_blocks_close(gh, rh, tol=E2E_BLOCK_REL_L2, what="tiny prefill end to end")
    assert_logits_close(gl, rl, what="tiny prefill")
    blocks_local_prefill(tiny, toks, (rl, rh, cache))
    assert am == oracle.greedy_select(rl) or abs(rl[am] - rl.max()) < 2 * np.abs(gl - rl).max()
    for l in range(tiny.shape.n_layers):
        k, v = kv.export(0, l, 0, 16)
        assert rel_l2(oracle_tensor(k), cache.k[l]) <= BLOCK_REL_L2
        assert rel_l2(oracle_tensor(v), cache.v[l]) <= BLOCK_REL_L2
    assert kv.length(0) == 16


def test_tiny_decode_teacher_forced(tiny):
    toks = synth.token_ids(16, tiny.shape.vocab, seed=0).tolist()
    ids, why, ref_logits = oracle.generate_greedy(tiny.oracle, toks, 17)
    kv = tiny.model.kv(1, 64)
    gl, _, am = prefill_with_capture(tiny, kv, 0, toks)
    check_greedy_step(am, gl, ref_logits[0])
    amb, hid = decode_teacher_forced(tiny, kv, 0, ids[0], ids[1:], ref_logits[1:],
                                     capture_steps=(0, 15))
    # per-block hidden states at two decode steps, against a cached oracle run
    cache = tiny.oracle.forward(toks)[2]
    prefix_ids = [ids[0]] + ids[1:16]
    for i, tok in enumerate(prefix_ids):
        _, rh, cache = tiny.oracle.forward([tok], cache)
        if i in hid:
            assert_blocks_close(hid[i], rh, tol=E2E_BLOCK_REL_L2, what=f"tiny decode step {i}")
    assert amb <= 4
    blocks_local_decode(tiny, toks + ids[:10], ids[10])


def _min_top2_gap(ref_logits):
    return min(float(np.sort(l)[-1] - np.sort(l)[-2]) for l in ref_logits)


def test_tiny_fs_greedy_matches_oracle(tiny):
    """Free-running fs_greedy, 16 ids identical to the oracle's. The prompt
    (seed 7) is one whose oracle top-2 logit gaps all stay above twice the
    logit bound, so no step is ambiguous and every id must match."""
    toks = synth.token_ids(16, tiny.shape.vocab, seed=7).tolist()
    ref, why, ref_logits = oracle.generate_greedy(tiny.oracle, toks, 16)
    assert _min_top2_gap(ref_logits) >= 2 * LOGIT_ABS
    kv = tiny.model.kv(1, 64)
    ids, reason = tiny.model.greedy(kv, 0, toks, 16)
    assert reason == abi.FS_STOP_BUDGET and ids == ref
    assert kv.length(0) == 16 + 15


def test_tiny_stop_rules(tiny):
    m = tiny.model
    prompt = synth.token_ids(5, tiny.shape.vocab, seed=4).tolist()
    kv = m.kv(1, 64)
    assert m.greedy(kv, 0, prompt, 0) == ([], abi.FS_STOP_BUDGET)
    assert kv.length(0) == 0
    first, _ = m.greedy(kv, 0, prompt, 1)
    kv.reset(0)
    ids, why = m.greedy(kv, 0, prompt, 5, eos=[first[0]])
    assert ids == first and why == abi.FS_STOP_EOS
    assert kv.length(0) == 5
    # capacity 7: forwards at prefix lengths 5, 6, 7 -> 3 ids, then the context stop
    for max_new, want_n, want_why in ((4, 3, abi.FS_STOP_CONTEXT), (3, 3, abi.FS_STOP_BUDGET)):
        kv7 = m.kv(1, 7)
        ids, why = m.greedy(kv7, 0, prompt, max_new)
        ref, rwhy, _ = oracle.generate_greedy(tiny.oracle, prompt, max_new, max_context=7)
        assert (len(ids), why) == (want_n, want_why)
        assert rwhy == {abi.FS_STOP_CONTEXT: oracle.STOP_CONTEXT,
                        abi.FS_STOP_BUDGET: oracle.STOP_BUDGET}[want_why]
        assert kv7.length(0) == 7
    kv4 = m.kv(1, 4)
    with pytest.raises(abi.FsError) as e:
        m.greedy(kv4, 0, prompt, 3)
    assert e.value.status == abi.FS_ERR_CONTEXT
    with pytest.raises(abi.FsError) as e:
        m.greedy(kv, 0, [], 3)
    assert e.value.status == abi.FS_ERR_EMPTY


def test_tiny_chunked_prefill_and_page_crossing(tiny):
    toks = synth.token_ids(150, tiny.shape.vocab, seed=11).tolist()
    rl, rh, cache = tiny.oracle.forward(toks)
    kv = tiny.model.kv(3, 256)
    s = tiny.shape
    logits = torch.empty(s.vocab, device=DEV)
    # one call, and three calls ending on / across page boundaries (64, 128)
    tiny.model.prefill(kv, 0, _dev_i32(toks), logits)
    torch.cuda.synchronize()
    assert_logits_close(oracle_tensor(logits), rl, what="one-shot 150")
    for cut in ((64, 100), (63, 129)):
        kv.reset(1)
        a, b = cut
        tiny.model.prefill(kv, 1, torch.tensor(toks[:a], dtype=torch.int32), None)  # host ids
        tiny.model.prefill(kv, 1, _dev_i32(toks[a:b]), None)
        tiny.model.prefill(kv, 1, _dev_i32(toks[b:]), logits)
        torch.cuda.synchronize()
        assert_logits_close(oracle_tensor(logits), rl, what=f"chunks {cut}")
        for l in range(s.n_layers):
            k, v = kv.export(1, l, 0, 150)
            assert rel_l2(oracle_tensor(k), cache.k[l]) <= BLOCK_REL_L2
            assert rel_l2(oracle_tensor(v), cache.v[l]) <= BLOCK_REL_L2


def test_tiny_tensor_core_prefill_chunks(tiny):
    """Chunks of >= 128 rows take the tensor-core blocks (GEMMs and attention):
    chunks that start mid-page (positions 30 and 170), ragged query tiles
    (140 and 130 rows), queries of one tile spanning three KV pages."""
    toks = synth.token_ids(300, tiny.shape.vocab, seed=12).tolist()
    rl, rh, cache = tiny.oracle.forward(toks)
    s = tiny.shape
    kv = tiny.model.kv(2, 320)
    logits = torch.empty(s.vocab, device=DEV)
    hidden = torch.zeros((s.n_layers + 1, 130, s.hidden), dtype=torch.float32, device=DEV)
    tiny.model.prefill(kv, 1, _dev_i32(toks[:30]), None)
    tiny.model.prefill(kv, 1, _dev_i32(toks[30:170]), None)
    tiny.model.capture(hidden, 130)
    tiny.model.prefill(kv, 1, _dev_i32(toks[170:]), logits)
    torch.cuda.synchronize()
    assert_logits_close(oracle_tensor(logits), rl, what="chunks 30/140/130")
    assert_blocks_close(oracle_tensor(hidden), rh[:, 170:], tol=E2E_BLOCK_REL_L2,
                        what="last chunk")
    # end to end the cache takes the sanity bound; block-local below takes the bar
    for l in range(s.n_layers):
        k, v = kv.export(1, l, 0, 300)
        assert rel_l2(oracle_tensor(k), cache.k[l]) <= E2E_BLOCK_REL_L2, l
        assert rel_l2(oracle_tensor(v), cache.v[l]) <= E2E_BLOCK_REL_L2, l
    # each block alone on the oracle's input, 300 rows from position 0
    errs = blocks_local_prefill(tiny, toks, (rl, rh, cache))
    print("tiny tensor-core block-local rel-L2:", errs)


def test_tiny_single_token_prefill_returns_v_path(tiny):
    kv = tiny.model.kv(1, 8)
    gl, gh, _ = prefill_with_capture(tiny, kv, 0, [7])
    rl, rh, _ = tiny.oracle.forward([7])
    assert_blocks_close(gh, rh, tol=E2E_BLOCK_REL_L2, what="S=1")
    assert_logits_close(gl, rl, what="S=1")


def test_tiny_batched_decode_mixed_positions(tiny):
    s = tiny.shape
    lens = [5, 64, 63, 1]
    prompts = [synth.token_ids(n, s.vocab, seed=20 + i).tolist() for i, n in enumerate(lens)]
    kv = tiny.model.kv(4, 128)
    caches = []
    for i, p in enumerate(prompts):
        tiny.model.prefill(kv, i, _dev_i32(p))
        caches.append(tiny.oracle.forward(p)[2])
    nxt = [3, 4000, 17, 99]
    order = [2, 0, 3, 1]  # batch rows in a different order than sequence ids
    logits = torch.empty((4, s.vocab), device=DEV)
    am = torch.empty(4, dtype=torch.int32, device=DEV)
    tiny.model.decode_step(kv, order, _dev_i32([nxt[q] for q in order]), logits, am)
    torch.cuda.synchronize()
    for b, q in enumerate(order):
        rl = tiny.oracle.forward([nxt[q]], caches[q])[0]
        assert_logits_close(oracle_tensor(logits[b]), rl, what=f"batch row {b}")
        check_greedy_step(int(am[b]), oracle_tensor(logits[b]), rl)
        assert kv.length(q) == lens[q] + 1


def test_tiny_split_kv_decode_batch_of_seven(tiny):
    """A batch above the persistent kernel's 4 rows takes the split-KV decode
    attention: contexts from 1 to 900 positions in one launch, so most rows
    own fewer pages than the longest one (empty splits), and page-boundary
    positions (64, 128, 512)."""
    s = tiny.shape
    lens = [900, 1, 64, 128, 5, 512, 300]
    prompts = [synth.token_ids(n, s.vocab, seed=40 + i).tolist() for i, n in enumerate(lens)]
    kv = tiny.model.kv(7, 1024)
    caches = []
    for i, p in enumerate(prompts):
        tiny.model.prefill(kv, i, _dev_i32(p))
        caches.append(tiny.oracle.forward(p)[2])
    nxt = [11, 22, 33, 44, 55, 66, 77]
    order = [6, 0, 5, 1, 4, 2, 3]
    logits = torch.empty((7, s.vocab), device=DEV)
    am = torch.empty(7, dtype=torch.int32, device=DEV)
    tiny.model.decode_step(kv, order, _dev_i32([nxt[q] for q in order]), logits, am)
    torch.cuda.synchronize()
    for b, q in enumerate(order):
        rl = tiny.oracle.forward([nxt[q]], caches[q])[0]
        assert_logits_close(oracle_tensor(logits[b]), rl, what=f"batch row {b} (len {lens[q]})")
        check_greedy_step(int(am[b]), oracle_tensor(logits[b]), rl)
        assert kv.length(q) == lens[q] + 1


def test_tiny_decode_largest_batch(tiny):
    """The largest decode batch the boundary accepts (64 rows): the tiled
    CUDA-core GEMMs, split-KV attention over 64 rows and the LM head for 64
    rows, sequences of different lengths in one step."""
    s = tiny.shape
    B = 64
    lens = [1 + (7 * i) % 37 for i in range(B)]
    prompts = [synth.token_ids(n, s.vocab, seed=100 + i).tolist() for i, n in enumerate(lens)]
    kv = tiny.model.kv(B, 48)
    for i, p in enumerate(prompts):
        tiny.model.prefill(kv, i, _dev_i32(p))
    nxt = synth.token_ids(B, s.vocab, seed=99).tolist()
    order = list(range(B - 1, -1, -1))
    logits = torch.empty((B, s.vocab), device=DEV)
    am = torch.empty(B, dtype=torch.int32, device=DEV)
    tiny.model.decode_step(kv, order, _dev_i32([nxt[q] for q in order]), logits, am)
    torch.cuda.synchronize()
    for b in (0, 1, 17, 40, 63):
        q = order[b]
        cache = tiny.oracle.forward(prompts[q])[2]
        rl = tiny.oracle.forward([nxt[q]], cache)[0]
        assert_logits_close(oracle_tensor(logits[b]), rl, what=f"batch row {b} (len {lens[q]})")
        check_greedy_step(int(am[b]), oracle_tensor(logits[b]), rl)
    assert all(kv.length(q) == lens[q] + 1 for q in range(B))


def test_tiny_errors_are_reported_not_faulted(tiny):
    m, s = tiny.model, tiny.shape
    kv = m.kv(2, 16)
    with pytest.raises(abi.FsError) as e:
        m.prefill(kv, 0, torch.tensor([1, s.vocab], dtype=torch.int32))  # host id out of range
    assert e.value.status == abi.FS_ERR_TOKEN
    with pytest.raises(abi.FsError) as e:
        m.prefill(kv, 0, torch.tensor([], dtype=torch.int32))
    assert e.value.status == abi.FS_ERR_EMPTY
    with pytest.raises(abi.FsError) as e:
        m.prefill(kv, 0, torch.zeros(17, dtype=torch.int32))
    assert e.value.status == abi.FS_ERR_CONTEXT
    with pytest.raises(abi.FsError) as e:
        m.prefill(kv, 5, torch.zeros(2, dtype=torch.int32))
    assert e.value.status == abi.FS_ERR_SEQ
    with pytest.raises(abi.FsError) as e:
        m.decode_step(kv, [1, 1], torch.zeros(2, dtype=torch.int32))
    assert e.value.status == abi.FS_ERR_SEQ
    bad = torch.empty(s.vocab + 4, device=DEV)[1:]
    with pytest.raises(abi.FsError) as e:
        m.prefill(kv, 0, torch.zeros(2, dtype=torch.int32), bad)
    assert e.value.status == abi.FS_ERR_ALIGN
    assert kv.length(0) == 0
    # a device id out of range is replaced by 0 and flagged in the device error word
    assert m.device_error() == 0
    m.prefill(kv, 0, _dev_i32([3, s.vocab + 5]))
    torch.cuda.synchronize()
    assert m.device_error() == 1
    assert m.device_error() == 0


def test_tiny_random_gains_every_path(tiny_gains):
    """Non-unit norm gains on every kernel path of the tiny model: the general
    prefill (16 rows), the persistent decode kernel (teacher-forced steps and
    block-local), and the tensor-core blocks (a 300-row chunk, block-local).
    A kernel reading one gain in place of another fails the bars."""
    pair, s = tiny_gains, tiny_gains.shape
    toks = synth.token_ids(16, s.vocab, seed=0).tolist()
    ids, _, ref_logits = oracle.generate_greedy(pair.oracle, toks, 9)
    kv = pair.model.kv(1, 64)
    gl, gh, am = prefill_with_capture(pair, kv, 0, toks)
    _, rh, _ = pair.oracle.forward(toks)
    assert_blocks_close(gh, rh, tol=E2E_BLOCK_REL_L2, what="random gains prefill")
    assert_logits_close(gl, ref_logits[0], what="random gains prefill")
    check_greedy_step(am, gl, ref_logits[0])
    decode_teacher_forced(pair, kv, 0, ids[0], ids[1:], ref_logits[1:])
    blocks_local_prefill(pair, toks)
    blocks_local_decode(pair, toks + ids[:5], ids[5])
    long_toks = synth.token_ids(300, s.vocab, seed=12).tolist()
    blocks_local_prefill(pair, long_toks)


def test_q8_0_dequant_bit_exact():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    codes, scales = synth.q8_0_blocks(96, 1024, seed=77)
    codes[0, :3] = torch.tensor([-127, 127, 0], dtype=torch.int8)
    out = torch.empty((96, 1024), dtype=torch.float32, device=DEV)
    c, sc = codes.to(DEV), scales.to(DEV)
    abi.check(abi.fs_debug_dequant_q8_0(c.data_ptr(), sc.data_ptr(), 96, 1024, out.data_ptr(),
                                        torch.cuda.current_stream().cuda_stream), "dequant")
    torch.cuda.synchronize()
    want = oracle.q8_0_dequant(codes.numpy(), scales.numpy()).astype(np.float32)
    np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32), want.view(np.uint32))


def test_lm_head_exact_tie_goes_to_lowest_id():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    s = synth.TINY
    w = synth.model_weights(s, 0)
    E = w["embed"].clone()
    E[3001] = E[57]     # equal rows -> exactly equal logits
    E[4095] = E[57]
    w["embed"] = E
    m = Model(s, w, DEV)
    x = E[[57, 3001, 100]].float().to(DEV) * 7.0
    x[2] = x[0]
    logits = torch.empty((3, s.vocab), device=DEV)
    am = torch.empty(3, dtype=torch.int32, device=DEV)
    m.lm_head(x.contiguous(), logits, am)
    torch.cuda.synchronize()
    assert am.tolist() == [57, 57, 57]
    assert logits[0, 57].item() == logits[0, 3001].item() == logits[0, 4095].item()
    m.close()


# --------------------------------------------------------------------------- Qwen3-0.6B shape

def test_qwen_decode_bs1_parity(qwen):
    """8-token prompt, 32 greedy decode steps at batch 1 (teacher-forced)."""
    toks = synth.token_ids(8, qwen.shape.vocab, seed=1).tolist()
    ids, _, ref_logits = oracle.generate_greedy(qwen.oracle, toks, GREEDY_STEPS + 1)
    kv = qwen.model.kv(1, 512)
    gl, gh, am = prefill_with_capture(qwen, kv, 0, toks)
    _, rh, _ = qwen.oracle.forward(toks)
    assert_blocks_close(gh, rh, tol=E2E_BLOCK_REL_L2, what="qwen prefill 8 end to end")
    assert_logits_close(gl, ref_logits[0])
    check_greedy_step(am, gl, ref_logits[0])
    amb, hid = decode_teacher_forced(qwen, kv, 0, ids[0], ids[1:], ref_logits[1:],
                                     capture_steps=(0, 31))
    cache = qwen.oracle.forward(toks)[2]
    for i, tok in enumerate([ids[0]] + ids[1:32]):
        _, rh, cache = qwen.oracle.forward([tok], cache)
        if i in hid:
            assert_blocks_close(hid[i], rh, tol=E2E_BLOCK_REL_L2,
                                what=f"qwen decode step {i} end to end")
    REPORT.append(("qwen bf16 decode, 32 teacher-forced steps: ambiguous steps", amb, 8))
    assert amb <= 8
    blocks_local_decode(qwen, toks + ids[:31], ids[31])
    blocks_local_prefill(qwen, toks)


def test_qwen_fs_greedy_free_running(qwen):
    """Free-running fs_greedy on the Qwen3-0.6B shape: 32 ids identical to the
    oracle's. The 8-token prompt (seed 6) is one whose oracle top-2 gaps stay
    above twice the logit bound for all 32 steps, so every id must match."""
    toks = synth.token_ids(8, qwen.shape.vocab, seed=6).tolist()
    ref, _, ref_logits = oracle.generate_greedy(qwen.oracle, toks, GREEDY_STEPS)
    assert _min_top2_gap(ref_logits) >= 2 * LOGIT_ABS
    kv = qwen.model.kv(1, 512)
    ids, why = qwen.model.greedy(kv, 0, toks, GREEDY_STEPS)
    assert why == abi.FS_STOP_BUDGET and ids == ref


def test_qwen_q8_0_decode_parity():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pair = Pair(synth.QWEN3_0P6B, Q8_SEED, "q8_0", max_pos=1024)
    # prompt seed 5: the oracle's top-2 gaps stay >= 0.02 for 33 steps, more
    # than ten times the decode's measured logit error, so no step may be
    # ambiguous and the free-running ids must match too
    toks = synth.token_ids(8, pair.shape.vocab, seed=5).tolist()
    ids, _, ref_logits = oracle.generate_greedy(pair.oracle, toks, GREEDY_STEPS + 1)
    assert _min_top2_gap(ref_logits) >= 0.02
    kv = pair.model.kv(1, 512)
    gl, gh, am = prefill_with_capture(pair, kv, 0, toks)
    _, rh, _ = pair.oracle.forward(toks)
    assert_blocks_close(gh, rh, tol=E2E_BLOCK_REL_L2, what="q8_0 prefill 8 end to end")
    check_greedy_step(am, gl, ref_logits[0])
    amb, _ = decode_teacher_forced(pair, kv, 0, ids[0], ids[1:], ref_logits[1:])
    assert amb == 0
    free, why = pair.model.greedy(pair.model.kv(1, 64), 0, toks, GREEDY_STEPS)
    assert free == ids[:GREEDY_STEPS]
    blocks_local_decode(pair, toks + ids[:31], ids[31])
    blocks_local_prefill(pair, toks)
    pair.model.close()


def test_qwen_prefill_2048(qwen):
    """2048-token prefill: last-row logits, every block's hidden state and the
    filled KV cache against the oracle."""
    S = 2048
    toks = synth.token_ids(S, qwen.shape.vocab, seed=2).tolist()
    kv = qwen.model.kv(1, S)
    gl, gh, am = prefill_with_capture(qwen, kv, 0, toks)
    rl, rh, cache = qwen.oracle.forward(toks)
    assert_blocks_close(gh, rh, tol=E2E_BLOCK_REL_L2, what="prefill 2048 end to end")
    assert_logits_close(gl, rl, what="prefill 2048")
    check_greedy_step(am, gl, rl)
    for l in range(qwen.shape.n_layers):
        k, v = kv.export(0, l, 0, S)
        assert rel_l2(oracle_tensor(k), cache.k[l]) <= E2E_BLOCK_REL_L2, l
        assert rel_l2(oracle_tensor(v), cache.v[l]) <= E2E_BLOCK_REL_L2, l
    kv.close()
    blocks_local_prefill(qwen, toks, (rl, rh, cache))


def test_qwen_batched_decode_long_context(qwen):
    """Batch 16, 8192 pre-filled N(0,1) bf16 K/V per sequence, greedy steps;
    sequences 0 and 15 checked against the oracle at every step."""
    s, B, CTX, STEPS = qwen.shape, 16, 8192, 4
    kv = qwen.model.kv(B, CTX + 64)
    host_kv = {}
    for q in range(B):
        for l in range(s.n_layers):
            k, v = synth.prefilled_kv(s, CTX, seed=3, seq=q, layer=l, device=DEV)
            kv.import_(q, l, 0, k, v)
            if q in (0, B - 1):
                host_kv[(q, l)] = (oracle_tensor(k), oracle_tensor(v))
        kv.set_length(q, CTX)
    first = synth.token_ids(B, s.vocab, seed=3).tolist()
    caches = {q: oracle.KVCache(k=[host_kv[(q, l)][0] for l in range(s.n_layers)],
                                v=[host_kv[(q, l)][1] for l in range(s.n_layers)])
              for q in (0, B - 1)}
    del host_kv
    tok = list(first)
    logits = torch.empty((B, s.vocab), device=DEV)
    am = torch.empty(B, dtype=torch.int32, device=DEV)
    for step in range(STEPS):
        qwen.model.decode_step(kv, list(range(B)), _dev_i32(tok), logits, am)
        torch.cuda.synchronize()
        gpu_am = am.tolist()
        for q in (0, B - 1):
            rl, _, caches[q] = qwen.oracle.forward([tok[q]], caches[q])
            assert_logits_close(oracle_tensor(logits[q]), rl, what=f"seq {q} step {step}")
            check_greedy_step(gpu_am[q], oracle_tensor(logits[q]), rl)
            gpu_am[q] = oracle.greedy_select(rl)   # both continue on the oracle's id
        tok = gpu_am
    for q in range(B):
        assert kv.length(q) == CTX + STEPS


def test_qwen_random_gains_decode_kernel_and_tensor_cores():
    """Qwen3-0.6B shape with every RMSNorm gain vector drawn on its own: the
    persistent decode kernel block by block (context 40) and end to end
    (logits of 4 decode steps, which also apply the final-norm gain), and the
    tensor-core prefill blocks (256 rows) block by block."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pair = Pair(synth.QWEN3_0P6B, 5, max_pos=1024, gains="random")
    s = pair.shape
    toks = synth.token_ids(8, s.vocab, seed=5).tolist()
    ids, _, ref_logits = oracle.generate_greedy(pair.oracle, toks, 5)
    kv = pair.model.kv(1, 64)
    gl, _, am = prefill_with_capture(pair, kv, 0, toks)
    assert_logits_close(gl, ref_logits[0], what="random gains prefill 8")
    decode_teacher_forced(pair, kv, 0, ids[0], ids[1:], ref_logits[1:])
    ctx = synth.token_ids(40, s.vocab, seed=6).tolist()
    blocks_local_decode(pair, ctx, 123)
    blocks_local_prefill(pair, synth.token_ids(256, s.vocab, seed=7).tolist())
    pair.model.close()


@pytest.mark.parametrize("B", [2, 4])
def test_qwen_small_batch_stays_on_decode_kernel(qwen, B):
    """Batches of 2 and 4 on the Qwen3-0.6B shape run on the persistent
    decode kernel (one launch per step; their activation buffers leave a
    shorter weight ring than batch 1) and match the oracle per row."""
    s = qwen.shape
    lens = [5, 64, 63, 17][:B]
    prompts = [synth.token_ids(n, s.vocab, seed=60 + i).tolist() for i, n in enumerate(lens)]
    kv = qwen.model.kv(B, 128)
    caches = []
    for i, p in enumerate(prompts):
        qwen.model.prefill(kv, i, _dev_i32(p))
        caches.append(qwen.oracle.forward(p)[2])
    nxt = synth.token_ids(B, s.vocab, seed=70).tolist()
    order = list(range(B - 1, -1, -1))
    logits = torch.empty((B, s.vocab), device=DEV)
    am = torch.empty(B, dtype=torch.int32, device=DEV)
    toks = _dev_i32([nxt[q] for q in order])
    torch.cuda.synchronize()
    n0 = abi.fs_debug_kernel_launches()
    qwen.model.decode_step(kv, order, toks, logits, am)
    torch.cuda.synchronize()
    assert abi.fs_debug_kernel_launches() - n0 == 1
    assert qwen.model.device_error() == 0
    for b, q in enumerate(order):
        rl = qwen.oracle.forward([nxt[q]], caches[q])[0]
        assert_logits_close(oracle_tensor(logits[b]), rl, what=f"batch {B} row {b}")
        check_greedy_step(int(am[b]), oracle_tensor(logits[b]), rl)
    kv.close()


def test_decode_wait_timeout_is_reported_and_recovers(tiny):
    """The persistent decode kernel's bounded waits: with a 100 us limit and
    block 1's Q/K/V outputs withheld (nothing ever publishes them), the step
    returns, the device error word reads 3 (a wait gave up), and the next step
    with nothing withheld matches the oracle. No GPU fault is involved: the
    waits end by themselves and the kernel exits normally."""
    m, s = tiny.model, tiny.shape
    toks = synth.token_ids(16, s.vocab, seed=0).tolist()
    kv = m.kv(1, 64)
    m.prefill(kv, 0, _dev_i32(toks))
    cache = tiny.oracle.forward(toks)[2]
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
    kv.set_length(0, 16)  # the aborted step counted a position; take it back
    m.decode_step(kv, [0], _dev_i32([5]), logits, am)
    torch.cuda.synchronize()
    assert m.device_error() == 0
    rl = tiny.oracle.forward([5], cache)[0]
    assert_logits_close(oracle_tensor(logits), rl, what="step after a timeout")
    check_greedy_step(int(am.item()), oracle_tensor(logits), rl)


def test_tiny_mixed_prefill_and_decode_batch(tiny):
    """One fs_forward_batch call with a fresh 20-token prefill chunk, a decode
    row, a 7-token chunk onto a 60-position sequence (crossing the page
    boundary at 64) and a decode row at position 1: per segment the last-row
    logits and greedy id, the appended K/V and the per-block hidden states of
    every row against the oracle."""
    m, s = tiny.model, tiny.shape
    kv = m.kv(4, 128)
    hist = {1: synth.token_ids(37, s.vocab, seed=81).tolist(),
            2: synth.token_ids(60, s.vocab, seed=82).tolist(),
            3: synth.token_ids(1, s.vocab, seed=83).tolist()}
    caches = {0: None}
    for q, toks in hist.items():
        m.prefill(kv, q, _dev_i32(toks))
        caches[q] = tiny.oracle.forward(toks)[2]
    segs = [(0, synth.token_ids(20, s.vocab, seed=84).tolist()), (1, [123]),
            (2, synth.token_ids(7, s.vocab, seed=85).tolist()), (3, [4000])]
    rows = sum(len(t) for _, t in segs)
    hidden = torch.zeros((s.n_layers + 1, rows, s.hidden), device=DEV)
    logits = torch.empty((len(segs), s.vocab), device=DEV)
    am = torch.empty(len(segs), dtype=torch.int32, device=DEV)
    m.capture(hidden, rows)
    m.forward_batch(kv, segs, logits, am)
    torch.cuda.synchronize()
    gh = oracle_tensor(hidden)
    # processing order: all rows but each segment's last, then the last rows
    order = [(i, t) for i, (_, ts) in enumerate(segs) for t in range(len(ts) - 1)]
    order += [(i, len(ts) - 1) for i, (_, ts) in enumerate(segs)]
    for i, (q, toks) in enumerate(segs):
        rl, rh, cache = tiny.oracle.forward(toks, caches[q])
        assert_logits_close(oracle_tensor(logits[i]), rl, what=f"mixed batch segment {i}")
        check_greedy_step(int(am[i]), oracle_tensor(logits[i]), rl)
        got = np.stack([gh[:, order.index((i, t))] for t in range(len(toks))], axis=1)
        assert_blocks_close(got, rh, tol=E2E_BLOCK_REL_L2, what=f"mixed batch segment {i}")
        n = len(hist.get(q, [])) + len(toks)
        assert kv.length(q) == n
        for l in range(s.n_layers):
            k, v = kv.export(q, l, 0, n)
            assert rel_l2(oracle_tensor(k), cache.k[l]) <= BLOCK_REL_L2
            assert rel_l2(oracle_tensor(v), cache.v[l]) <= BLOCK_REL_L2
