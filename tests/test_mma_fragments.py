"""The k order of the 5..16-row tensor-core GEMV, checked on the CPU.

mma.sync m16n8k16 (row.col) computes D[16 x 8] += A[16 x 16] B[16 x 8]
from per-lane fragments (g = lane / 4, t = lane % 4):

* A: a0 a1 = A[g][2t], A[g][2t+1]; a2 a3 = A[g+8][2t], A[g+8][2t+1];
  a4 a5 = A[g][2t+8], A[g][2t+9]; a6 a7 = A[g+8][2t+8], A[g+8][2t+9];
* B: b0 b1 = B[2t][g], B[2t+1][g]; b2 b3 = B[2t+8][g], B[2t+9][g];
* D: d0 d1 = D[g][2t], D[g][2t+1]; d2 d3 = D[g+8][2t], D[g+8][2t+1].

The kernel gives lane (g, t) the eight consecutive physical k 8t .. 8t+7 of
a 32-wide group of the weight row n0 + g, and of the activation rows g and
g + 8, and feeds them to two MMAs (k 8t..8t+3, then 8t+4..8t+7). This model
builds the A and B matrices each MMA sees from those lane registers and
checks that the two products add up to the plain dot products over the 32
physical k: every product pairs matching k, and every k is used once.
"""

import numpy as np


def lane_fragments(x, w, half):
    """A and B as one MMA sees them; half 0 uses k 8t..8t+3, half 1 8t+4..8t+7.
    x: [16 rows][32 k], w: [8 rows][32 k] (one 32-wide group)."""
    A = np.full((16, 16), np.nan)
    B = np.full((16, 8), np.nan)
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        base = 8 * t + 4 * half
        # registers: xa = x[g][base .. base+3] as (.x pair, .y pair), xb the row g + 8
        A[g, 2 * t], A[g, 2 * t + 1] = x[g, base], x[g, base + 1]              # a0 a1
        A[g + 8, 2 * t], A[g + 8, 2 * t + 1] = x[g + 8, base], x[g + 8, base + 1]  # a2 a3
        A[g, 2 * t + 8], A[g, 2 * t + 9] = x[g, base + 2], x[g, base + 3]      # a4 a5
        A[g + 8, 2 * t + 8], A[g + 8, 2 * t + 9] = x[g + 8, base + 2], x[g + 8, base + 3]
        B[2 * t, g], B[2 * t + 1, g] = w[g, base], w[g, base + 1]              # b0 b1
        B[2 * t + 8, g], B[2 * t + 9, g] = w[g, base + 2], w[g, base + 3]      # b2 b3
    return A, B


def test_each_lane_register_lands_on_one_fragment_element():
    x = np.arange(16 * 32, dtype=np.float64).reshape(16, 32)
    w = np.arange(8 * 32, dtype=np.float64).reshape(8, 32)
    for half in (0, 1):
        A, B = lane_fragments(x, w, half)
        assert not np.isnan(A).any() and not np.isnan(B).any()


def test_two_mmas_give_the_dot_products_over_the_group():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((16, 32))
    w = rng.standard_normal((8, 32))
    D = np.zeros((16, 8))
    for half in (0, 1):
        A, B = lane_fragments(x, w, half)
        D += A @ B
    np.testing.assert_allclose(D, x @ w.T, rtol=1e-12, atol=1e-12)


def test_each_physical_k_is_used_exactly_once():
    # one-hot activations: D[r][n] counts how often x[r][k] met w[n][k]
    for k in range(32):
        x = np.zeros((16, 32))
        x[:, k] = 1.0
        w = np.zeros((8, 32))
        w[:, k] = 1.0
        D = sum(np.nan_to_num(a) @ np.nan_to_num(b)
                for a, b in (lane_fragments(x, w, h) for h in (0, 1)))
        assert np.array_equal(D, np.ones((16, 8))), k


def test_outputs_land_where_the_kernel_stores_them():
    # the kernel stores d_e to (row g + 8 (e >> 1), column n0 + 2t + (e & 1))
    seen = set()
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        for e in range(4):
            seen.add((g + (e >> 1) * 8, 2 * t + (e & 1)))
    assert seen == {(r, n) for r in range(16) for n in range(8)}


def bf16(v):
    """Round to bf16 (nearest even), as float64."""
    a = np.asarray(v, dtype=np.float32).copy()
    u = a.view(np.uint32)
    u += 0x7FFF + ((u >> 16) & 1)
    u &= 0xFFFF0000
    return a.astype(np.float64)


def test_attention_p_fragments_come_from_the_right_lanes():
    """Row-split decode attention, one 16-key half: after S = K q^T, lane
    (g, t) holds p(key g) and p(key g + 8) of head t (t < 2). The P V MMA's B
    column g is head g / 2, term g % 2 (bf16 hi, then the remainder); the
    kernel reads key 2t and 2t + 1 (b0 b1) and 2t + 8, 2t + 9 (b2 b3) from
    lanes (2t) * 4 + g / 2 and (2t + 1) * 4 + g / 2. With A = V^T, columns
    2h and 2h + 1 of D then add up to head h's P V."""
    rng = np.random.default_rng(3)
    p = rng.random((16, 2))           # p[key][head]
    V = rng.standard_normal((16, 16)) # V[key][dim]
    # lane registers after the softmax: pr0 = p(key g, head t), pr1 = p(key g + 8, head t)
    pr0 = np.zeros(32)
    pr1 = np.zeros(32)
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        if t < 2:
            pr0[lane], pr1[lane] = p[g, t], p[g + 8, t]
    B = np.zeros((16, 8))
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        hn, lo = g >> 1, g & 1
        if g >= 4:  # columns past the two heads' terms are zero
            continue
        q00, q01 = pr0[(2 * t) * 4 + hn], pr0[(2 * t + 1) * 4 + hn]
        q10, q11 = pr1[(2 * t) * 4 + hn], pr1[(2 * t + 1) * 4 + hn]

        def term(v):
            h = bf16(v)
            return bf16(v - h) if lo else h

        B[2 * t, g], B[2 * t + 1, g] = term(q00), term(q01)
        B[2 * t + 8, g], B[2 * t + 9, g] = term(q10), term(q11)
    D = V.T @ B  # A = V^T: rows = dims, columns = keys
    for h in range(2):
        np.testing.assert_allclose(D[:, 2 * h] + D[:, 2 * h + 1], V.T @ p[:, h],
                                   rtol=2e-5, atol=2e-5)
