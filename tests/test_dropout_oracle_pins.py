"""Pins for the dropout oracle (oracle/dropout_ref.py), on the CPU.

The generator is pinned to the published Philox4x32-10 known-answer vectors
(tests/golden/philox4x32_10_kat.json); the keep rate to the binomial law; the
1/(1-p) scaling to the expectation over seeds (E[O_drop] = O); p = 0 to the
plain oracle; the backward to central finite differences with the mask held
fixed, and D = rowsum(dO * O) to its definition through P and dP.
"""
import json
import os

import numpy as np
import pytest

from oracle import attn_ref as ref
from oracle import dropout_ref as dr

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.json")


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_philox_known_answers():
    with open(GOLDEN) as fh:
        vectors = json.load(fh)["vectors"]
    for vec in vectors:
        c = [int(x, 16) for x in vec["counter"]]
        k = [int(x, 16) for x in vec["key"]]
        out = dr.philox4x32(*[np.array([x]) for x in c], k[0], k[1])
        assert [int(o[0]) for o in out] == [int(x, 16) for x in vec["out"]]


def test_keep_rate_is_binomial():
    Nq, Nk, p = 256, 384, 0.3
    M = dr.keep_mask(0, 3, 8, Nq, Nk, p, seed=0x1234_5678_9ABC, offset=7)
    n = Nq * Nk
    mean = M.mean()
    assert abs(mean - (1 - p)) < 5 * np.sqrt(p * (1 - p) / n)
    # different heads, seeds and offsets give different masks
    assert (M != dr.keep_mask(0, 4, 8, Nq, Nk, p, 0x1234_5678_9ABC, 7)).mean() > 0.3
    assert (M != dr.keep_mask(0, 3, 8, Nq, Nk, p, 0x1234_5678_9ABD, 7)).mean() > 0.3
    assert (M != dr.keep_mask(0, 3, 8, Nq, Nk, p, 0x1234_5678_9ABC, 8)).mean() > 0.3


def test_mask_value_selection():
    # (i, j) takes 16-bit value e = 4 (i & 1) + (j & 3) of the call at counter (j >> 2, i >> 1, bh,
    # offset): the low half of word e >> 1 for even e, the high half for odd e.  Counter (3, 10)
    # covers queries 20, 21 and keys 12 .. 15.
    seed, off, bh = 0xDEADBEEF00C0FFEE, 5, 2 * 4 + 1
    w = dr.philox4x32(np.array([3]), np.array([10]), np.array([bh]), np.array([off]), seed & 0xFFFFFFFF, seed >> 32)
    words = [int(x[0]) for x in w]
    values = [words[0] & 0xFFFF, words[0] >> 16, words[1] & 0xFFFF, words[1] >> 16,
              words[2] & 0xFFFF, words[2] >> 16, words[3] & 0xFFFF, words[3] >> 16]
    for pr in (0.25, 0.5, 0.9):
        thr = dr.keep_threshold(pr)
        M = dr.keep_mask(2, 1, 4, 22, 16, pr, seed, off)
        for di in (0, 1):
            for dj in range(4):
                assert M[20 + di, 12 + dj] == (values[4 * di + dj] >= thr)
    # the neighbouring blocks come from other counters
    M = dr.keep_mask(2, 1, 4, 24, 20, 0.5, seed, off)
    w2 = dr.philox4x32(np.array([4]), np.array([11]), np.array([bh]), np.array([off]), seed & 0xFFFFFFFF, seed >> 32)
    assert M[23, 19] == ((int(w2[3][0]) >> 16) >= dr.keep_threshold(0.5))


def test_keep_threshold():
    assert dr.keep_threshold(0.0) == 0
    assert dr.keep_threshold(0.1) == 6553
    assert dr.keep_threshold(0.5) == 32768
    assert dr.keep_threshold(1 - 2 ** -20) == 65535
    with pytest.raises(ValueError):
        dr.keep_threshold(1.0)


def test_p_zero_is_plain_attention():
    q, k, v, do = rnd((1, 70, 2, 16), 1), rnd((1, 90, 1, 16), 2), rnd((1, 90, 1, 16), 3), rnd((1, 70, 2, 16), 4)
    O, L = dr.attention_fwd_dropout(q, k, v, True, 0.25, 0.0, 99, 0)
    O2, L2 = ref.attention_fwd(q, k, v, True, 0.25)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(L, L2)
    g = dr.attention_bwd_dropout(q, k, v, do, True, 0.25, 0.0, 99, 0)
    g2 = ref.attention_bwd(q, k, v, do, True, 0.25)
    for a, b in zip(g, g2):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_expectation_over_seeds_is_the_undropped_output():
    q, k, v = rnd((1, 8, 1, 4), 5), rnd((1, 8, 1, 4), 6), rnd((1, 8, 1, 4), 7)
    O0, _ = ref.attention_fwd(q, k, v, False, 0.5)
    p, n = 0.4, 3000
    acc = np.zeros_like(O0)
    sq = np.zeros_like(O0)
    for s in range(n):
        O, _ = dr.attention_fwd_dropout(q, k, v, False, 0.5, p, seed=1000 + s, offset=0)
        acc += O
        sq += O * O
    mean = acc / n
    sd = np.sqrt(np.maximum(sq / n - mean ** 2, 1e-30) / n)
    assert np.all(np.abs(mean - O0) <= 5 * sd + 1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_finite_differences(causal):
    q, k, v, do = rnd((1, 6, 2, 4), 8), rnd((1, 7, 1, 4), 9), rnd((1, 7, 1, 4), 10), rnd((1, 6, 2, 4), 11)
    p, seed, off, scale = 0.3, 77, 3, 0.6
    dq, dk, dv = dr.attention_bwd_dropout(q, k, v, do, causal, scale, p, seed, off)

    def loss(q_, k_, v_):
        O, _ = dr.attention_fwd_dropout(q_, k_, v_, causal, scale, p, seed, off)
        return float(np.sum(O * do))

    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in [(0, 0, 0, 0), (0, 3, 0, 2), (0, 5, x.shape[2] - 1, 3)]:
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, g[idx])


def test_planted_mistake_missing_rescale_is_caught():
    q, k, v = rnd((1, 8, 1, 4), 5), rnd((1, 8, 1, 4), 6), rnd((1, 8, 1, 4), 7)
    O0, _ = ref.attention_fwd(q, k, v, False, 0.5)
    p, n = 0.4, 400
    acc = np.zeros_like(O0)
    for s in range(n):
        O, _ = dr.attention_fwd_dropout(q, k, v, False, 0.5, p, seed=1000 + s, offset=0)
        acc += O * (1 - p)  # what a kernel without the 1/(1-p) factor would return
    assert np.max(np.abs(acc / n - O0)) > 0.1


def test_block_evaluated_mask_equals_one_call_per_element():
    # brute force: one Philox call per (i, j) at the counter of its 2 x 4 block, value picked
    # by e = 4 (i & 1) + (j & 3); odd sizes leave partial blocks at both edges
    Nq, Nk, p, seed, off, b, h, Hq = 13, 23, 0.37, 0xA5A5_0F0F_1234_5678, 11, 1, 2, 3
    M = dr.keep_mask(b, h, Hq, Nq, Nk, p, seed, off)
    thr = dr.keep_threshold(p)
    for i in range(Nq):
        for j in range(Nk):
            w = dr.philox4x32(np.array([j >> 2]), np.array([i >> 1]), np.array([b * Hq + h]), np.array([off]),
                              seed & 0xFFFFFFFF, seed >> 32)
            e = 4 * (i & 1) + (j & 3)
            value = (int(w[e >> 1][0]) >> (16 * (e & 1))) & 0xFFFF
            assert M[i, j] == (value >= thr), (i, j)
    rows = [12, 0, 5, 6, 5]
    np.testing.assert_array_equal(dr.keep_mask(b, h, Hq, Nq, Nk, p, seed, off, rows), M[rows])


def test_sampled_heads_and_row_chunks_change_nothing():
    q, k, v, do = rnd((2, 37, 4, 8), 21), rnd((2, 41, 2, 8), 22), rnd((2, 41, 2, 8), 23), rnd((2, 37, 4, 8), 24)
    args = (True, 0.4, 0.2, 1234, 5)
    O, L = dr.attention_fwd_dropout(q, k, v, *args)
    O2, L2 = dr.attention_fwd_dropout(q, k, v, *args, heads=[(1, 3), (0, 0)], row_chunk=6)
    for b, h in [(1, 3), (0, 0)]:
        np.testing.assert_allclose(O2[b, :, h], O[b, :, h], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(L2[b, h], L[b, h], rtol=1e-12, atol=1e-14)
    assert np.isnan(O2[0, :, 1]).all()
    g = dr.attention_bwd_dropout(q, k, v, do, *args)
    g2 = dr.attention_bwd_dropout(q, k, v, do, *args, kv_heads=[(1, 1)], row_chunk=7)
    np.testing.assert_allclose(g2[0][1, :, 2:4], g[0][1, :, 2:4], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(g2[1][1, :, 1], g[1][1, :, 1], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(g2[2][1, :, 1], g[2][1, :, 1], rtol=1e-11, atol=1e-13)
    assert np.isnan(g2[1][0]).all()
