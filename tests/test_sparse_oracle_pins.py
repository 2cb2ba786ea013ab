"""Pins for the block-sparse oracle (oracle/sparse_ref.py), on the CPU.

Tied to things other than itself: the dense oracle (all-ones mask), dense
attention of sliced inputs (a block-diagonal mask is independent attention per
block; a single visible key block is attention over that slice), the
empty-row convention, and invariance under permuting whole key blocks.
"""
import numpy as np
import pytest

from oracle import attn_ref as ref
from oracle import sparse_ref as sp


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("causal", [False, True])
def test_all_ones_equals_dense(causal):
    q, k, v = rnd((1, 300, 4, 32), 1), rnd((1, 300, 2, 32), 2), rnd((1, 300, 2, 32), 3)
    bm = np.ones((1, 4, 3, 3), np.uint8)
    O, L = sp.attention_fwd_blocksparse(q, k, v, bm, causal, 0.2)
    O2, L2 = ref.attention_fwd(q, k, v, causal, 0.2)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(L, L2)


def test_block_diagonal_is_independent_blocks():
    q, k, v = rnd((1, 384, 2, 16), 4), rnd((1, 384, 2, 16), 5), rnd((1, 384, 2, 16), 6)
    bm = np.zeros((1, 2, 3, 3), np.uint8)
    for i in range(3):
        bm[0, :, i, i] = 1
    O, L = sp.attention_fwd_blocksparse(q, k, v, bm, False, 0.3)
    for i in range(3):
        s = slice(128 * i, 128 * (i + 1))
        Oi, Li = ref.attention_fwd(q[:, s], k[:, s], v[:, s], False, 0.3)
        np.testing.assert_allclose(O[:, s], Oi, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(L[:, :, s], Li, rtol=1e-12, atol=1e-12)


def test_single_key_block_per_row_and_empty_rows():
    q, k, v = rnd((1, 200, 1, 16), 7), rnd((1, 330, 1, 16), 8), rnd((1, 330, 1, 16), 9)
    bm = np.zeros((1, 1, 2, 3), np.uint8)
    bm[0, 0, 0, 2] = 1  # rows 0..127 see keys 256..329 only; rows 128..199 see nothing
    O, L = sp.attention_fwd_blocksparse(q, k, v, bm, False, 0.25)
    O2, L2 = ref.attention_fwd(q[:, :128], k[:, 256:], v[:, 256:], False, 0.25)
    np.testing.assert_allclose(O[:, :128], O2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(L[:, :, :128], L2, rtol=1e-12, atol=1e-12)
    assert np.all(O[:, 128:] == 0) and np.all(L[:, :, 128:] == -np.inf)


def test_permuting_key_blocks_with_the_mask_is_invariant():
    rng = np.random.default_rng(10)
    q, k, v = rnd((1, 256, 2, 16), 11), rnd((1, 512, 1, 16), 12), rnd((1, 512, 1, 16), 13)
    bm = (rng.random((1, 2, 2, 4)) < 0.6).astype(np.uint8)
    bm[..., 0] = 1
    perm = np.array([2, 0, 3, 1])
    kp = np.concatenate([k[:, 128 * p:128 * (p + 1)] for p in perm], axis=1)
    vp = np.concatenate([v[:, 128 * p:128 * (p + 1)] for p in perm], axis=1)
    O, L = sp.attention_fwd_blocksparse(q, k, v, bm, False, 0.25)
    Op, Lp = sp.attention_fwd_blocksparse(q, kp, vp, bm[..., perm], False, 0.25)
    np.testing.assert_allclose(O, Op, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(L, Lp, rtol=1e-12, atol=1e-12)


def test_planted_mistake_transposed_mask_is_caught():
    q, k, v = rnd((1, 256, 1, 16), 14), rnd((1, 256, 1, 16), 15), rnd((1, 256, 1, 16), 16)
    bm = np.array([[[[1, 0], [1, 1]]]], np.uint8)
    O, _ = sp.attention_fwd_blocksparse(q, k, v, bm, False, 0.25)
    Ot, _ = sp.attention_fwd_blocksparse(q, k, v, bm.transpose(0, 1, 3, 2), False, 0.25)
    assert np.max(np.abs(O - Ot)) > 0.1


def test_flops_count_visible_pairs():
    bm = np.array([[[[1, 0], [1, 1]]]], np.uint8)
    assert sp.blocksparse_flops(bm, 256, 256, 8, False) == 4 * 8 * (3 * 128 * 128)
    assert sp.blocksparse_flops(bm, 256, 256, 8, True) == 4 * 8 * (128 * 129 // 2 + 128 * 128 + 128 * 129 // 2)


def test_rows_variant_equals_full():
    q, k, v = rnd((2, 300, 4, 16), 20), rnd((2, 400, 2, 16), 21), rnd((2, 400, 2, 16), 22)
    bm = (np.random.default_rng(23).random((2, 4, 3, 4)) < 0.5).astype(np.uint8)
    O, L = sp.attention_fwd_blocksparse(q, k, v, bm, True, 0.25)
    rows = [0, 5, 127, 128, 299]
    Or, Lr = sp.attention_fwd_blocksparse_rows(q, k, v, bm, True, 0.25, 1, 3, rows)
    np.testing.assert_array_equal(Or, O[1, rows, 3, :])
    np.testing.assert_array_equal(Lr, L[1, 3, rows])
