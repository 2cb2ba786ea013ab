"""CPU oracle for block-sparse attention -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs use
this module; it never imports the CUDA product package.

Source: "FlashAttention-2 (KO)" (systems-analysis.info), "결과
(FlashAttention-1)": extending the IO-aware kernel with a block-sparse pattern
gives an approximate attention that is faster than earlier approximate
methods.  The pages give neither the block size nor the mask format.  Readings:

* the mask is a table of 128 x 128 blocks, ``block_mask[b, h, I, J]`` for query
  block I (rows 128 I .. 128 I + 127) and key block J, of shape
  [B, Hq, ceil(Nq / 128), ceil(Nk / 128)]; nonzero means the block is computed;
* key j is visible from query i iff block_mask[b, h, i // 128, j // 128] is
  nonzero and, when causal, j <= i + (Nk - Nq); a row with no visible key has
  O = 0 and LSE = -inf;
* within the visible set the result is exact attention (the approximation is
  the pattern itself), computed here from the materialised scores.
"""
from __future__ import annotations

import numpy as np

from .attn_ref import _check_shapes, _f64, scores, softmax_rows, visible_mask

__all__ = ["BLOCK", "expand_block_mask", "attention_fwd_blocksparse", "attention_fwd_blocksparse_rows",
           "blocksparse_flops"]

BLOCK = 128


def expand_block_mask(block_mask_bh, Nq: int, Nk: int, causal: bool) -> np.ndarray:
    """Boolean [Nq, Nk] visibility of one (b, h) from its [nqb, nkb] block table."""
    bm = np.asarray(block_mask_bh) != 0
    vis = np.repeat(np.repeat(bm, BLOCK, axis=0), BLOCK, axis=1)[:Nq, :Nk]
    return vis & visible_mask(Nq, Nk, causal)


def attention_fwd_blocksparse(q, k, v, block_mask, causal: bool, scale: float, heads=None):
    """O [B, Nq, Hq, d] and LSE [B, Hq, Nq] (fp64) of attention restricted to the block pattern."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Nk, Hq, Hkv, d = _check_shapes(q, k, v)
    bm = np.asarray(block_mask)
    if bm.shape != (B, Hq, -(-Nq // BLOCK), -(-Nk // BLOCK)):
        raise ValueError("block_mask must be [B, Hq, ceil(Nq/128), ceil(Nk/128)]")
    G = Hq // Hkv
    O = np.full((B, Nq, Hq, d), np.nan)
    LSE = np.full((B, Hq, Nq), np.nan)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in todo:
        mask = expand_block_mask(bm[b, h], Nq, Nk, causal)
        S = scores(q[b, :, h, :], k[b, :, h // G, :], scale, mask)
        P, lse = softmax_rows(S)
        O[b, :, h, :] = P @ v[b, :, h // G, :]
        LSE[b, h, :] = lse
    return O, LSE


def attention_fwd_blocksparse_rows(q, k, v, block_mask, causal: bool, scale: float, b: int, h: int, rows):
    """O [len(rows), d] and LSE [len(rows)] of selected query rows of one (b, h_q)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Nk, Hq, Hkv, d = _check_shapes(q, k, v)
    rows = np.asarray(rows, dtype=np.int64)
    mask = expand_block_mask(np.asarray(block_mask)[b, h], Nq, Nk, causal)[rows]
    hk = h // (Hq // Hkv)
    S = scores(q[b, rows, h, :], k[b, :, hk, :], scale, mask)
    P, lse = softmax_rows(S)
    return P @ v[b, :, hk, :], lse


def blocksparse_flops(block_mask, Nq: int, Nk: int, d: int, causal: bool) -> float:
    """FLOPs of the visible (query, key) pairs: 4 d per pair (the two GEMMs)."""
    bm = np.asarray(block_mask) != 0
    pairs = 0
    for b in range(bm.shape[0]):
        for h in range(bm.shape[1]):
            pairs += int(expand_block_mask(bm[b, h], Nq, Nk, causal).sum())
    return 4.0 * d * pairs
