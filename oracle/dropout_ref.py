"""CPU oracle for attention with fused dropout -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs use
this module; it never imports the CUDA product package.

Sources: "FlashAttention 심층 분석" (ryotta.opik.net), section 2: dropout is one
of the steps the kernel fuses (scaling, masking, softmax, dropout, the P V
product); section 4: the backward pass recomputes what it needs instead of
storing it -- for dropout that means regenerating the same mask.  The pages
name no generator and no keep rule.  Readings:

* generator: Philox4x32 with 10 rounds (Salmon, Moraes, Dror, Shaw, "Parallel
  random numbers: as easy as 1, 2, 3", SC 2011), written here from that
  definition: per round, (c0, c1, c2, c3) -> (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2),
  hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)) with M0 = 0xD2511F53, M1 = 0xCD9E8D57, and
  the key bumped by (0x9E3779B9, 0xBB67AE85) before every round but the first;
* one call covers a 2 x 4 block of (query i, key j) for one (b, h_q):
  counter = (j >> 2, i >> 1, b * Hq + h, offset), key = (seed_lo, seed_hi);
  its four 32-bit words are read as eight 16-bit values, the low half of a
  word first, and value e = 4 (i & 1) + (j & 3) belongs to (i, j);
* keep (i, j) iff that value >= floor(p * 2^16) (p in [0, 1)); kept weights are
  scaled by 1 / (1 - p), dropped ones are 0;
* O = (P * M / (1 - p)) V with P the softmax of the scores (unchanged by
  dropout) and LSE that of the scores; backward by the chain rule with the
  same mask: dV = (P * M)^T dO / (1 - p), dP = M * (dO V^T) / (1 - p),
  D_i = sum_j P_ij dP_ij = sum_c dO_ic O_ic, dS = P * (dP - D),
  dQ = scale dS K, dK = scale dS^T Q.
"""
from __future__ import annotations

import numpy as np

from .attn_ref import _check_shapes, _f64, scores, softmax_rows, visible_mask

__all__ = ["philox4x32", "keep_threshold", "keep_mask", "attention_fwd_dropout", "attention_bwd_dropout"]

_M0, _M1 = np.uint64(0xD2511F53), np.uint64(0xCD9E8D57)
_W0, _W1 = 0x9E3779B9, 0xBB67AE85
_LO = np.uint64(0xFFFFFFFF)


def philox4x32(c0, c1, c2, c3, k0: int, k1: int, rounds: int = 10):
    """Philox4x32-R on arrays of 32-bit counter words; returns the four output word arrays (uint64 holding 32 bits)."""
    c = [np.asarray(x, dtype=np.uint64) & _LO for x in (c0, c1, c2, c3)]
    k0, k1 = k0 & 0xFFFFFFFF, k1 & 0xFFFFFFFF
    for r in range(rounds):
        if r > 0:
            k0 = (k0 + _W0) & 0xFFFFFFFF
            k1 = (k1 + _W1) & 0xFFFFFFFF
        p0 = _M0 * c[0]
        p1 = _M1 * c[2]
        c = [(p1 >> np.uint64(32)) ^ c[1] ^ np.uint64(k0), p1 & _LO, (p0 >> np.uint64(32)) ^ c[3] ^ np.uint64(k1),
             p0 & _LO]
    return c


def keep_threshold(p: float) -> int:
    """floor(p * 2^16), capped to 2^16 - 1."""
    if not 0.0 <= p < 1.0:
        raise ValueError("dropout probability must be in [0, 1)")
    return min(int(np.floor(p * 65536.0)), 0xFFFF)


def keep_mask(b: int, h: int, Hq: int, Nq: int, Nk: int, p: float, seed: int, offset: int, rows=None) -> np.ndarray:
    """Boolean [Nq, Nk] (or [len(rows), Nk]): True where (i, j) of head (b, h) is kept.

    One Philox call per 2 x 4 block of (query pair i >> 1, key quad j >> 2) that the
    requested rows touch; element (i, j) reads 16-bit value e = 4 (i & 1) + (j & 3)
    of its block's call (half e & 1 of word e >> 1).
    """
    rows = np.arange(Nq, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    pairs = np.unique(rows >> 1)
    quads = np.arange((Nk + 3) // 4, dtype=np.int64)
    pp, qq = np.meshgrid(pairs.astype(np.uint64), quads.astype(np.uint64), indexing="ij")
    words = philox4x32(qq, pp, np.full(pp.shape, b * Hq + h, np.uint64), np.full(pp.shape, offset, np.uint64),
                       seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    values = np.stack([((words[e >> 1] >> np.uint64(16 * (e & 1))) & np.uint64(0xFFFF)).astype(np.uint16)
                       for e in range(8)])  # [8, pairs, quads]
    j = np.arange(Nk, dtype=np.int64)
    e = 4 * (rows & 1)[:, None] + (j & 3)[None, :]
    value = values[e, np.searchsorted(pairs, rows >> 1)[:, None], (j >> 2)[None, :]]
    return value >= keep_threshold(p)


def attention_fwd_dropout(q, k, v, causal: bool, scale: float, p: float, seed: int, offset: int, heads=None,
                          row_chunk: int = 2048):
    """O [B, Nq, Hq, d] and LSE [B, Hq, Nq] (fp64) with dropout on P.

    ``heads`` optionally restricts the work to a list of (b, h_q) pairs (the other
    outputs stay NaN).  Query rows are taken ``row_chunk`` at a time to bound
    memory; every row's softmax still spans its whole score row, so the chunking
    changes no value.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Nk, Hq, Hkv, d = _check_shapes(q, k, v)
    G = Hq // Hkv
    vis = visible_mask(Nq, Nk, causal)
    O = np.full((B, Nq, Hq, d), np.nan)
    LSE = np.full((B, Hq, Nq), np.nan)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in todo:
        for i0 in range(0, Nq, row_chunk):
            rows = np.arange(i0, min(i0 + row_chunk, Nq))
            S = scores(q[b, rows, h, :], k[b, :, h // G, :], scale, vis[rows])
            P, lse = softmax_rows(S)
            M = keep_mask(b, h, Hq, Nq, Nk, p, seed, offset, rows)
            O[b, rows, h, :] = (P * M / (1.0 - p)) @ v[b, :, h // G, :]
            LSE[b, h, rows] = lse
    return O, LSE


def attention_bwd_dropout(q, k, v, do, causal: bool, scale: float, p: float, seed: int, offset: int, kv_heads=None,
                          row_chunk: int = 2048):
    """dQ, dK, dV (fp64) of sum(dO * O) for the dropout forward above (same mask).

    ``kv_heads`` optionally restricts the work to a list of (b, h_kv) pairs (their
    query heads' dQ and their own dK, dV; the rest stays NaN).  Query rows are
    taken ``row_chunk`` at a time; dK and dV add up the chunks' contributions.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Nq, Nk, Hq, Hkv, d = _check_shapes(q, k, v)
    G = Hq // Hkv
    vis = visible_mask(Nq, Nk, causal)
    dq = np.full_like(q, np.nan)
    dk = np.full_like(k, np.nan)
    dv = np.full_like(v, np.nan)
    r = 1.0 / (1.0 - p)
    todo = kv_heads if kv_heads is not None else [(b, hk) for b in range(B) for hk in range(Hkv)]
    for b, hk in todo:
        K, V = k[b, :, hk, :], v[b, :, hk, :]
        dK = np.zeros((Nk, d))
        dV = np.zeros((Nk, d))
        for h in range(hk * G, (hk + 1) * G):
            for i0 in range(0, Nq, row_chunk):
                rows = np.arange(i0, min(i0 + row_chunk, Nq))
                Q, dO = q[b, rows, h, :], do[b, rows, h, :]
                P, _ = softmax_rows(scores(Q, K, scale, vis[rows]))
                M = keep_mask(b, h, Hq, Nq, Nk, p, seed, offset, rows)
                Pd = P * M * r
                O = Pd @ V
                dV += Pd.T @ dO
                dP = M * r * (dO @ V.T)
                D = np.sum(dO * O, axis=1, keepdims=True)
                dS = P * (dP - D)
                dq[b, rows, h, :] = scale * dS @ K
                dK += scale * dS.T @ Q
        dk[b, :, hk, :] = dK
        dv[b, :, hk, :] = dV
    return dq, dk, dv
