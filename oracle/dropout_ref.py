"""CPU oracle for attention with fused dropout -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs use
this module; it never imports the CUDA product package.

Sources: "FlashAttention 심층 분석" (ryotta.opik.net), section 2: dropout is one
of the steps the kernel fuses (scaling, masking, softmax, dropout, the P V
product); section 4: the backward pass recomputes what it needs instead of
storing it -- for dropout that means regenerating the same mask.  The pages
name no generator and no keep rule.  Readings (listed in the design doc):

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


def keep_mask(b: int, h: int, Hq: int, Nq: int, Nk: int, p: float, seed: int, offset: int) -> np.ndarray:
    """Boolean [Nq, Nk]: True where (i, j) of head (b, h) is kept."""
    i = np.arange(Nq, dtype=np.uint64)[:, None]
    j = np.arange(Nk, dtype=np.uint64)[None, :]
    ii, jj = np.broadcast_arrays(i, j)
    words = philox4x32(jj >> np.uint64(2), ii >> np.uint64(1), np.full(ii.shape, b * Hq + h, np.uint64),
                       np.full(ii.shape, offset, np.uint64), seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    e = (4 * (ii & np.uint64(1)) + (jj & np.uint64(3))).astype(np.int64)
    w = np.choose(e >> 1, words)
    value = (w >> (np.uint64(16) * (e & 1).astype(np.uint64))) & np.uint64(0xFFFF)
    return value >= np.uint64(keep_threshold(p))


def attention_fwd_dropout(q, k, v, causal: bool, scale: float, p: float, seed: int, offset: int):
    """O [B, Nq, Hq, d] and LSE [B, Hq, Nq] (fp64) with dropout on P."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Nk, Hq, Hkv, d = _check_shapes(q, k, v)
    G = Hq // Hkv
    vis = visible_mask(Nq, Nk, causal)
    O = np.empty((B, Nq, Hq, d))
    LSE = np.empty((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            S = scores(q[b, :, h, :], k[b, :, h // G, :], scale, vis)
            P, lse = softmax_rows(S)
            M = keep_mask(b, h, Hq, Nq, Nk, p, seed, offset)
            O[b, :, h, :] = (P * M / (1.0 - p)) @ v[b, :, h // G, :]
            LSE[b, h, :] = lse
    return O, LSE


def attention_bwd_dropout(q, k, v, do, causal: bool, scale: float, p: float, seed: int, offset: int):
    """dQ, dK, dV (fp64) of sum(dO * O) for the dropout forward above (same mask)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Nq, Nk, Hq, Hkv, d = _check_shapes(q, k, v)
    G = Hq // Hkv
    vis = visible_mask(Nq, Nk, causal)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    r = 1.0 / (1.0 - p)
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            S = scores(q[b, :, h, :], k[b, :, hk, :], scale, vis)
            P, _ = softmax_rows(S)
            M = keep_mask(b, h, Hq, Nq, Nk, p, seed, offset)
            Pd = P * M * r
            O = Pd @ v[b, :, hk, :]
            dv[b, :, hk, :] += Pd.T @ do[b, :, h, :]
            dP = M * r * (do[b, :, h, :] @ v[b, :, hk, :].T)
            D = np.sum(do[b, :, h, :] * O, axis=1, keepdims=True)
            dS = P * (dP - D)
            dq[b, :, h, :] = scale * dS @ k[b, :, hk, :]
            dk[b, :, hk, :] += scale * dS.T @ q[b, :, h, :]
    return dq, dk, dv
