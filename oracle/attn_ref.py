"""Plain, slow, fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  This module is imported by ``tests/``, by
``__graft_entry__.smoke()`` and by the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` -- nothing else.  The product path (the CUDA library and
its Python binding) never imports, links or executes it, and this module never
imports the product package.  It shares no code, table or constant with the
CUDA kernels.

Sources (page title, section):

* "FlashAttention 심층 분석" (ryotta.opik.net), section 1 ("문제 -- 표준 어텐션은
  메모리 바운드"): standard attention is S = Q K^T, P = softmax(S), O = P V with
  the N x N matrices materialised.  That plain definition is what this oracle
  computes, because the pages state that the tiled method returns exactly the
  same result ("FlashAttention-2 (KO)", lead paragraph; "FlashAttention 심층
  분석", section 3, third bullet).
* same page, section 2 (memory hierarchy): the fused steps are scaling,
  masking, softmax, dropout and the PV product.  Scaling and causal masking are
  applied here; dropout probability is zero (the Qwen3-4B shape in the
  smithlab guide, "학습할 때 어텐션 메모리, 길이별 계산", has
  attention_dropout 0.0).
* same page, section 3 (tiling + online softmax), the online recurrence with
  running max m and running sum l: ``attention_fwd_online`` follows it step by
  step, with the scale and the mask added.
* same page, section 4 (recomputation) and the smithlab guide's memory table:
  one fp32 log-sum-exp per query row is what the forward pass keeps.
* same page, "Flash-Decoding": one-token decode splits the key axis, computes
  partial attention per split and merges them by log-sum-exp
  (``decode_splitkv`` / ``decode_combine``).
* smithlab guide, "FlashAttention 도입 체크리스트": causal is a flag and GQA is
  expressed by the KV-head count, with no K/V replication.

Readings where the pages are silent:

* layout BSHD: q, o, do, dq are [B, Nq, Hq, d]; k, v, dk, dv are
  [B, Nk, Hkv, d]; lse is [B, Hq, Nq];
* S includes ``scale`` and LSE is taken over the scaled scores, in natural log;
* causal keeps key j for query i iff j <= i + (Nk - Nq) (bottom-right);
* a row with no visible key has O = 0 and LSE = -inf;
* GQA groups are contiguous: h_kv = h_q // (Hq // Hkv);
* the backward pass is the chain rule of the definition (the pages give no
  equations for it): dV = P^T dO, dP = dO V^T, D_i = sum_j P_ij dP_ij
  (= sum_c dO_ic O_ic), dS = P * (dP - D), dQ = scale dS K, dK = scale dS^T Q,
  with dK and dV summed over the query heads of a group.

Every function takes numpy-convertible arrays, upcasts them exactly to fp64 and
returns fp64.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "visible_mask",
    "scores",
    "softmax_rows",
    "attention_fwd",
    "attention_fwd_rows",
    "attention_fwd_online",
    "attention_bwd",
    "attention_bwd_dq_rows",
    "attention_bwd_kv_rows",
    "bwd_preprocess",
    "decode",
    "decode_splitkv",
    "decode_combine",
    "attention_flops",
    "lse_bytes",
    "eager_softmax_bytes",
    "brute_force_attention",
    "attention_bwd_partial",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def visible_mask(Nq: int, Nk: int, causal: bool) -> np.ndarray:
    """Boolean [Nq, Nk]: True where query i may attend to key j.

    Causal masking is applied before the softmax ("FlashAttention 심층 분석",
    section 2, the masking step).  Reading: bottom-right alignment,
    j <= i + (Nk - Nq); for Nq == Nk this is the lower triangle.
    """
    if not causal:
        return np.ones((Nq, Nk), dtype=bool)
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    return j <= i + (Nk - Nq)


def scores(q_h: np.ndarray, k_h: np.ndarray, scale: float, mask: np.ndarray) -> np.ndarray:
    """S = scale * Q K^T for one head, masked entries set to -inf.

    q_h: [Nq, d], k_h: [Nk, d] ("FlashAttention 심층 분석", section 1).
    """
    S = scale * (_f64(q_h) @ _f64(k_h).T)
    return np.where(mask, S, -np.inf)


def softmax_rows(S: np.ndarray):
    """Two-pass row softmax of a materialised score matrix.

    Returns (P, LSE) where P = exp(S - m) / sum exp(S - m), m the row max and
    LSE = m + ln sum_j exp(S_ij - m).  Rows that are entirely -inf give P = 0
    and LSE = -inf (reading: such a row attends to nothing).
    """
    m = np.max(S, axis=-1, keepdims=True)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    E = np.exp(S - m_safe)  # exp(-inf) = 0 for masked entries
    l = np.sum(E, axis=-1, keepdims=True)
    l_safe = np.where(empty, 1.0, l)
    P = np.where(empty, 0.0, E / l_safe)
    LSE = np.where(empty, -np.inf, m_safe + np.log(l_safe))
    return P, LSE[..., 0]


def _check_shapes(q, k, v):
    B, Nq, Hq, d = q.shape
    Bk, Nk, Hkv, dk = k.shape
    if v.shape != k.shape or Bk != B or dk != d:
        raise ValueError("q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d] expected")
    if Hkv < 1 or Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return B, Nq, Nk, Hq, Hkv, d


def attention_fwd(q, k, v, causal: bool, scale: float, heads=None):
    """Exact attention forward: O [B, Nq, Hq, d] and LSE [B, Hq, Nq] in fp64.

    For every (b, h_q) it materialises S and P, then O = P V.  ``heads``
    optionally restricts the work to a list of (b, h_q) pairs; outputs for the
    other heads are left as NaN (used to sample large workloads).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Nk, Hq, Hkv, d = _check_shapes(q, k, v)
    G = Hq // Hkv
    mask = visible_mask(Nq, Nk, causal)
    O = np.full((B, Nq, Hq, d), np.nan)
    LSE = np.full((B, Hq, Nq), np.nan)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in todo:
        hk = h // G
        S = scores(q[b, :, h, :], k[b, :, hk, :], scale, mask)
        P, lse = softmax_rows(S)
        O[b, :, h, :] = P @ v[b, :, hk, :]
        LSE[b, h, :] = lse
    return O, LSE


def attention_fwd_rows(q, k, v, causal: bool, scale: float, b: int, h: int, rows):
    """O and LSE for selected query rows of one (b, h_q): ([len(rows), d], [len(rows)])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Nk, Hq, Hkv, d = _check_shapes(q, k, v)
    hk = h // (Hq // Hkv)
    rows = np.asarray(rows, dtype=np.int64)
    mask = visible_mask(Nq, Nk, causal)[rows]
    S = scores(q[b, rows, h, :], k[b, :, hk, :], scale, mask)
    P, lse = softmax_rows(S)
    return P @ v[b, :, hk, :], lse


def attention_fwd_online(q, k, v, causal: bool, scale: float, block: int):
    """The tiled online-softmax recurrence, in the pages' order and notation.

    "FlashAttention 심층 분석", section 3: for a fixed query block, walk the key
    blocks j, and per row keep m (running max), l (running sum) and O:
      m_new = max(m, rowmax(S_ij)); P_ij = exp(S_ij - m_new);
      l = exp(m - m_new) l + rowsum(P_ij); O = exp(m - m_new) O + P_ij V_j;
      m = m_new;  after the last block O = O / l.
    Added here: the scale on S and the causal mask.  Reading for a row whose
    visible keys have not started yet (m_new = -inf): the correction factor is
    taken as 0 and P as 0, so no NaN appears.  The query block is the whole
    row range (the recurrence is per row, so the query blocking does not
    change any value).  Returns O and LSE = m + ln l.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Nk, Hq, Hkv, d = _check_shapes(q, k, v)
    G = Hq // Hkv
    mask = visible_mask(Nq, Nk, causal)
    O_all = np.zeros((B, Nq, Hq, d))
    LSE_all = np.zeros((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            Q_i = q[b, :, h, :]
            m = np.full((Nq, 1), -np.inf)
            l = np.zeros((Nq, 1))
            O = np.zeros((Nq, d))
            for j0 in range(0, Nk, block):
                K_j = k[b, j0:j0 + block, hk, :]
                V_j = v[b, j0:j0 + block, hk, :]
                S_ij = np.where(mask[:, j0:j0 + block], scale * (Q_i @ K_j.T), -np.inf)
                m_new = np.maximum(m, np.max(S_ij, axis=1, keepdims=True))
                alive = np.isfinite(m_new)
                m_new_safe = np.where(alive, m_new, 0.0)
                P_ij = np.where(alive, np.exp(S_ij - m_new_safe), 0.0)
                corr = np.where(alive, np.exp(np.where(np.isfinite(m), m, -np.inf) - m_new_safe), 0.0)
                l = corr * l + np.sum(P_ij, axis=1, keepdims=True)
                O = corr * O + P_ij @ V_j
                m = m_new
            live = l[:, 0] > 0
            O_all[b, :, h, :] = np.where(live[:, None], O / np.where(l > 0, l, 1.0), 0.0)
            LSE_all[b, h, :] = np.where(live, m[:, 0] + np.log(np.where(l[:, 0] > 0, l[:, 0], 1.0)), -np.inf)
    return O_all, LSE_all


def bwd_preprocess(o, do):
    """D[b, h, i] = sum_c dO[b, i, h, c] * O[b, i, h, c]  ([B, Hq, Nq], fp64).

    Reading (the pages give no backward equations): this is the row term of the
    softmax Jacobian, equal to sum_j P_ij dP_ij.
    """
    o, do = _f64(o), _f64(do)
    return np.einsum("bihc,bihc->bhi", do, o)


def attention_bwd(q, k, v, do, causal: bool, scale: float, kv_heads=None):
    """Gradients of L = sum(dO * O) w.r.t. Q, K, V, from the chain rule.

    The pages say only that the backward pass recomputes S and P from the
    stored statistics ("FlashAttention 심층 분석", section 4); the equations are
    the plain derivative of the definition:
      P = softmax(S), S = scale Q K^T (masked), O = P V,
      dV = P^T dO,  dP = dO V^T,  D_i = sum_j P_ij dP_ij,
      dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q,
    with dK, dV of a KV head summed over its group of query heads.
    ``kv_heads`` optionally restricts the work to a list of (b, h_kv) pairs
    (their query heads' dQ and their own dK, dV); the rest stays NaN.
    Returns (dQ, dK, dV) in fp64.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Nq, Nk, Hq, Hkv, d = _check_shapes(q, k, v)
    G = Hq // Hkv
    mask = visible_mask(Nq, Nk, causal)
    dq = np.full_like(q, np.nan)
    dk = np.full_like(k, np.nan)
    dv = np.full_like(v, np.nan)
    todo = kv_heads if kv_heads is not None else [(b, hk) for b in range(B) for hk in range(Hkv)]
    for b, hk in todo:
        K = k[b, :, hk, :]
        V = v[b, :, hk, :]
        dK = np.zeros((Nk, d))
        dV = np.zeros((Nk, d))
        for h in range(hk * G, (hk + 1) * G):
            Q = q[b, :, h, :]
            dO = do[b, :, h, :]
            P, _ = softmax_rows(scores(Q, K, scale, mask))
            dV += P.T @ dO
            dP = dO @ V.T
            D = np.sum(P * dP, axis=1, keepdims=True)
            dS = P * (dP - D)
            dq[b, :, h, :] = scale * (dS @ K)
            dK += scale * (dS.T @ Q)
        dk[b, :, hk, :] = dK
        dv[b, :, hk, :] = dV
    return dq, dk, dv


def attention_bwd_dq_rows(q, k, v, do, causal: bool, scale: float, b: int, h: int, rows):
    """dQ for selected query rows of one (b, h_q), row by row.

    Every quantity dQ_i needs is a function of row i alone: its scores S_i,
    its softmax P_i, O_i = P_i V, D_i = dO_i . O_i, dP_i = dO_i V^T,
    dS_i = P_i (dP_i - D_i) and dQ_i = scale dS_i K.  Returns [len(rows), d].
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Nq, Nk, Hq, Hkv, d = _check_shapes(q, k, v)
    hk = h // (Hq // Hkv)
    rows = np.asarray(rows, dtype=np.int64)
    K, V = k[b, :, hk, :], v[b, :, hk, :]
    P, _ = softmax_rows(scores(q[b, rows, h, :], K, scale, visible_mask(Nq, Nk, causal)[rows]))
    dO = do[b, rows, h, :]
    O = P @ V
    D = np.sum(dO * O, axis=1, keepdims=True)
    dS = P * (dO @ V.T - D)
    return scale * (dS @ K)


def attention_bwd_kv_rows(q, k, v, do, causal: bool, scale: float, b: int, hk: int, keys, row_chunk: int = 1024):
    """dK and dV for selected key rows j of one (b, h_kv).

    dK_j = scale sum_{h in group} sum_i dS_ij Q_i and dV_j = sum_h sum_i P_ij dO_i
    need column j of P and dS for every query row i; each row's softmax still
    needs its whole score row, so the query rows are visited in chunks of
    ``row_chunk`` (to bound memory), each chunk evaluated exactly as in
    ``attention_bwd``.  Returns ([len(keys), d], [len(keys), d]).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Nq, Nk, Hq, Hkv, d = _check_shapes(q, k, v)
    G = Hq // Hkv
    keys = np.asarray(keys, dtype=np.int64)
    K, V = k[b, :, hk, :], v[b, :, hk, :]
    mask = visible_mask(Nq, Nk, causal)
    dK = np.zeros((len(keys), d))
    dV = np.zeros((len(keys), d))
    for h in range(hk * G, (hk + 1) * G):
        for i0 in range(0, Nq, row_chunk):
            rows = slice(i0, min(i0 + row_chunk, Nq))
            Q, dO = q[b, rows, h, :], do[b, rows, h, :]
            P, _ = softmax_rows(scores(Q, K, scale, mask[rows]))
            D = np.sum(dO * (P @ V), axis=1, keepdims=True)
            Pj = P[:, keys]
            dSj = Pj * (dO @ V[keys].T - D)
            dV += Pj.T @ dO
            dK += scale * (dSj.T @ Q)
    return dK, dV


def decode(q, k_cache, v_cache, seqlens_k, scale: float):
    """One-token decode: attention of q [B, 1, Hq, d] over the first seqlens_k[b]
    keys of a padded cache [B, Nk_max, Hkv, d].  Non-causal (the single query is
    the last position).  Returns O [B, 1, Hq, d] and LSE [B, Hq, 1]."""
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    B, Nq, Hq, d = q.shape
    if Nq != 1:
        raise ValueError("decode takes one query token")
    O = np.zeros((B, 1, Hq, d))
    LSE = np.zeros((B, Hq, 1))
    for b in range(B):
        n = int(seqlens_k[b])
        if n == 0:
            LSE[b] = -np.inf
            continue
        o, lse = attention_fwd(q[b:b + 1], kc[b:b + 1, :n], vc[b:b + 1, :n], False, scale)
        O[b] = o[0]
        LSE[b] = lse[0]
    return O, LSE


def decode_splitkv(q, k_cache, v_cache, seqlens_k, scale: float, chunk: int, num_splits: int):
    """Flash-Decoding partials ("FlashAttention 심층 분석", Flash-Decoding).

    Split s of sequence b covers keys [s*chunk, min((s+1)*chunk, seqlens_k[b])).
    Per split: O_s = softmax(S_s) V_s over that range and LSE_s = ln sum exp(S_s)
    (an empty split gives O_s = 0, LSE_s = -inf).
    Returns O_part [B, Hq, num_splits, d] and LSE_part [B, Hq, num_splits].
    """
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    B, _, Hq, d = q.shape
    O_part = np.zeros((B, Hq, num_splits, d))
    LSE_part = np.full((B, Hq, num_splits), -np.inf)
    for b in range(B):
        n = int(seqlens_k[b])
        for s in range(num_splits):
            lo, hi = s * chunk, min((s + 1) * chunk, n)
            if hi <= lo:
                continue
            o, lse = attention_fwd(q[b:b + 1], kc[b:b + 1, lo:hi], vc[b:b + 1, lo:hi], False, scale)
            O_part[b, :, s, :] = o[0, 0]
            LSE_part[b, :, s] = lse[0, :, 0]
    return O_part, LSE_part


def decode_combine(O_part, LSE_part):
    """Log-sum-exp reduction of split partials ("FlashAttention 심층 분석",
    Flash-Decoding): LSE = ln sum_s exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s.
    Returns O [B, 1, Hq, d] and LSE [B, Hq, 1]."""
    O_part, LSE_part = _f64(O_part), _f64(LSE_part)
    mx = np.max(LSE_part, axis=-1, keepdims=True)
    empty = ~np.isfinite(mx)
    mx_safe = np.where(empty, 0.0, mx)
    w = np.exp(LSE_part - mx_safe)
    tot = np.sum(w, axis=-1, keepdims=True)
    lse = np.where(empty, -np.inf, mx_safe + np.log(np.where(empty, 1.0, tot)))
    wn = np.where(empty, 0.0, w / np.where(empty, 1.0, tot))
    O = np.einsum("bhs,bhsd->bhd", wn, O_part)
    return O[:, None, :, :], lse


def attention_bwd_partial(q, k, v, do, lse, dvec, causal: bool, scale: float):
    """Gradient contributions of one block of keys, given the full rows' LSE and D.

    With P = exp(scale Q K^T - LSE) (the probabilities of the whole row, restricted
    to these keys), dP = dO V^T and dS = P * (dP - D): dQ_part = scale dS K,
    dK = scale dS^T Q, dV = P^T dO (dK, dV summed over the query heads of a
    group).  Summing the parts over a partition of the keys gives the full
    backward (the chain rule is linear in the keys once LSE and D are fixed);
    used for context-parallel (ring) attention.  ``lse``, ``dvec``: [B, Hq, Nq].
    Returns (dQ_part, dK, dV).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    lse, dvec = _f64(lse), _f64(dvec)
    B, Nq, Nk, Hq, Hkv, d = _check_shapes(q, k, v)
    G = Hq // Hkv
    mask = visible_mask(Nq, Nk, causal)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            S = scores(q[b, :, h, :], k[b, :, hk, :], scale, mask)
            P = np.exp(S - lse[b, h][:, None])
            dP = do[b, :, h, :] @ v[b, :, hk, :].T
            dS = P * (dP - dvec[b, h][:, None])
            dq[b, :, h, :] = scale * dS @ k[b, :, hk, :]
            dk[b, :, hk, :] += scale * dS.T @ q[b, :, h, :]
            dv[b, :, hk, :] += P.T @ do[b, :, h, :]
    return dq, dk, dv


def attention_flops(B: int, Hq: int, Nq: int, Nk: int, d: int, causal: bool, backward: bool = False) -> float:
    """Nominal attention FLOPs.

    Forward: 4 B Hq Nq Nk d (two matmuls of 2 FLOPs per multiply-add), halved
    when causal -- for Nq = Nk = N that is 2 N Hq d per token, the smithlab
    guide's causal-forward figure ("어텐션 연산량과 학습 비용 비교").  Backward:
    2.5 x forward, the same guide's convention (recomputation included).
    """
    f = 4.0 * B * Hq * Nq * Nk * d
    if causal:
        f *= 0.5
    return f * 2.5 if backward else f


def lse_bytes(B: int, Hq: int, Nq: int, layers: int = 1) -> int:
    """Bytes of the per-row fp32 log-sum-exp kept for the backward pass
    (smithlab guide, memory table: one fp32 value per row and head)."""
    return B * Hq * Nq * 4 * layers


def eager_softmax_bytes(B: int, Hq: int, Nq: int, Nk: int, layers: int = 1) -> int:
    """Bytes an eager implementation keeps per score for backward: the fp32
    softmax output (4 B) plus the bf16 probabilities fed to the PV matmul (2 B)
    (smithlab guide, memory table)."""
    return B * Hq * Nq * Nk * 6 * layers



def brute_force_attention(q, k, v, causal: bool, scale: float):
    """Pure-Python loops (math.exp, math.fsum) over tiny inputs, for pinning.

    Independent of numpy's reductions: every score, weight and output is a
    scalar expression.  Returns nested lists O[b][i][h][c] and LSE[b][h][i].
    """
    B, Nq, Hq, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Nk, Hkv = len(k[0]), len(k[0][0])
    G = Hq // Hkv
    O = [[[[0.0] * d for _ in range(Hq)] for _ in range(Nq)] for _ in range(B)]
    LSE = [[[0.0] * Nq for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            for i in range(Nq):
                vis = [j for j in range(Nk) if (not causal) or j <= i + (Nk - Nq)]
                if not vis:
                    LSE[b][h][i] = -math.inf
                    continue
                s = {j: scale * math.fsum(float(q[b][i][h][c]) * float(k[b][j][hk][c]) for c in range(d)) for j in vis}
                mx = max(s.values())
                w = {j: math.exp(s[j] - mx) for j in vis}
                tot = math.fsum(w.values())
                LSE[b][h][i] = mx + math.log(tot)
                for c in range(d):
                    O[b][i][h][c] = math.fsum(w[j] * float(v[b][j][hk][c]) for j in vis) / tot
    return O, LSE
