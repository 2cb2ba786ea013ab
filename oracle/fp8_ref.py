"""CPU oracle for the FP8 forward pass -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs use
this module; it never imports the CUDA product package and shares no code,
table or constant with it.

Sources (page title, section):

* "FlashAttention 심층 분석" (ryotta.opik.net), section on the FA versions
  ("FP8 지원"): FlashAttention-3 adds an 8-bit floating-point forward pass for
  extra speed.
* "FlashAttention-2 (KO)" (systems-analysis.info), FA-3 paragraph: the FP8
  pass relies on low precision with incoherent processing.
* smithlab guide (tool.smithlab.co.kr), version table: FP8 is forward only;
  and the closing note on exactness: the FP8 forward is low precision, so its
  result is not expected to equal the 16-bit one (the FA-3 paper reports a
  2.6x lower error than a baseline FP8 attention).

The pages name the technique but give no formats, scales or rotation.  The
readings used here:

* 8-bit format: E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
  largest finite 448, subnormals down to 2^-9, no infinities), conversion by
  round-to-nearest-even with saturation to +-448.
* incoherent processing: Q and K rows are multiplied by diag(signs) and then by
  the d x d Sylvester-Hadamard matrix (entries +-1), both in fp32, with the
  butterflies taken in the order h = 1, 2, 4, ..., d/2.  Because H H^T = d I,
  the scores of the rotated operands are d times the original ones; the
  factor 1/d goes into the softmax scale.  ``signs`` is a +-1 vector supplied
  by the caller (the method's random numbers are inputs).
* scales: one fp32 scale per (batch, head, 128-row block) for Q and for K,
  s = amax / 448 (amax = 0 gives s = 1), codes = E4M3(x / s) with the
  division in fp32; one scale per (batch, kv head) for V over all keys.
  V is stored transposed, [B, Hkv, d, Nk_pad] with Nk_pad = Nk rounded up to
  16 and zero codes in the padding.
* attention on the dequantized operands is the exact attention definition;
  the GPU additionally rounds P to E4M3 for the P V product.
  ``p_rounding_bound`` gives a per-element bound on what that rounding can
  change (derivation in its docstring).
"""
from __future__ import annotations

import math

import numpy as np

from .attn_ref import attention_fwd

__all__ = [
    "E4M3_MAX",
    "e4m3_encode",
    "e4m3_decode",
    "fwht_f32",
    "rotate_f32",
    "quantize_qk",
    "quantize_v",
    "dequantize_qk",
    "dequantize_v",
    "attention_fp8_ref",
    "p_rounding_bound",
]

E4M3_MAX = 448.0
_BLOCK = 128


def e4m3_decode(codes) -> np.ndarray:
    """fp64 value of every E4M3 code (NaN for the two NaN codes 0x7F, 0xFF)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(x) -> np.ndarray:
    """E4M3 codes of fp32 values: round to nearest, ties to even, saturate to +-448.

    The representable magnitudes in the binade [2^e, 2^(e+1)) are multiples of
    2^(e-3); below 2^-6 (subnormals) they are multiples of 2^-9.  The value is
    divided by that quantum (exact in fp64), rounded half-to-even, scaled back
    and clamped to 448; the code is then rebuilt from the rounded magnitude.
    The sign bit is kept, also when the magnitude rounds to zero.
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    if np.isnan(x).any():
        raise ValueError("NaN has no saturating E4M3 encoding here")
    sign = np.signbit(x)
    a = np.abs(x)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    q = np.exp2(e - 3.0)
    r = np.rint(a / q) * q  # np.rint: round half to even
    r = np.minimum(r, E4M3_MAX)
    # rebuild the code from the rounded magnitude
    sub = r < 2.0 ** -6
    with np.errstate(divide="ignore"):
        er = np.floor(np.log2(np.where(r > 0, r, 1.0)))
    E = np.where(sub, 0, er + 7).astype(np.int64)
    M = np.where(sub, np.rint(r / 2.0 ** -9), np.rint((r / np.exp2(er) - 1.0) * 8.0)).astype(np.int64)
    code = (E << 3) | M
    return (code | np.where(sign, 0x80, 0)).astype(np.uint8)


def fwht_f32(x) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform along the last axis, in fp32.

    Butterflies (a, b) -> (a + b, a - b) on pairs h apart, for h = 1, 2, 4, ...;
    the result equals x @ H for the Sylvester-Hadamard matrix H up to fp32
    rounding, and exactly when every partial sum is representable.
    """
    y = np.array(x, dtype=np.float32, copy=True)
    d = y.shape[-1]
    if d & (d - 1):
        raise ValueError("length must be a power of two")
    lead = y.shape[:-1]
    h = 1
    while h < d:
        z = y.reshape(*lead, d // (2 * h), 2, h)
        a = z[..., 0, :].copy()
        b = z[..., 1, :].copy()
        z[..., 0, :] = a + b
        z[..., 1, :] = a - b
        y = z.reshape(*lead, d)
        h *= 2
    return y


def rotate_f32(x, signs) -> np.ndarray:
    """fwht_f32(x * signs): the incoherent-processing rotation of rows of x."""
    s = np.asarray(signs, dtype=np.float32)
    if not np.all(np.abs(s) == 1):
        raise ValueError("signs must be +-1")
    return fwht_f32(np.asarray(x, dtype=np.float32) * s)


def quantize_qk(x, signs=None):
    """Block-quantise Q or K ([B, N, H, d], 16-bit values) to E4M3.

    Returns (codes uint8 [B, N, H, d], scales fp32 [B, H, ceil(N / 128)]).
    With ``signs`` the rows are rotated first (rotate_f32).  Per (b, h, block of
    128 rows): amax = max |y| in fp32, s = amax / 448 in fp32 (1 if amax is 0),
    codes = e4m3_encode(y / s) with the division in fp32.
    """
    x = np.asarray(x, dtype=np.float32)
    B, N, H, d = x.shape
    y = rotate_f32(x, signs) if signs is not None else x.copy()
    nb = (N + _BLOCK - 1) // _BLOCK
    codes = np.zeros((B, N, H, d), dtype=np.uint8)
    scales = np.zeros((B, H, nb), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            for j in range(nb):
                blk = y[b, j * _BLOCK:(j + 1) * _BLOCK, h, :]
                amax = np.float32(np.max(np.abs(blk)))
                s = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
                scales[b, h, j] = s
                codes[b, j * _BLOCK:(j + 1) * _BLOCK, h, :] = e4m3_encode(blk / s)
    return codes, scales


def quantize_v(v):
    """Quantise V ([B, Nk, Hkv, d]) with one scale per (b, kv head).

    Returns (codes uint8 [B, Hkv, d, Nk_pad] -- V transposed, Nk_pad = Nk
    rounded up to 16, padding codes 0 -- and scales fp32 [B, Hkv]).
    """
    v = np.asarray(v, dtype=np.float32)
    B, Nk, H, d = v.shape
    npad = (Nk + 15) // 16 * 16
    codes = np.zeros((B, H, d, npad), dtype=np.uint8)
    scales = np.zeros((B, H), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            blk = v[b, :, h, :]
            amax = np.float32(np.max(np.abs(blk)))
            s = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
            scales[b, h] = s
            codes[b, h, :, :Nk] = e4m3_encode(blk / s).T
    return codes, scales


def dequantize_qk(codes, scales) -> np.ndarray:
    """fp64 [B, N, H, d] from block codes and scales."""
    B, N, H, d = codes.shape
    x = e4m3_decode(codes)
    s = np.repeat(np.asarray(scales, dtype=np.float64), _BLOCK, axis=2)[:, :, :N]  # [B, H, N]
    return x * s.transpose(0, 2, 1)[..., None]


def dequantize_v(codes_t, scales, Nk: int) -> np.ndarray:
    """fp64 [B, Nk, Hkv, d] from the transposed codes and per-head scales."""
    x = e4m3_decode(codes_t[..., :Nk])  # [B, H, d, Nk]
    x = x * np.asarray(scales, dtype=np.float64)[:, :, None, None]
    return x.transpose(0, 3, 1, 2)


def attention_fp8_ref(q8, q_scale, k8, k_scale, v8t, v_scale, Nk: int, causal: bool, scale: float,
                      rotated: bool, heads=None):
    """Exact attention (fp64) of the dequantized FP8 operands.

    With ``rotated`` the operands are the rotated Q and K, whose scores are
    d times the original ones, so the softmax scale is scale / d.
    Returns (O [B, Nq, Hq, d], LSE [B, Hq, Nq]).
    """
    q = dequantize_qk(q8, q_scale)
    k = dequantize_qk(k8, k_scale)
    v = dequantize_v(v8t, v_scale, Nk)
    d = q.shape[-1]
    return attention_fwd(q, k, v, causal, scale / d if rotated else scale, heads=heads)


def p_rounding_bound(q8, q_scale, k8, k_scale, v8t, v_scale, Nk: int, causal: bool, scale: float,
                     rotated: bool, b: int, h: int, rows):
    """Per-element bound on |O_gpu - O_ref| caused by rounding P to E4M3.

    The GPU computes p = 2^(t - m_ref) with a reference maximum m_ref that never
    exceeds the row maximum (it is a past running maximum) and stays within 8
    of it, rounds p to E4M3 for the P V product, and divides by l = sum of the
    unrounded p.  With weights normalised to the row maximum (w_j = e^(s_j -
    s_max) <= 1), the GPU's p is w_j 2^(m - m_ref) >= w_j, so an element with
    w_j >= 2^-6 is a normal E4M3 value (relative error <= 2^-4) and any other
    has absolute error <= 2^-10 in GPU units, i.e. <= 2^-10 after normalising;
    l in normalised units is >= 1.  Hence, per output column c,

        |dO_ic| <= (2^-4 sum_j w_ij |V_jc| + 2^-10 sum_{j: w_ij < 2^-6} |V_jc|) / l_i

    with l_i = sum_j w_ij.  Returns that bound, shape [len(rows), d].
    """
    q = dequantize_qk(q8, q_scale)
    k = dequantize_qk(k8, k_scale)
    v = dequantize_v(v8t, v_scale, Nk)
    B, Nq, Hq, d = q.shape
    Hkv = k.shape[2]
    hk = h // (Hq // Hkv)
    sc = scale / d if rotated else scale
    rows = np.asarray(rows, dtype=np.int64)
    S = sc * (q[b, rows, h, :] @ k[b, :, hk, :].T)
    if causal:
        vis = np.arange(Nk)[None, :] <= rows[:, None] + (Nk - Nq)
        S = np.where(vis, S, -np.inf)
    mx = np.max(S, axis=1, keepdims=True)
    w = np.exp(S - np.where(np.isfinite(mx), mx, 0.0))
    l = np.sum(w, axis=1, keepdims=True)
    av = np.abs(v[b, :, hk, :])
    small = (w < 2.0 ** -6) & (w > 0)
    bound = (2.0 ** -4 * (w @ av) + 2.0 ** -10 * (small.astype(np.float64) @ av)) / np.where(l > 0, l, 1.0)
    return bound


def _self_check():  # pragma: no cover - a quick manual smoke
    c = e4m3_encode(np.array([1.0, 448.0, 1000.0, 2.0 ** -9, -0.0], dtype=np.float32))
    assert list(c) == [0x38, 0x7E, 0x7E, 0x01, 0x80], c
    assert math.isclose(float(e4m3_decode(np.uint8(0x7E))), 448.0)
