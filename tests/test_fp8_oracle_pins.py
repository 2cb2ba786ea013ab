"""Pins for the FP8 forward oracle (oracle/fp8_ref.py), on the CPU.

Each check ties the oracle to something other than itself: the E4M3 format
definition and an independent library codec (torch.float8_e4m3fn), the
Sylvester-Hadamard matrix from scipy, exact arithmetic on integer inputs, the
16-bit attention oracle on inputs the quantizer represents exactly, and a CPU
emulation of the P rounding that the error bound covers.  Planted mistakes
(a missing rotation of K, a wrong 1/d, a transposed V) fail at least one pin.
"""
import math

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import attn_ref as ref
from oracle import fp8_ref as f8


# ----------------------------------------------------------------------------- E4M3 codec
def test_e4m3_decode_matches_library_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = f8.e4m3_decode(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    nan = np.isnan(ours)
    assert list(np.flatnonzero(nan)) == [0x7F, 0xFF]
    assert np.isnan(lib[nan]).all()
    assert np.array_equal(ours[~nan], lib[~nan])


def test_e4m3_values_from_the_format_definition():
    # sign | 4-bit exponent (bias 7) | 3-bit mantissa; subnormals m * 2^-9
    assert f8.e4m3_decode(np.uint8(0x01)) == 2.0 ** -9
    assert f8.e4m3_decode(np.uint8(0x07)) == 7 * 2.0 ** -9
    assert f8.e4m3_decode(np.uint8(0x08)) == 2.0 ** -6
    assert f8.e4m3_decode(np.uint8(0x38)) == 1.0
    assert f8.e4m3_decode(np.uint8(0x7E)) == 448.0
    assert f8.e4m3_decode(np.uint8(0xB8)) == -1.0


def test_e4m3_round_trip_and_monotone():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = f8.e4m3_decode(codes)
    assert np.array_equal(f8.e4m3_encode(vals.astype(np.float32)), codes)
    pos = np.sort(vals[vals > 0])
    assert np.all(np.diff(pos) > 0) and pos[-1] == 448.0


def test_e4m3_encode_matches_library_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000) * 40, rng.standard_normal(100000) * 0.01,
                        rng.uniform(-448, 448, 50000)]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(f8.e4m3_encode(x), lib)


def test_e4m3_ties_to_even_and_saturation():
    enc = lambda v: int(f8.e4m3_encode(np.float32(v)))  # noqa: E731
    assert enc(2.0 ** -10) == 0x00          # halfway 0 .. 2^-9 -> even (0)
    assert enc(3 * 2.0 ** -10) == 0x02      # halfway 2^-9 .. 2^-8 -> even (2 * 2^-9)
    assert enc(1.0625) == 0x38              # halfway 1 .. 1.125 -> 1
    assert enc(1.1875) == 0x3A              # halfway 1.125 .. 1.25 -> 1.25
    for big in (449.0, 464.0, 480.0, 1e6, 3e38):
        assert enc(big) == 0x7E and enc(-big) == 0xFE
    assert enc(-0.0) == 0x80 and enc(-1e-4) == 0x80


# ----------------------------------------------------------------------------- rotation
def test_fwht_equals_hadamard_matrix_on_exact_inputs():
    rng = np.random.default_rng(1)
    for d in (64, 128):
        x = rng.integers(-16, 16, (7, d)).astype(np.float32)
        want = x.astype(np.float64) @ scipy.linalg.hadamard(d)
        assert np.array_equal(f8.fwht_f32(x).astype(np.float64), want)


def test_rotation_scales_inner_products_by_d():
    rng = np.random.default_rng(2)
    d = 128
    signs = rng.choice([-1.0, 1.0], d)
    x = rng.integers(-8, 8, (5, d)).astype(np.float32)
    y = rng.integers(-8, 8, (6, d)).astype(np.float32)
    rx, ry = f8.rotate_f32(x, signs).astype(np.float64), f8.rotate_f32(y, signs).astype(np.float64)
    assert np.array_equal(rx @ ry.T, d * (x.astype(np.float64) @ y.T.astype(np.float64)))


# ----------------------------------------------------------------------------- quantizers
def test_quantize_qk_scales_and_error_bound():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 300, 3, 64)).astype(np.float32)
    codes, scales = f8.quantize_qk(x)
    assert scales.shape == (2, 3, 3)
    for b in range(2):
        for h in range(3):
            for j in range(3):
                blk = x[b, 128 * j:128 * (j + 1), h, :]
                assert scales[b, h, j] == np.float32(np.max(np.abs(blk)) / np.float32(448.0))
                mags = codes[b, 128 * j:128 * (j + 1), h, :] & 0x7F
                assert mags.max() == 0x7E  # the block maximum maps to 448
    xhat = f8.dequantize_qk(codes, scales)
    s = np.repeat(scales.astype(np.float64), 128, axis=2)[:, :, :300].transpose(0, 2, 1)[..., None]
    y = x / s
    bound = s * np.where(np.abs(y) >= 2.0 ** -6, 2.0 ** -4 * np.abs(y), 2.0 ** -10)
    assert np.all(np.abs(xhat - x) <= bound * (1 + 1e-6))


def test_quantize_v_layout_and_padding():
    rng = np.random.default_rng(4)
    v = rng.standard_normal((1, 37, 2, 64)).astype(np.float32)
    codes, scales = f8.quantize_v(v)
    assert codes.shape == (1, 2, 64, 48) and np.all(codes[..., 37:] == 0)
    for h in range(2):
        assert scales[0, h] == np.float32(np.max(np.abs(v[0, :, h, :])) / np.float32(448.0))
        assert np.array_equal(codes[0, h, :, :37], f8.e4m3_encode(v[0, :, h, :] / scales[0, h]).T)
    vhat = f8.dequantize_v(codes, scales, 37)
    assert vhat.shape == v.shape and np.max(np.abs(vhat - v)) <= 2.0 ** -4 * np.max(np.abs(v))


# ----------------------------------------------------------------------------- attention
def _representable(rng, shape):
    """Values that E4M3 holds exactly, with the block maximum 448 so that every scale is 1."""
    codes = rng.integers(0, 0x7E, shape).astype(np.uint8) | (rng.integers(0, 2, shape).astype(np.uint8) << 7)
    x = f8.e4m3_decode(codes).astype(np.float32)
    x[:, ::128, :, 0] = 448.0
    return x


@pytest.mark.parametrize("causal", [False, True])
def test_attention_on_representable_inputs_equals_16bit_oracle(causal):
    rng = np.random.default_rng(5)
    q = _representable(rng, (1, 150, 2, 64)) / 64
    k = _representable(rng, (1, 150, 1, 64)) / 64
    v = _representable(rng, (1, 150, 1, 64))
    q8, qs = f8.quantize_qk(q)
    k8, ks = f8.quantize_qk(k)
    v8, vs = f8.quantize_v(v)
    O, L = f8.attention_fp8_ref(q8, qs, k8, ks, v8, vs, 150, causal, 0.125, rotated=False)
    O2, L2 = ref.attention_fwd(q, k, v, causal, 0.125)
    np.testing.assert_allclose(O, O2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(L, L2, rtol=1e-12, atol=1e-12)


def _fp8_error(q, k, v, causal, scale, signs):
    q8, qs = f8.quantize_qk(q, signs)
    k8, ks = f8.quantize_qk(k, signs)
    v8, vs = f8.quantize_v(v)
    O, _ = f8.attention_fp8_ref(q8, qs, k8, ks, v8, vs, k.shape[1], causal, scale, rotated=signs is not None)
    O0, _ = ref.attention_fwd(q, k, v, causal, scale)
    return np.sqrt(np.mean((O - O0) ** 2)) / np.sqrt(np.mean(O0 ** 2))


def test_rotated_scores_keep_attention_close():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 256, 2, 128)).astype(np.float32)
    k = rng.standard_normal((1, 256, 1, 128)).astype(np.float32)
    v = rng.standard_normal((1, 256, 1, 128)).astype(np.float32)
    signs = rng.choice([-1.0, 1.0], 128)
    assert _fp8_error(q, k, v, True, 128 ** -0.5, signs) < 0.08


def test_incoherent_processing_lowers_error_with_outlier_channels():
    # the FA-3 claim the pages repeat: rotating Q and K before FP8 lowers the error
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 256, 2, 128)).astype(np.float32)
    k = rng.standard_normal((1, 256, 1, 128)).astype(np.float32)
    v = rng.standard_normal((1, 256, 1, 128)).astype(np.float32)
    q[..., :4] *= 30
    k[..., :4] *= 30
    scale = 1.0 / (30 * math.sqrt(128))
    signs = rng.choice([-1.0, 1.0], 128)
    plain = _fp8_error(q, k, v, False, scale, None)
    rot = _fp8_error(q, k, v, False, scale, signs)
    assert rot < plain / 1.5, (rot, plain)


def test_planted_mistakes_are_caught():
    rng = np.random.default_rng(8)
    # 64 keys and d = 64, so that a transposed V still has a valid shape
    q = rng.standard_normal((1, 64, 1, 64)).astype(np.float32)
    k = rng.standard_normal((1, 64, 1, 64)).astype(np.float32)
    v = rng.standard_normal((1, 64, 1, 64)).astype(np.float32)
    signs = rng.choice([-1.0, 1.0], 64)
    O0, _ = ref.attention_fwd(q, k, v, False, 0.125)
    q8, qs = f8.quantize_qk(q, signs)
    k8, ks = f8.quantize_qk(k, signs)
    k8p, ksp = f8.quantize_qk(k)  # K not rotated
    v8, vs = f8.quantize_v(v)
    good, _ = f8.attention_fp8_ref(q8, qs, k8, ks, v8, vs, 64, False, 0.125, rotated=True)
    no_rot, _ = f8.attention_fp8_ref(q8, qs, k8p, ksp, v8, vs, 64, False, 0.125, rotated=True)
    no_div, _ = f8.attention_fp8_ref(q8, qs, k8, ks, v8, vs, 64, False, 0.125, rotated=False)
    v_t, _ = f8.attention_fp8_ref(q8, qs, k8, ks, v8.transpose(0, 1, 3, 2).copy(), vs, 64, False, 0.125, rotated=True)
    err = lambda O: np.max(np.abs(O - O0))  # noqa: E731
    assert err(good) < 0.1
    assert err(no_rot) > 0.3 and err(no_div) > 0.3 and err(v_t) > 0.3


def test_p_rounding_bound_covers_an_emulated_rounding():
    """Round P to E4M3 on the CPU at two reference maxima; the bound must cover both."""
    rng = np.random.default_rng(9)
    q = rng.standard_normal((1, 200, 1, 64)).astype(np.float32) * 2
    k = rng.standard_normal((1, 200, 1, 64)).astype(np.float32)
    v = rng.standard_normal((1, 200, 1, 64)).astype(np.float32)
    q8, qs = f8.quantize_qk(q)
    k8, ks = f8.quantize_qk(k)
    v8, vs = f8.quantize_v(v)
    rows = np.arange(0, 200, 7)
    bound = f8.p_rounding_bound(q8, qs, k8, ks, v8, vs, 200, True, 0.125, False, 0, 0, rows)
    O, _ = f8.attention_fp8_ref(q8, qs, k8, ks, v8, vs, 200, True, 0.125, rotated=False)
    qd, kd, vd = f8.dequantize_qk(q8, qs), f8.dequantize_qk(k8, ks), f8.dequantize_v(v8, vs, 200)
    S = 0.125 * qd[0, rows, 0, :] @ kd[0, :, 0, :].T
    S = np.where(np.arange(200)[None, :] <= rows[:, None], S, -np.inf)
    for lift in (0.0, 3.0):  # reference max at the row max, or 3 (log2 units) below it
        m = S.max(axis=1, keepdims=True) / math.log(2) - lift
        p = np.exp2(S / math.log(2) - m)
        p8 = f8.e4m3_decode(f8.e4m3_encode(p.astype(np.float32)))
        Oe = (p8 @ vd[0, :, 0, :]) / p.sum(axis=1, keepdims=True)
        dev = np.abs(Oe - O[0, rows, 0, :])
        assert np.all(dev <= bound * (1 + 1e-9) + 1e-12)
        assert dev.max() > 0  # the rounding is visible
