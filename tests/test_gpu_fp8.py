"""Parity of the FP8 forward path (through the C ABI) with the FP8 oracle.

* Quantizers: E4M3 codes and fp32 scales must equal the oracle's bit for bit
  (a quantised code is an integer decision; both sides take it in fp32 with the
  same division and butterfly order).
* Attention: the oracle computes exact attention of the dequantized operands;
  the GPU also rounds P to E4M3 for the P V product.  Every element must lie
  within the oracle's per-element bound for that rounding
  (oracle.fp8_ref.p_rounding_bound) plus 2^-8 |O| (16-bit output rounding, the
  polynomial exp2 and fp32 accumulation) plus 2e-3.  LSE does not see the P
  rounding (l sums the unrounded p): max-abs <= 1e-3 as in the 16-bit path.
"""
import math

import numpy as np
import pytest

import workloads
from oracle import fp8_ref as f8

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

LSE_TOL = 1e-3


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_io_aware_80_b200 as m
    from exact_io_aware_80_b200 import _lib
    _lib.load()
    return m


def npf(t):
    return t.detach().float().cpu().numpy()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("rotate", [False, True])
def test_quantize_qk_bit_exact(fa, d, rotate):
    x = workloads.make_inputs(2, 3, 3, 300, 300, d, torch.bfloat16, seed_base=7100)[0]
    signs = workloads.rotation_signs(d, 7199) if rotate else None
    x8, sc = fa.fp8_quantize_qk(x.cuda(), None if signs is None else signs.cuda())
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    c_ref, s_ref = f8.quantize_qk(npf(x), None if signs is None else npf(signs))
    assert np.array_equal(sc.cpu().numpy(), s_ref)
    assert np.array_equal(x8.cpu().numpy(), c_ref)


@pytest.mark.parametrize("Nk", [1, 37, 300, 1024])
def test_quantize_v_bit_exact(fa, Nk):
    v = workloads.make_inputs(1, 2, 2, Nk, Nk, 128, torch.float16, seed_base=7200)[2]
    v8t, sc = fa.fp8_quantize_v(v.cuda())
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    c_ref, s_ref = f8.quantize_v(npf(v))
    assert np.array_equal(sc.cpu().numpy(), s_ref)
    assert np.array_equal(v8t.cpu().numpy(), c_ref)


@pytest.mark.parametrize("d,dt,rotate,Nq,Nk", [(128, torch.bfloat16, True, 300, 1000), (64, torch.float16, False, 77, 129),
                                               (128, torch.float16, False, 1, 16), (64, torch.bfloat16, True, 513, 257)])
def test_quantize_qkv_fused_bit_exact(fa, d, dt, rotate, Nq, Nk):
    """The fused Q+K+V quantizer gives the oracle's codes and scales bit for bit."""
    q, k, v = workloads.make_inputs(2, 4, 2, Nq, Nk, d, dt, seed_base=7250 + Nq)
    signs = workloads.rotation_signs(d, 7299) if rotate else None
    q8, qs, k8, ks, v8t, vs = fa.fp8_quantize_qkv(q.cuda(), k.cuda(), v.cuda(), None if signs is None else signs.cuda())
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    sg = None if signs is None else npf(signs)
    for got, gs, ref in ((q8, qs, f8.quantize_qk(npf(q), sg)), (k8, ks, f8.quantize_qk(npf(k), sg)),
                         (v8t, vs, f8.quantize_v(npf(v)))):
        assert np.array_equal(gs.cpu().numpy(), ref[1])
        assert np.array_equal(got.cpu().numpy(), ref[0])


def check_fwd(fa, q, k, v, causal, rotate, heads_rows, seed, out_dtype=torch.bfloat16):
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d)
    signs = workloads.rotation_signs(d, seed) if rotate else None
    # GPU: quantize and attend
    q8, qs = fa.fp8_quantize_qk(q.cuda(), None if signs is None else signs.cuda())
    k8, ks = fa.fp8_quantize_qk(k.cuda(), None if signs is None else signs.cuda())
    v8t, vs = fa.fp8_quantize_v(v.cuda())
    o, lse = fa.attention_fwd_fp8(q8, qs, k8, ks, v8t, vs, k.shape[1], causal, scale, rotate, out_dtype)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    # oracle: its own quantization of the same inputs
    sg = None if signs is None else npf(signs)
    rq, rqs = f8.quantize_qk(npf(q), sg)
    rk, rks = f8.quantize_qk(npf(k), sg)
    rv, rvs = f8.quantize_v(npf(v))
    assert np.array_equal(q8.cpu().numpy(), rq) and np.array_equal(k8.cpu().numpy(), rk)
    assert np.array_equal(v8t.cpu().numpy(), rv)
    heads = sorted({(b, h) for b, h, _ in heads_rows})
    O, L = f8.attention_fp8_ref(rq, rqs, rk, rks, rv, rvs, k.shape[1], causal, scale, rotate, heads=heads)
    og, lg = npf(o).astype(np.float64), lse.cpu().numpy().astype(np.float64)
    worst = 0.0
    for b, h, rows in heads_rows:
        rows = np.asarray(rows)
        bound = f8.p_rounding_bound(rq, rqs, rk, rks, rv, rvs, k.shape[1], causal, scale, rotate, b, h, rows)
        ref = O[b, rows, h, :]
        dev = np.abs(og[b, rows, h, :] - ref)
        lim = bound + 2.0 ** -8 * np.abs(ref) + 2e-3
        assert np.all(dev <= lim), f"(b={b}, h={h}) worst excess {np.max(dev - lim):.3e}"
        worst = max(worst, float(np.max(dev / lim)))
        assert np.max(np.abs(lg[b, h, rows] - L[b, h, rows])) <= LSE_TOL
    return worst


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("rotate", [False, True])
def test_fwd_fp8_small(fa, causal, rotate):
    B, Hq, Hkv, N = 2, 4, 2, 333
    q, k, v = workloads.make_inputs(B, Hq, Hkv, N, N, 128, torch.bfloat16, seed_base=7300)
    hr = [(b, h, np.arange(N)) for b in range(B) for h in range(Hq)]
    check_fwd(fa, q, k, v, causal, rotate, hr, 7399)


def test_fwd_fp8_ragged_fp16_out(fa):
    q, k, v = workloads.make_inputs(1, 2, 1, 130, 461, 128, torch.float16, seed_base=7400)
    hr = [(0, h, np.arange(130)) for h in range(2)]
    check_fwd(fa, q, k, v, False, True, hr, 7499, out_dtype=torch.float16)


def test_fwd_fp8_gqa_training_shape_sampled(fa):
    # the GQA training-step shape (B1 Hq32 Hkv8 N8192 d128 causal), sampled rows of two heads
    w = workloads.get(3)
    q, k, v = workloads.workload_inputs(w, with_do=False, device="cuda")
    rows = np.unique(np.concatenate([np.arange(0, 8192, 61), [0, 1, 127, 128, 8191]]))
    hr = [(0, 0, rows), (0, 29, rows)]
    check_fwd(fa, q, k, v, True, True, hr, 7599)
