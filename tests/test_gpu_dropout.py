"""Parity of the dropout forward/backward (through the C ABI) with the dropout oracle.

The mask itself is compared bit for bit: with Q = 0 and V = I the forward's O
shows which (query, key) pairs were kept; with dO = I the dK/dV kernel's dV
shows the mask it regenerated.  Values: LSE <= 1e-3 and dQ/dK/dV relative L2
<= 2e-2 as for the plain path; O within 1e-2 + 2^-8 |O| per element -- the
kept weights are scaled by 1 / (1 - p), so |O| can pass 4, where the 16-bit
rounding of O alone (half an ulp, up to 2^-8 |O| in bf16) exceeds 1e-2.
"""
import math

import numpy as np
import pytest

import workloads
from oracle import dropout_ref as dr

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL, GRAD_TOL = 1e-2, 1e-3, 2e-2
SEED, OFFSET = 0x0123456789ABCDEF, 3


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_io_aware_80_b200 as m
    from exact_io_aware_80_b200 import _lib
    _lib.load()
    return m


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def test_forward_mask_is_the_oracle_mask(fa):
    Nq, Nk, d, Hq, p = 256, 128, 128, 2, float(np.float32(0.3))
    q = torch.zeros(1, Nq, Hq, d, dtype=torch.bfloat16)
    k = workloads.make_inputs(1, 1, 1, Nk, Nk, d, torch.bfloat16, seed_base=8500)[1]
    v = torch.eye(Nk, d, dtype=torch.bfloat16)[None, :, None, :].contiguous()
    o, _ = fa.attention_fwd_dropout(q.cuda(), k.cuda(), v.cuda(), p, SEED, OFFSET, causal=False)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    og = f64(o)
    for h in range(Hq):
        M = dr.keep_mask(0, h, Hq, Nq, Nk, p, SEED, OFFSET)
        assert np.array_equal(og[0, :, h, :Nk] != 0, M)
        np.testing.assert_allclose(og[0, :, h, :Nk][M], 1.0 / (Nk * (1 - p)), rtol=4e-3)


def test_backward_mask_is_the_oracle_mask(fa):
    # dV = (P * M)^T dO / (1 - p) with dO = I shows the mask the dK/dV kernel regenerates
    N, d, p = 128, 128, float(np.float32(0.25))
    q = torch.zeros(1, N, 1, d, dtype=torch.bfloat16)
    k, v = workloads.make_inputs(1, 1, 1, N, N, d, torch.bfloat16, seed_base=8600)[1:]
    do = torch.eye(N, d, dtype=torch.bfloat16)[None, :, None, :].contiguous()
    o, lse = fa.attention_fwd_dropout(q.cuda(), k.cuda(), v.cuda(), p, SEED, OFFSET)
    dq, dk, dv = fa.attention_bwd_dropout(q.cuda(), k.cuda(), v.cuda(), o, do.cuda(), lse, p, SEED, OFFSET)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    M = dr.keep_mask(0, 0, 1, N, N, p, SEED, OFFSET)
    assert np.array_equal(f64(dv)[0, :, 0, :N] != 0, M.T)


CASES = [
    # B, Hq, Hkv, N, d, dtype, causal, p
    (2, 4, 2, 333, 128, torch.bfloat16, True, 0.25),
    (1, 4, 1, 300, 128, torch.bfloat16, False, 0.1),
    (1, 2, 2, 200, 64, torch.float16, True, 0.5),
]


@pytest.mark.parametrize("case", CASES)
def test_forward_backward_values(fa, case):
    B, Hq, Hkv, N, d, dt, causal, p = case
    p = float(np.float32(p))
    q, k, v, do = workloads.make_inputs(B, Hq, Hkv, N, N, d, dt, seed_base=8700 + N, with_do=True)
    o, lse = fa.attention_fwd_dropout(q.cuda(), k.cuda(), v.cuda(), p, SEED, OFFSET, causal=causal)
    dq, dk, dv = fa.attention_bwd_dropout(q.cuda(), k.cuda(), v.cuda(), o, do.cuda(), lse, p, SEED, OFFSET,
                                          causal=causal)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    scale = 1 / math.sqrt(d)
    O, L = dr.attention_fwd_dropout(f64(q), f64(k), f64(v), causal, scale, p, SEED, OFFSET)
    assert np.all(np.abs(f64(o) - O) <= O_TOL + 2.0 ** -8 * np.abs(O))
    assert np.max(np.abs(lse.cpu().numpy() - L)) <= LSE_TOL
    DQ, DK, DV = dr.attention_bwd_dropout(f64(q), f64(k), f64(v), f64(do), causal, scale, p, SEED, OFFSET)
    for g, G in ((dq, DQ), (dk, DK), (dv, DV)):
        assert rel_l2(f64(g), G) <= GRAD_TOL


def test_p_zero_equals_plain_path(fa):
    q, k, v, do = workloads.make_inputs(1, 4, 2, 260, 260, 128, torch.bfloat16, seed_base=8800, with_do=True)
    q, k, v, do = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o1, l1 = fa.attention_fwd_dropout(q, k, v, 0.0, SEED, 0, causal=True)
    o2, l2 = fa.attention_fwd(q, k, v, True)
    g1 = fa.attention_bwd_dropout(q, k, v, o1, do, l1, 0.0, SEED, 0, causal=True)
    g2 = fa.attention_bwd(q, k, v, o2, do, l2, True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
