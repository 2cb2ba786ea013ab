"""Parity of the dropout forward/backward (through the C ABI) with the dropout oracle.

The mask itself is compared bit for bit, in each of the three kernels that
applies it.  With Q = 0 every visible score is 0, so every unnormalised weight
is exactly 1; inputs built from unit vectors then expose the mask: the
forward's O (V rows = unit vectors), the dQ kernel's dQ (K rows = unit
vectors, dP = 1, D = 0) and the dK/dV kernel's dV (dO rows = unit vectors).
Scaling the unit vectors of different key (or query) tiles by distinct powers
of two packs several tiles into one output element as an integer code whose
bits are the keep bits, read back exactly after the 16-bit rounding.

Values: LSE <= 1e-3 and dQ/dK/dV relative L2 <= 2e-2 as for the plain path;
O within 1e-2 + 2^-8 |O| per element -- the kept weights are scaled by
1 / (1 - p), so |O| can pass 4, where the bf16 rounding of O alone (half an
ulp, up to 2^-8 |O|) exceeds 1e-2.
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


# ---------------------------------------------------------------------------
# the mask at larger sizes: every kernel's regenerated mask, bit for bit
# ---------------------------------------------------------------------------

def _unit_rows(n_rows, d, tiles, n_tiles_total, H, dtype):
    """[1, n_rows, H, d]: row 128 T + c = 2^(T - tiles[0]) e_c for T in ``tiles``, zero elsewhere."""
    x = torch.zeros(1, n_rows, H, d, dtype=torch.float32)
    for T in tiles:
        r = torch.arange(128 * T, min(128 * T + 128, n_rows))
        x[0, r, :, r - 128 * T] = float(2 ** (T - tiles[0]))
    return x.to(dtype)


def _decode_bits(code, tiles):
    """Integer codes -> {tile: boolean array} of their bits."""
    return {T: ((code >> (T - tiles[0])) & 1).astype(bool) for T in tiles}


@pytest.mark.parametrize("causal", [False, True])
def test_forward_mask_persistent_many_work_tiles(fa, causal):
    """320 work tiles of 256 rows on 148 CTAs, so each CTA runs the persistent loop two or
    three times with dropout on; O exposes the mask of four key tiles per call."""
    B, Hq, Hkv, N, d, p = 2, 40, 8, 1024, 128, 0.5
    q = torch.zeros(B, N, Hq, d, dtype=torch.bfloat16).cuda()
    k = workloads.make_inputs(B, Hkv, Hkv, N, N, d, torch.bfloat16, seed_base=8900)[1].cuda()
    heads = [(0, 0), (0, 17), (0, 39), (1, 5), (1, 22), (1, 39)]
    masks = {bh: dr.keep_mask(bh[0], bh[1], Hq, N, N, p, SEED, OFFSET) for bh in heads}
    i = np.arange(N)[:, None]
    nvis = (i + 1) if causal else np.full((N, 1), N)
    for tiles in ([0, 1, 2, 3], [4, 5, 6, 7]):
        v = _unit_rows(N, d, tiles, 8, Hkv, torch.bfloat16).expand(B, N, Hkv, d).contiguous().cuda()
        o, _ = fa.attention_fwd_dropout(q, k, v, p, SEED, OFFSET, causal=causal)
        torch.cuda.synchronize()
        assert fa.device_status() == 0
        og = f64(o)
        for (b, h), M in masks.items():
            code = np.rint(og[b, :, h, :] * nvis * (1 - p)).astype(np.int64)  # [N, 128]: keys 128 T + c
            bits = _decode_bits(code, tiles)
            for T in tiles:
                j = np.arange(128 * T, 128 * T + 128)[None, :]
                want = M[:, 128 * T:128 * T + 128] & ((j <= i) if causal else True)
                assert np.array_equal(bits[T], want), (b, h, T)


@pytest.mark.parametrize("causal", [False, True])
def test_dq_kernel_mask_is_the_oracle_mask(fa, causal):
    """dQ = scale dS K with Q = 0, dP = dO V^T = 1 and D = 0 (o passed as zeros):
    dS = P M / (1 - p), so with K rows = scaled unit vectors each dQ element is an
    integer code of the keep bits of up to four key tiles (five tiles, ragged tail)."""
    B, Hq, Hkv, N, d, p = 1, 4, 2, 600, 128, 0.5
    scale = 1 / math.sqrt(d)
    q = torch.zeros(B, N, Hq, d, dtype=torch.bfloat16).cuda()
    e0q = torch.zeros(B, N, Hq, d, dtype=torch.bfloat16)
    e0q[..., 0] = 1
    e0k = torch.zeros(B, N, Hkv, d, dtype=torch.bfloat16)
    e0k[..., 0] = 1
    do, v = e0q.cuda(), e0k.cuda()
    o0 = torch.zeros_like(q)
    masks = {h: dr.keep_mask(0, h, Hq, N, N, p, SEED, OFFSET) for h in range(Hq)}
    i = np.arange(N)[:, None]
    nvis = (i + 1) if causal else np.full((N, 1), N)
    for tiles in ([0, 1, 2, 3], [4]):
        k = _unit_rows(N, d, tiles, 5, Hkv, torch.bfloat16).cuda()
        _, lse = fa.attention_fwd(q, k, v, causal)  # Q = 0: LSE = ln(visible keys), whatever K is
        dq, _, _ = fa.attention_bwd_dropout(q, k, v, o0, do, lse, p, SEED, OFFSET, causal=causal)
        torch.cuda.synchronize()
        assert fa.device_status() == 0
        g = f64(dq)
        for h, M in masks.items():
            code = np.rint(g[0, :, h, :] * nvis * (1 - p) / scale).astype(np.int64)
            bits = _decode_bits(code, tiles)
            for T in tiles:
                w = min(128, N - 128 * T)
                j = np.arange(128 * T, 128 * T + w)[None, :]
                want = M[:, 128 * T:128 * T + w] & ((j <= i) if causal else True)
                assert np.array_equal(bits[T][:, :w], want), (h, T)
                assert not bits[T][:, w:].any()


def test_dkdv_kernel_mask_over_group_and_query_tiles(fa):
    """G = 4 query heads x 3 query tiles = 12 tiles per dK/dV CTA (the keep-bit ring wraps six
    times): dO rows of one head's tile = scaled unit vectors make each dV element an integer
    code of the keep bits of up to four (head, query tile) pairs."""
    B, Hq, Hkv, N, d, p = 1, 4, 1, 300, 128, 0.5
    q = torch.zeros(B, N, Hq, d, dtype=torch.bfloat16).cuda()
    k, v = workloads.make_inputs(B, Hkv, Hkv, N, N, d, torch.bfloat16, seed_base=9000)[1:]
    k, v = k.cuda(), v.cuda()
    o, lse = fa.attention_fwd_dropout(q, k, v, p, SEED, OFFSET)
    masks = {h: dr.keep_mask(0, h, Hq, N, N, p, SEED, OFFSET) for h in range(Hq)}
    pairs = [(h, S) for h in range(Hq) for S in range(3)]
    for c0 in range(0, len(pairs), 4):
        group = pairs[c0:c0 + 4]
        do = torch.zeros(B, N, Hq, d, dtype=torch.float32)
        for n, (h, S) in enumerate(group):
            r = torch.arange(128 * S, min(128 * S + 128, N))
            do[0, r, h, r - 128 * S] = float(2 ** n)
        _, _, dv = fa.attention_bwd_dropout(q, k, v, o, do.to(torch.bfloat16).cuda(), lse, p, SEED, OFFSET)
        torch.cuda.synchronize()
        assert fa.device_status() == 0
        code = np.rint(f64(dv)[0, :, 0, :] * N * (1 - p)).astype(np.int64)  # [keys, c]
        for n, (h, S) in enumerate(group):
            w = min(128, N - 128 * S)
            got = ((code[:, :w] >> n) & 1).astype(bool)  # [key j, query 128 S + c]
            assert np.array_equal(got, masks[h][128 * S:128 * S + w, :].T), (h, S)


# ---------------------------------------------------------------------------
# the configuration the bench times
# ---------------------------------------------------------------------------

@pytest.mark.slow
def test_gqa_training_shape_values_against_oracle(fa):
    """B=1, Hq=32, Hkv=8, N=8192, d=128, causal, p=0.1 -- the dropout step the bench
    times (1024 forward work tiles on 148 CTAs): whole heads 0, 13 and 31 for O and
    LSE, whole KV groups 0 and 7 for dK, dV and their query heads' dQ."""
    w = workloads.get(3)
    p = float(np.float32(0.1))
    q, k, v, do = workloads.workload_inputs(w)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.attention_fwd_dropout(qd, kd, vd, p, SEED, OFFSET, causal=True)
    dq, dk, dv = fa.attention_bwd_dropout(qd, kd, vd, o, dod, lse, p, SEED, OFFSET, causal=True)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    qn, kn, vn, don = f64(q), f64(k), f64(v), f64(do)
    og, lg = f64(o), lse.cpu().numpy()
    heads = [(0, 0), (0, 13), (0, 31)]
    O, L = dr.attention_fwd_dropout(qn, kn, vn, True, w.scale, p, SEED, OFFSET, heads=heads)
    for b, h in heads:
        assert np.all(np.abs(og[b, :, h] - O[b, :, h]) <= O_TOL + 2.0 ** -8 * np.abs(O[b, :, h])), h
        assert np.max(np.abs(lg[b, h] - L[b, h])) <= LSE_TOL, h
    dqg, dkg, dvg = f64(dq), f64(dk), f64(dv)
    for hk in (0, 7):
        DQ, DK, DV = dr.attention_bwd_dropout(qn, kn, vn, don, True, w.scale, p, SEED, OFFSET, kv_heads=[(0, hk)])
        hs = slice(4 * hk, 4 * hk + 4)
        assert rel_l2(dqg[0, :, hs], DQ[0, :, hs]) <= GRAD_TOL, hk
        assert rel_l2(dkg[0, :, hk], DK[0, :, hk]) <= GRAD_TOL, hk
        assert rel_l2(dvg[0, :, hk], DV[0, :, hk]) <= GRAD_TOL, hk
