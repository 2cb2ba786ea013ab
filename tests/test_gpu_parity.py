"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tolerances: O max-abs <= 1e-2, LSE max-abs <= 1e-3, dQ/dK/dV relative L2
<= 2e-2.  Small cases compare every element; the full-size workloads compare
whole heads / sequences / rows sampled from the launch the bench times.
"""
import math

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL, GRAD_TOL = 1e-2, 1e-3, 2e-2


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


def dtype_of(name):
    return torch.float16 if name == "fp16" else torch.bfloat16


def run_fwd(fa, q, k, v, causal):
    o, lse = fa.attention_fwd(q.cuda(), k.cuda(), v.cuda(), causal)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return f64(o), lse.cpu().numpy().astype(np.float64)


SMALL_FWD = [
    # B, Hq, Hkv, Nq, Nk, d, dtype, causal
    (1, 2, 2, 128, 128, 64, "fp16", False),
    (1, 2, 2, 128, 128, 64, "fp16", True),
    (2, 4, 2, 300, 451, 128, "bf16", False),
    (2, 4, 2, 333, 333, 128, "bf16", True),
    (1, 4, 1, 200, 333, 64, "fp16", True),
    (1, 2, 2, 1, 1, 128, "bf16", False),
    (1, 2, 2, 1, 1, 128, "bf16", True),
    (1, 2, 1, 1, 77, 64, "bf16", True),
    (3, 6, 3, 65, 129, 128, "fp16", False),
    (1, 8, 2, 257, 257, 128, "bf16", True),
    (1, 2, 1, 512, 1000, 128, "fp16", True),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,dt,causal", SMALL_FWD)
def test_fwd_small(fa, B, Hq, Hkv, Nq, Nk, d, dt, causal):
    q, k, v = workloads.make_inputs(B, Hq, Hkv, Nq, Nk, d, dtype_of(dt), seed_base=7 * Nq + Nk)
    o, lse = run_fwd(fa, q, k, v, causal)
    O, L = oracle.attention_fwd(f64(q), f64(k), f64(v), causal, 1 / math.sqrt(d))
    assert np.abs(o - O).max() <= O_TOL
    assert np.abs(lse - L).max() <= LSE_TOL


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_tiny_workload(fa, causal):
    w = workloads.get(1)
    q, k, v = workloads.workload_inputs(w)
    o, lse = run_fwd(fa, q, k, v, causal)
    O, L = oracle.attention_fwd(f64(q), f64(k), f64(v), causal, w.scale)
    assert np.abs(o - O).max() <= O_TOL
    assert np.abs(lse - L).max() <= LSE_TOL


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_mha_prefill_full(fa, causal):
    """B=4, H=16, N=2048, d=128 bf16: every element against the oracle."""
    w = workloads.get(2)
    q, k, v = workloads.workload_inputs(w)
    o, lse = run_fwd(fa, q, k, v, causal)
    O, L = oracle.attention_fwd(f64(q), f64(k), f64(v), causal, w.scale)
    assert np.abs(o - O).max() <= O_TOL
    assert np.abs(lse - L).max() <= LSE_TOL


def _sampled_fwd(fa, wid, heads):
    w = workloads.get(wid)
    q, k, v = workloads.workload_inputs(w, with_do=False)
    o, lse = run_fwd(fa, q, k, v, True)
    qn, kn, vn = f64(q), f64(k), f64(v)
    for b, h in heads:
        O, L = oracle.attention_fwd(qn[b:b + 1], kn[b:b + 1], vn[b:b + 1], True, w.scale, heads=[(0, h)])
        assert np.abs(o[b, :, h] - O[0, :, h]).max() <= O_TOL, (b, h)
        assert np.abs(lse[b, h] - L[0, h]).max() <= LSE_TOL, (b, h)


def test_fwd_gqa_training_sampled_heads(fa):
    """B=1, Hq=32, Hkv=8, N=8192 causal: whole heads 0, 13 and 31 (three KV groups)."""
    _sampled_fwd(fa, 3, [(0, 0), (0, 13), (0, 31)])


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------

def run_bwd(fa, q, k, v, do, causal):
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.attention_fwd(qd, kd, vd, causal)
    dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, dod, lse, causal)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return f64(dq), f64(dk), f64(dv)


SMALL_BWD = [
    (1, 2, 2, 128, 128, 64, "fp16", False),
    (1, 2, 2, 128, 128, 64, "fp16", True),
    (2, 4, 2, 300, 451, 128, "bf16", False),
    (1, 4, 2, 333, 333, 128, "bf16", True),
    (1, 4, 1, 200, 333, 64, "fp16", True),
    (1, 2, 1, 1, 77, 128, "bf16", True),
    (2, 8, 2, 257, 257, 128, "bf16", True),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,dt,causal", SMALL_BWD)
def test_bwd_small(fa, B, Hq, Hkv, Nq, Nk, d, dt, causal):
    q, k, v, do = workloads.make_inputs(B, Hq, Hkv, Nq, Nk, d, dtype_of(dt), seed_base=11 * Nq + Nk, with_do=True)
    dq, dk, dv = run_bwd(fa, q, k, v, do, causal)
    DQ, DK, DV = oracle.attention_bwd(f64(q), f64(k), f64(v), f64(do), causal, 1 / math.sqrt(d))
    assert rel_l2(dq, DQ) <= GRAD_TOL
    assert rel_l2(dk, DK) <= GRAD_TOL
    assert rel_l2(dv, DV) <= GRAD_TOL


@pytest.mark.parametrize("B,H,N,d,dt", [(2, 3, 333, 128, "bf16"), (1, 5, 77, 64, "fp16"), (3, 2, 1, 128, "fp16"),
                                         (1, 32, 8192, 128, "bf16")])
def test_bwd_preprocess_rowsum(fa, B, H, N, d, dt):
    """D = rowsum(dO * O) from fa_bwd_preprocess against the oracle's definition.  The
    kernel sums d exact products in fp32, so |error| <= d * 2^-24 * sum_c |dO_c O_c|
    (the recursive-summation bound; 2^-23 leaves a factor 2 of margin)."""
    from exact_io_aware_80_b200 import _lib
    o, _, _, do = workloads.make_inputs(B, H, H, N, N, d, dtype_of(dt), seed_base=31 * N + d, with_do=True)
    od, dod = o.cuda(), do.cuda()
    ws = torch.full((B * H * N,), float("nan"), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    _lib.fa_bwd_preprocess(0, 0, 0, od.data_ptr(), dod.data_ptr(), 0, 0, 0, 0, ws.data_ptr(), B, H, H, N, N, d, 0,
                           1.0, _lib.FA_BF16 if dt == "bf16" else _lib.FA_FP16, stream)
    torch.cuda.synchronize()
    Dref = oracle.bwd_preprocess(f64(o), f64(do))
    Dg = ws.view(B, H, N).cpu().numpy().astype(np.float64)
    Sabs = np.einsum("bihc,bihc->bhi", np.abs(f64(do)), np.abs(f64(o)))
    assert np.all(np.abs(Dg - Dref) <= d * 2.0 ** -23 * Sabs)


def test_bwd_gqa_training_sampled_groups(fa):
    """B=1, Hq=32, Hkv=8, N=8192 causal: KV groups 0 and 7 (their dK, dV and the
    dQ of their 4 query heads each) against the oracle."""
    w = workloads.get(3)
    q, k, v, do = workloads.workload_inputs(w)
    dq, dk, dv = run_bwd(fa, q, k, v, do, True)
    qn, kn, vn, don = f64(q), f64(k), f64(v), f64(do)
    for hk in (0, 7):
        DQ, DK, DV = oracle.attention_bwd(qn, kn, vn, don, True, w.scale, kv_heads=[(0, hk)])
        hs = slice(4 * hk, 4 * hk + 4)
        assert rel_l2(dq[0, :, hs], DQ[0, :, hs]) <= GRAD_TOL
        assert rel_l2(dk[0, :, hk], DK[0, :, hk]) <= GRAD_TOL
        assert rel_l2(dv[0, :, hk], DV[0, :, hk]) <= GRAD_TOL


@pytest.mark.slow
def test_long_context_sampled_rows_and_memory(fa):
    """B=1, Hq=32, Hkv=8, N=16384 causal: forward rows and backward rows sampled
    across the sequence, and the peak allocation stays O(N) (no N x N buffer)."""
    w = workloads.get(4)
    q, k, v, do = workloads.workload_inputs(w)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.attention_fwd(qd, kd, vd, True)
    dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, dod, lse, True)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    peak = torch.cuda.max_memory_allocated() - base
    assert peak < 2**30, f"peak {peak / 2**20:.0f} MiB"
    qn, kn, vn, don = f64(q), f64(k), f64(v), f64(do)
    o64, lse64, dq64, dk64, dv64 = f64(o), lse.cpu().numpy(), f64(dq), f64(dk), f64(dv)
    rows = [0, 1, 127, 128, 4095, 8191, 12000, 16383]
    for h in (0, 17, 31):
        Or, Lr = oracle.attention_fwd_rows(qn, kn, vn, True, w.scale, 0, h, rows)
        assert np.abs(o64[0, rows, h] - Or).max() <= O_TOL
        assert np.abs(lse64[0, h, rows] - Lr).max() <= LSE_TOL
        dQr = oracle.attention_bwd_dq_rows(qn, kn, vn, don, True, w.scale, 0, h, rows)
        assert rel_l2(dq64[0, rows, h], dQr) <= GRAD_TOL
    keys = [0, 1, 5000, 16383]
    dKr, dVr = oracle.attention_bwd_kv_rows(qn, kn, vn, don, True, w.scale, 0, 3, keys)
    assert rel_l2(dk64[0, keys, 3], dKr) <= GRAD_TOL
    assert rel_l2(dv64[0, keys, 3], dVr) <= GRAD_TOL


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------

def run_decode(fa, q, kc, vc, sl, num_splits=None):
    o, lse = fa.decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), num_splits)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return f64(o), lse.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("splits", [1, 3, 8, None])
def test_decode_small(fa, splits):
    B, Hq, Hkv, N, d = 5, 8, 2, 1000, 128
    q, kc, vc, _ = workloads.make_decode_inputs(B, Hq, Hkv, N, d, torch.bfloat16, seed_base=77)
    sl = torch.tensor([1000, 1, 500, 0, 999], dtype=torch.int32)
    o, lse = run_decode(fa, q, kc, vc, sl, splits)
    O, L = oracle.decode(f64(q), f64(kc), f64(vc), sl.numpy(), 1 / math.sqrt(d))
    assert np.abs(o - O).max() <= O_TOL
    fin = np.isfinite(L)
    assert (np.isfinite(lse) == fin).all()
    assert np.abs(lse[fin] - L[fin]).max() <= LSE_TOL
    assert (o[3] == 0).all()


@pytest.mark.parametrize("G,d,dt", [(1, 64, "fp16"), (4, 64, "bf16"), (8, 128, "fp16"), (16, 128, "bf16")])
def test_decode_group_sizes(fa, G, d, dt):
    B, Hkv, N = 3, 2, 777
    q, kc, vc, sl = workloads.make_decode_inputs(B, G * Hkv, Hkv, N, d, dtype_of(dt), seed_base=5 * G + d, lo=100)
    o, lse = run_decode(fa, q, kc, vc, sl, 4)
    O, L = oracle.decode(f64(q), f64(kc), f64(vc), sl.numpy(), 1 / math.sqrt(d))
    assert np.abs(o - O).max() <= O_TOL
    assert np.abs(lse - L).max() <= LSE_TOL


def test_decode_partials_match_oracle_splits(fa):
    """The split pass itself (before the combine) against the oracle's partials."""
    B, Hq, Hkv, N, d = 2, 4, 1, 640, 128
    q, kc, vc, _ = workloads.make_decode_inputs(B, Hq, Hkv, N, d, torch.bfloat16, seed_base=99)
    sl = torch.tensor([640, 300], dtype=torch.int32)
    S = 4
    chunk = fa.fa_decode_chunk(N, S)
    ws = fa.decode_splitkv(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), S)
    torch.cuda.synchronize()
    part = ws.view(torch.float32)
    Op = part[:B * Hq * S * d].view(B, Hq, S, d).cpu().numpy()
    Lp = part[B * Hq * S * d:B * Hq * S * d + B * Hq * S].view(B, Hq, S).cpu().numpy()
    Oo, Lo = oracle.decode_splitkv(f64(q), f64(kc), f64(vc), sl.numpy(), 1 / math.sqrt(d), chunk, S)
    assert np.abs(Op - Oo).max() <= O_TOL
    fin = np.isfinite(Lo)
    assert (np.isfinite(Lp) == fin).all()
    assert np.abs(Lp[fin] - Lo[fin]).max() <= LSE_TOL


def test_decode_full_workload_sampled_sequences(fa):
    """B=64, Hq=32, Hkv=8, Nk_max=32768, d=128 bf16, ragged second half: the
    bench's launch (default split count), sequences sampled from both halves."""
    w = workloads.get(5)
    q, kc, vc, sl = workloads.workload_inputs(w, device="cuda")
    sld = sl.cuda()
    o, lse = fa.decode(q, kc, vc, sld)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    o64, lse64 = f64(o), lse.cpu().numpy()
    for b in (0, 31, 32, 47, 63):
        n = int(sl[b])
        O, L = oracle.decode(f64(q[b:b + 1]), f64(kc[b:b + 1, :n]), f64(vc[b:b + 1, :n]), [n], w.scale)
        assert np.abs(o64[b] - O[0]).max() <= O_TOL, b
        assert np.abs(lse64[b] - L[0]).max() <= LSE_TOL, b


# ---------------------------------------------------------------------------
# determinism and the status word
# ---------------------------------------------------------------------------

def test_bitwise_determinism(fa):
    q, k, v, do = workloads.make_inputs(1, 8, 2, 700, 700, 128, torch.bfloat16, seed_base=3, with_do=True)
    q, k, v, do = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    outs = []
    for _ in range(2):
        o, lse = fa.attention_fwd(q, k, v, True)
        dq, dk, dv = fa.attention_bwd(q, k, v, o, do, lse, True)
        outs.append([t.clone() for t in (o, lse, dq, dk, dv)])
    torch.cuda.synchronize()
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    qd, kc, vc, sl = workloads.make_decode_inputs(4, 8, 2, 3000, 128, torch.bfloat16, seed_base=4)
    r1 = fa.decode(qd.cuda(), kc.cuda(), vc.cuda(), sl.cuda())
    r2 = fa.decode(qd.cuda(), kc.cuda(), vc.cuda(), sl.cuda())
    assert torch.equal(r1[0], r2[0]) and torch.equal(r1[1], r2[1])
    assert fa.device_status() == 0


def test_one_call_backward_equals_separate_launches_and_orders_the_stream(fa):
    """Inside fa_bwd the dQ kernel is a programmatic dependent of dK/dV (it may start while dK/dV
    runs).  Its gradients must equal those of the three entry points called one at a time, and
    work enqueued on the stream right after fa_bwd must see every gradient complete: the sums
    taken there, before any host synchronisation, must equal the sums of the final tensors."""
    from exact_io_aware_80_b200 import _lib
    B, Hq, Hkv, N, d = 1, 16, 4, 4096, 128  # dK/dV: 128 CTAs; dQ: 512 CTAs
    q, k, v, do = [t.cuda() for t in workloads.make_inputs(B, Hq, Hkv, N, N, d, torch.bfloat16, seed_base=51,
                                                           with_do=True)]
    o, lse = fa.attention_fwd(q, k, v, True)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, Hq, N), device="cuda", dtype=torch.uint8)
    grads = [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]
    st = torch.cuda.current_stream().cuda_stream
    args = [t.data_ptr() for t in (q, k, v, o, do, lse, *grads, ws)] + [B, Hq, Hkv, N, N, d, 1, 1.0 / math.sqrt(d),
                                                                       _lib.FA_BF16, st]
    _lib.fa_bwd_preprocess(*args)
    _lib.fa_bwd_dkdv(*args)
    _lib.fa_bwd_dq(*args)
    torch.cuda.synchronize()
    ref = [g.clone() for g in grads]
    sums = []
    for _ in range(12):
        for g in grads:
            g.zero_()
        _lib.fa_bwd(*args)
        sums.append([g.float().sum() for g in grads])  # enqueued behind fa_bwd, no host sync
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    for g, r in zip(grads, ref):
        assert torch.equal(g, r)
    final = [g.float().sum() for g in grads]
    for s3 in sums:
        for a, b in zip(s3, final):
            assert torch.equal(a, b)


def test_watchdog_times_out_cleanly_and_context_survives(fa):
    """A bounded wait on a barrier nothing arrives on reports FA_ERR_TIMEOUT
    through the status word (no trap, no hang), which then reads clean again,
    and the next attention call works."""
    from exact_io_aware_80_b200 import _lib
    stream = torch.cuda.current_stream().cuda_stream
    assert fa.device_status() == 0
    _lib.fa_watchdog_selftest(20000, stream)  # 20 ms limit
    assert fa.device_status() == _lib.FA_ERR_TIMEOUT
    assert fa.device_status() == 0
    q, k, v = workloads.make_inputs(1, 2, 2, 200, 200, 128, torch.bfloat16, seed_base=9)
    o, lse = run_fwd(fa, q, k, v, True)
    O, L = oracle.attention_fwd(f64(q), f64(k), f64(v), True, 1 / math.sqrt(128))
    assert np.abs(o - O).max() <= O_TOL
