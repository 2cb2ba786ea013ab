"""Parity of the block-sparse forward (through the C ABI) with its oracle.

Same tolerances as the dense forward (O max-abs <= 1e-2, LSE max-abs <= 1e-3);
rows with no visible key must be exactly O = 0 and LSE = -inf.
"""
import math

import numpy as np
import pytest

import workloads
from oracle import sparse_ref as sp

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 1e-2, 1e-3


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


def run(fa, q, k, v, bm, causal, heads=None):
    o, lse = fa.attention_fwd_blocksparse(q.cuda(), k.cuda(), v.cuda(), bm.cuda(), causal)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    O, L = sp.attention_fwd_blocksparse(f64(q), f64(k), f64(v), bm.numpy(), causal, 1 / math.sqrt(q.shape[-1]),
                                        heads=heads)
    og, lg = f64(o), lse.cpu().numpy().astype(np.float64)
    todo = heads or [(b, h) for b in range(q.shape[0]) for h in range(q.shape[2])]
    for b, h in todo:
        ref, got = O[b, :, h, :], og[b, :, h, :]
        empty = ~np.isfinite(L[b, h])
        assert np.all(got[empty] == 0) and np.all(lg[b, h][empty] == -np.inf)
        assert np.max(np.abs(got - ref)) <= O_TOL, (b, h, np.max(np.abs(got - ref)))
        assert np.max(np.abs(lg[b, h][~empty] - L[b, h][~empty]), initial=0) <= LSE_TOL
    return og


CASES = [
    # B, Hq, Hkv, Nq, Nk, d, dtype, causal, density, seed
    (2, 4, 2, 333, 333, 128, torch.bfloat16, True, 0.5, 1),
    (2, 4, 2, 300, 700, 128, torch.bfloat16, False, 0.4, 2),
    (1, 2, 1, 520, 520, 64, torch.float16, False, 0.3, 3),
    (1, 3, 3, 129, 257, 64, torch.float16, True, 0.6, 4),
]


@pytest.mark.parametrize("case", CASES)
def test_random_masks(fa, case):
    B, Hq, Hkv, Nq, Nk, d, dt, causal, dens, seed = case
    q, k, v = workloads.make_inputs(B, Hq, Hkv, Nq, Nk, d, dt, seed_base=8000 + 10 * seed)
    bm = workloads.block_mask_random(B, Hq, -(-Nq // 128), -(-Nk // 128), dens, 8009 + seed)
    run(fa, q, k, v, bm, causal)


def test_all_ones_matches_dense_kernel(fa):
    q, k, v = workloads.make_inputs(1, 4, 2, 400, 400, 128, torch.bfloat16, seed_base=8100)
    bm = torch.ones(1, 4, 4, 4, dtype=torch.uint8)
    o1, l1 = fa.attention_fwd_blocksparse(q.cuda(), k.cuda(), v.cuda(), bm.cuda(), True)
    o2, l2 = fa.attention_fwd(q.cuda(), k.cuda(), v.cuda(), True)
    torch.cuda.synchronize()
    # the same arithmetic in the same order: bitwise equal
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_empty_rows_and_empty_work_tiles(fa):
    q, k, v = workloads.make_inputs(1, 2, 2, 600, 384, 128, torch.bfloat16, seed_base=8200)
    bm = torch.zeros(1, 2, 5, 3, dtype=torch.uint8)
    bm[0, 0, 0, 1] = 1      # head 0: query block 0 sees key block 1; block 1 (same work tile) sees nothing
    bm[0, 0, 3, 2] = 1      # work tile 1: only its second query tile has a block
    bm[0, 1, 4, :] = 1      # head 1: only the ragged last query block sees anything
    run(fa, q, k, v, bm, False)


def test_local_window_gqa_training_shape_sampled(fa):
    w = workloads.get(3)
    q, k, v = workloads.workload_inputs(w, with_do=False, device="cuda")
    nb = w.Nq // 128
    bm = workloads.block_mask_local(1, w.Hq, nb, nb, window=8, sink=1)
    o, lse = fa.attention_fwd_blocksparse(q, k, v, bm.cuda(), True)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    for h in (0, 17):
        rows = np.unique(np.concatenate([np.arange(0, w.Nq, 97), [0, 127, 128, 1023, 1024, w.Nq - 1]]))
        O, L = sp.attention_fwd_blocksparse_rows(f64(q.cpu()), f64(k.cpu()), f64(v.cpu()), bm.numpy(), True, w.scale,
                                                 0, h, rows)
        assert np.max(np.abs(f64(o[0, rows, h, :].cpu()) - O)) <= O_TOL
        assert np.max(np.abs(lse[0, h, rows].cpu().numpy() - L)) <= LSE_TOL
