"""fa_decode_noalloc: split-KV decode for callers that cannot allocate device
memory (a runtime that forbids allocation on its request path, code inside
another allocator's callback).  It keeps the split partials in a static device
array inside libfa.so instead of a caller workspace, so its output must equal
that of the workspace entry points (fa_decode_splitkv + fa_decode_combine).

Both paths run the same split and combine kernels with the same split count
and chunk, so their outputs must be bitwise equal.  Checked through the C ABI
on two calls in a row with different inputs (a call that read the previous
call's leftovers from the shared array would fail), against the fp64 oracle
within the decode tolerances, and on a request whose suggested split count
does not fit the array, so that the automatic count has to shrink.
This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes
import math

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 1e-2, 1e-3


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_io_aware_80_b200 as fa
    from exact_io_aware_80_b200 import _lib
    return fa, _lib, _lib.load()


def _noalloc(lib, _lib, q, kc, vc, sl, splits, o, lse):
    B, _, Hq, d = q.shape
    _, Nk_max, Hkv, _ = kc.shape
    stream = torch.cuda.current_stream().cuda_stream
    return lib.fa_decode_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), sl.data_ptr(), o.data_ptr(),
                                 lse.data_ptr(), B, Hq, Hkv, Nk_max, d, ctypes.c_float(d ** -0.5), splits,
                                 _lib.FA_BF16, ctypes.c_void_p(stream))


def test_noalloc_decode_matches_workspace_decode_twice(libs):
    fa, _lib, lib = libs
    B, Hq, Hkv, N, d = 6, 16, 4, 3000, 128
    cases = [(601, [3000, 1, 0, 1500, 2999, 64], 5), (602, [17, 3000, 2048, 0, 777, 2500], 0)]
    for seed, lens, splits in cases:
        q, kc, vc, _ = workloads.make_decode_inputs(B, Hq, Hkv, N, d, torch.bfloat16, seed_base=seed, device="cuda")
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        s_ref = splits if splits > 0 else fa.fa_decode_num_splits(B, Hkv, N, d, 0)
        o_ref, lse_ref = fa.decode(q, kc, vc, sl, s_ref)
        o = torch.full((B, 1, Hq, d), 7.0, dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, Hq, 1), 7.0, dtype=torch.float32, device="cuda")
        assert _noalloc(lib, _lib, q, kc, vc, sl, splits, o, lse) == _lib.FA_OK
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref)
        assert torch.equal(torch.isneginf(lse), torch.isneginf(lse_ref))
        fin = torch.isfinite(lse_ref)
        assert torch.equal(lse[fin], lse_ref[fin])
        for b in range(B):
            if lens[b] == 0:
                assert (o[b] == 0).all()
        # and against the oracle, within the decode tolerances
        O, L = oracle.decode(q.float().cpu().numpy().astype(np.float64), kc.float().cpu().numpy().astype(np.float64),
                             vc.float().cpu().numpy().astype(np.float64), lens, 1 / math.sqrt(d))
        assert np.abs(o.float().cpu().numpy() - O).max() <= O_TOL
        lg = lse.cpu().numpy().astype(np.float64)
        fin_o = np.isfinite(L)
        assert (np.isfinite(lg) == fin_o).all()
        assert np.abs(lg[fin_o] - L[fin_o]).max() <= LSE_TOL


def test_noalloc_rejects_partials_beyond_the_scratch_array(libs):
    fa, _lib, lib = libs
    B, Hq, Hkv, N, d = 64, 32, 8, 1024, 128
    need = B * Hq * 16 * d * 4 + B * Hq * 16 * 4  # 16 splits
    assert need > (16 << 20)
    q = torch.zeros(B, 1, Hq, d, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(B, N, Hkv, d, dtype=torch.bfloat16, device="cuda")
    sl = torch.full((B,), N, dtype=torch.int32, device="cuda")
    o = torch.empty(B, 1, Hq, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, 1, dtype=torch.float32, device="cuda")
    assert _noalloc(lib, _lib, q, kc, kc, sl, 16, o, lse) == _lib.FA_ERR_UNSUPPORTED
    # the automatic split count (4 here) fits; with Q = K = V = 0 every key has weight
    # 1/N, so O = 0 and LSE = ln N whatever the split count
    assert _noalloc(lib, _lib, q, kc, kc, sl, 0, o, lse) == _lib.FA_OK
    torch.cuda.synchronize()
    assert (o == 0).all()
    assert (lse - float(torch.log(torch.tensor(float(N))))).abs().max().item() <= LSE_TOL


def _partial_bytes(B, Hq, S, d):
    o = B * Hq * S * d * 4
    return (o + 255) // 256 * 256 + B * Hq * S * 4


def test_noalloc_shrinks_the_automatic_split_count_to_fit(libs):
    """B=16, Hq=16, Hkv=1, Nk=65536: the suggested split count needs more than the
    16 MiB array, so the entry point lowers it until the partials fit; the result
    equals the workspace path's at that lower count, bit for bit."""
    fa, _lib, lib = libs
    B, Hq, Hkv, N, d = 16, 16, 1, 65536, 128
    limit = 16 << 20
    s_sug = fa.fa_decode_num_splits(B, Hkv, N, d, 0)
    assert _partial_bytes(B, Hq, s_sug, d) > limit
    S = s_sug
    while S > 1 and _partial_bytes(B, Hq, S, d) > limit:
        S -= 1
    assert S < s_sug
    q, kc, vc, sl = workloads.make_decode_inputs(B, Hq, Hkv, N, d, torch.bfloat16, seed_base=603, lo=1, device="cuda")
    sld = sl.cuda()
    o_ref, lse_ref = fa.decode(q, kc, vc, sld, S)
    o = torch.full((B, 1, Hq, d), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, Hq, 1), 7.0, dtype=torch.float32, device="cuda")
    assert _noalloc(lib, _lib, q, kc, vc, sld, 0, o, lse) == _lib.FA_OK
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref)
    assert torch.equal(lse, lse_ref)
