"""Pins for the fp64 oracle: facts the pages and the mathematics fix.

Each check is a function of the oracle callable it checks, so that the
mutation tests at the bottom can plant a plausible mistake in a copy of the
oracle (on the CPU) and show that at least one pin fails.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(20261202)


def rnd(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def tiny(B=1, Hq=2, Hkv=1, Nq=5, Nk=7, d=4):
    return rnd(B, Nq, Hq, d), rnd(B, Nk, Hkv, d), rnd(B, Nk, Hkv, d)


SHAPES = [
    dict(B=1, Hq=2, Hkv=2, Nq=5, Nk=5, d=4),
    dict(B=2, Hq=4, Hkv=2, Nq=3, Nk=6, d=3),
    dict(B=1, Hq=3, Hkv=1, Nq=6, Nk=6, d=5),
    dict(B=1, Hq=2, Hkv=1, Nq=1, Nk=9, d=4),
]


# ---------------------------------------------------------------------------
# checks (parameterised by the forward / backward callables under test)
# ---------------------------------------------------------------------------

def check_brute_force(fwd):
    """Pure-Python loops (math.fsum) agree with the oracle on tiny inputs."""
    for sh in SHAPES:
        for causal in (False, True):
            q, k, v = tiny(**sh)
            scale = 0.37
            O, L = fwd(q, k, v, causal, scale)
            Ob, Lb = oracle.brute_force_attention(q.tolist(), k.tolist(), v.tolist(), causal, scale)
            np.testing.assert_allclose(O, np.array(Ob), rtol=0, atol=1e-12)
            np.testing.assert_allclose(L, np.array(Lb), rtol=0, atol=1e-12)


def check_constant_v(fwd):
    q, k, v = tiny(Nq=6, Nk=6)
    v[:] = rnd(1, 1, 1, 4)  # the same value row for every key
    for causal in (False, True):
        O, _ = fwd(q, k, v, causal, 0.5)
        np.testing.assert_allclose(O, np.broadcast_to(v[:, :1], O.shape), atol=1e-12)


def check_zero_q_mean(fwd):
    """Q = 0 gives uniform weights over the visible keys: the mean of V over
    them (the causal prefix mean, bottom-right aligned when Nq < Nk)."""
    for Nq, Nk in ((6, 6), (3, 7)):
        q, k, v = tiny(Hq=2, Hkv=1, Nq=Nq, Nk=Nk)
        q[:] = 0.0
        O, L = fwd(q, k, v, False, 0.5)
        np.testing.assert_allclose(O[0, :, 0], np.broadcast_to(v[0, :, 0].mean(0), (Nq, 4)), atol=1e-12)
        O, L = fwd(q, k, v, True, 0.5)
        for i in range(Nq):
            last = i + Nk - Nq
            np.testing.assert_allclose(O[0, i, 1], v[0, :last + 1, 0].mean(0), atol=1e-12)
            assert abs(L[0, 1, i] - math.log(last + 1)) < 1e-12


def check_causal_row0(fwd):
    q, k, v = tiny(Nq=6, Nk=6)
    O, L = fwd(q, k, v, True, 0.9)
    np.testing.assert_allclose(O[0, 0, 0], v[0, 0, 0], atol=1e-14)
    s00 = 0.9 * float(np.dot(q[0, 0, 0], k[0, 0, 0]))
    assert abs(L[0, 0, 0] - s00) < 1e-12


def check_lse_direct(fwd):
    """LSE_i = ln sum_j exp(S_ij), summed directly (no max shift) with fsum."""
    q, k, v = tiny(Hq=2, Hkv=2, Nq=4, Nk=4)
    scale = 0.3
    for causal in (False, True):
        _, L = fwd(q, k, v, causal, scale)
        for h in range(2):
            for i in range(4):
                js = range(4) if not causal else range(i + 1)
                ref = math.log(math.fsum(math.exp(scale * float(np.dot(q[0, i, h], k[0, j, h]))) for j in js))
                assert abs(L[0, h, i] - ref) < 1e-12


def check_key_shift(fwd):
    """K_j -> K_j + u shifts every score of row i by c_i = scale Q_i.u:
    O is unchanged and LSE_i moves by exactly c_i."""
    q, k, v = tiny(Hq=2, Hkv=1, Nq=5, Nk=5)
    u = rnd(4)
    scale = 0.6
    for causal in (False, True):
        O1, L1 = fwd(q, k, v, causal, scale)
        O2, L2 = fwd(q, k + u, v, causal, scale)
        np.testing.assert_allclose(O2, O1, atol=1e-12)
        c = scale * np.einsum("bihd,d->bhi", q, u)
        np.testing.assert_allclose(L2 - L1, c, atol=1e-12)


def check_permutation(fwd):
    q, k, v = tiny(Nq=4, Nk=7)
    perm = RNG.permutation(7)
    O1, L1 = fwd(q, k, v, False, 0.5)
    O2, L2 = fwd(q, k[:, perm], v[:, perm], False, 0.5)
    np.testing.assert_allclose(O2, O1, atol=1e-12)
    np.testing.assert_allclose(L2, L1, atol=1e-12)


def check_gqa_replication(fwd):
    q, k, v = tiny(B=2, Hq=6, Hkv=2, Nq=5, Nk=5)
    for causal in (False, True):
        O1, L1 = fwd(q, k, v, causal, 0.5)
        kr, vr = np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2)
        O2, L2 = fwd(q, kr, vr, causal, 0.5)
        np.testing.assert_allclose(O1, O2, atol=1e-13)
        np.testing.assert_allclose(L1, L2, atol=1e-13)


def check_finite_differences(bwd, fwd=oracle.attention_fwd):
    """Central differences of L = sum(dO * O) in every input element."""
    h = 1e-6
    for sh, causal in ((dict(B=1, Hq=2, Hkv=2, Nq=5, Nk=5, d=4), True),
                       (dict(B=1, Hq=4, Hkv=2, Nq=3, Nk=5, d=3), False),
                       (dict(B=1, Hq=4, Hkv=2, Nq=4, Nk=6, d=3), True)):
        q, k, v = tiny(**sh)
        do = rnd(*q.shape)
        scale = 0.45
        dq, dk, dv = bwd(q, k, v, do, causal, scale)

        def loss(qq, kk, vv):
            O, _ = fwd(qq, kk, vv, causal, scale)
            return float(np.sum(do * O))

        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                xp, xm = x.copy(), x.copy()
                xp[idx] += h
                xm[idx] -= h
                args_p = dict(q=q, k=k, v=v)
                args_m = dict(q=q, k=k, v=v)
                args_p[name], args_m[name] = xp, xm
                num[idx] = (loss(**{"qq": args_p["q"], "kk": args_p["k"], "vv": args_p["v"]})
                            - loss(**{"qq": args_m["q"], "kk": args_m["k"], "vv": args_m["v"]})) / (2 * h)
            np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-7, err_msg=f"d{name}")


def check_grad_invariants(bwd):
    """Every row of dS sums to zero, so sum_j dK_j = 0; the rows of P sum to
    one, so sum_j dV_j = sum over the group's heads and rows of dO."""
    q, k, v = tiny(B=2, Hq=4, Hkv=2, Nq=6, Nk=6, d=3)
    do = rnd(*q.shape)
    for causal in (False, True):
        dq, dk, dv = bwd(q, k, v, do, causal, 0.7)
        np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
        want = do.reshape(2, 6, 2, 2, 3).sum(axis=(1, 3))
        np.testing.assert_allclose(dv.sum(axis=1), want, atol=1e-12)


# ---------------------------------------------------------------------------
# the pins, run on the oracle as it stands
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("check", [check_brute_force, check_constant_v, check_zero_q_mean,
                                   check_causal_row0, check_lse_direct, check_key_shift,
                                   check_permutation, check_gqa_replication])
def test_forward_pins(check):
    check(oracle.attention_fwd)


def test_rows_of_p_sum_to_one():
    q, k, v = tiny(Nq=6, Nk=9)
    for causal in (False, True):
        P, _ = oracle.softmax_rows(oracle.scores(q[0, :, 0], k[0, :, 0], 0.8, oracle.visible_mask(6, 9, causal)))
        np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-14)
        assert (P >= 0).all()
        if causal:
            assert (P[~oracle.visible_mask(6, 9, True)] == 0).all()


@pytest.mark.parametrize("block", [1, 3, 16, None])
def test_online_recurrence_equals_two_pass(block):
    for sh in SHAPES + [dict(B=1, Hq=2, Hkv=1, Nq=17, Nk=40, d=8)]:
        q, k, v = tiny(**sh)
        for causal in (False, True):
            blk = block or sh["Nk"]
            O1, L1 = oracle.attention_fwd(q, k, v, causal, 0.4)
            O2, L2 = oracle.attention_fwd_online(q, k, v, causal, 0.4, blk)
            np.testing.assert_allclose(O2, O1, atol=1e-12)
            np.testing.assert_allclose(L2, L1, atol=1e-12)


def test_online_recurrence_large_scores_no_overflow():
    """The running max keeps exp() finite where a naive sum would overflow."""
    q, k, v = tiny(Nq=4, Nk=8)
    O1, L1 = oracle.attention_fwd(q * 200, k, v, True, 1.0)
    O2, L2 = oracle.attention_fwd_online(q * 200, k, v, True, 1.0, 3)
    assert np.isfinite(O1).all() and np.isfinite(L1).all()
    np.testing.assert_allclose(O2, O1, atol=1e-10)
    np.testing.assert_allclose(L2, L1, rtol=1e-13)


def test_rows_with_no_visible_key():
    """Reading: a row that sees no key (causal with Nq > Nk) has O = 0, LSE = -inf,
    in both the two-pass and the online form."""
    q, k, v = tiny(Nq=5, Nk=3)
    O, L = oracle.attention_fwd(q, k, v, True, 0.5)
    O2, L2 = oracle.attention_fwd_online(q, k, v, True, 0.5, 2)
    assert (O[0, :2] == 0).all() and np.isneginf(L[0, :, :2]).all()
    assert (O2[0, :2] == 0).all() and np.isneginf(L2[0, :, :2]).all()
    np.testing.assert_allclose(O2[0, 2:], O[0, 2:], atol=1e-12)


def test_rows_sampled_equal_full():
    q, k, v = tiny(B=2, Hq=4, Hkv=2, Nq=9, Nk=9)
    O, L = oracle.attention_fwd(q, k, v, True, 0.5)
    rows = [0, 4, 8]
    Or, Lr = oracle.attention_fwd_rows(q, k, v, True, 0.5, 1, 3, rows)
    np.testing.assert_allclose(Or, O[1, rows, 3], atol=1e-14)
    np.testing.assert_allclose(Lr, L[1, 3, rows], atol=1e-14)


def test_backward_finite_differences():
    check_finite_differences(oracle.attention_bwd)


def test_backward_invariants():
    check_grad_invariants(oracle.attention_bwd)


def test_preprocess_equals_rowsum_p_dp():
    q, k, v = tiny(B=1, Hq=2, Hkv=1, Nq=6, Nk=6, d=3)
    do = rnd(*q.shape)
    O, _ = oracle.attention_fwd(q, k, v, True, 0.5)
    D = oracle.bwd_preprocess(O, do)
    for h in range(2):
        P, _ = oracle.softmax_rows(oracle.scores(q[0, :, h], k[0, :, 0], 0.5, oracle.visible_mask(6, 6, True)))
        dP = do[0, :, h] @ v[0, :, 0].T
        np.testing.assert_allclose(D[0, h], (P * dP).sum(axis=1), atol=1e-12)


def test_backward_sampled_rows_match_full():
    q, k, v = tiny(B=2, Hq=4, Hkv=2, Nq=7, Nk=9, d=3)
    do = rnd(*q.shape)
    for causal in (False, True):
        dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal, 0.5)
        rows = [0, 3, 6]
        np.testing.assert_allclose(oracle.attention_bwd_dq_rows(q, k, v, do, causal, 0.5, 1, 2, rows),
                                   dq[1, rows, 2], atol=1e-13)
        keys = [0, 4, 8]
        dk_s, dv_s = oracle.attention_bwd_kv_rows(q, k, v, do, causal, 0.5, 1, 1, keys, row_chunk=3)
        np.testing.assert_allclose(dk_s, dk[1, keys, 1], atol=1e-13)
        np.testing.assert_allclose(dv_s, dv[1, keys, 1], atol=1e-13)


def test_backward_head_subset_matches_full():
    q, k, v = tiny(B=2, Hq=4, Hkv=2, Nq=5, Nk=5, d=3)
    do = rnd(*q.shape)
    full = oracle.attention_bwd(q, k, v, do, True, 0.5)
    part = oracle.attention_bwd(q, k, v, do, True, 0.5, kv_heads=[(1, 0)])
    np.testing.assert_allclose(part[0][1, :, 0:2], full[0][1, :, 0:2], atol=1e-14)
    np.testing.assert_allclose(part[1][1, :, 0], full[1][1, :, 0], atol=1e-14)
    np.testing.assert_allclose(part[2][1, :, 0], full[2][1, :, 0], atol=1e-14)


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------

def test_decode_brute_force():
    B, Hq, Hkv, Nmax, d = 4, 4, 2, 9, 3
    q, kc, vc = rnd(B, 1, Hq, d), rnd(B, Nmax, Hkv, d), rnd(B, Nmax, Hkv, d)
    sl = [9, 1, 5, 0]
    O, L = oracle.decode(q, kc, vc, sl, 0.6)
    for b in range(B):
        n = sl[b]
        if n == 0:
            assert (O[b] == 0).all() and np.isneginf(L[b]).all()
            continue
        Ob, Lb = oracle.brute_force_attention(q[b:b + 1].tolist(), kc[b:b + 1, :n].tolist(),
                                              vc[b:b + 1, :n].tolist(), False, 0.6)
        np.testing.assert_allclose(O[b], np.array(Ob)[0], atol=1e-12)
        np.testing.assert_allclose(L[b], np.array(Lb)[0], atol=1e-12)


@pytest.mark.parametrize("chunk", [1, 2, 3, 4, 16])
def test_split_combine_invariant_to_split_count(chunk):
    B, Hq, Hkv, Nmax, d = 3, 4, 1, 11, 3
    q, kc, vc = rnd(B, 1, Hq, d), rnd(B, Nmax, Hkv, d), rnd(B, Nmax, Hkv, d)
    sl = [11, 4, 0]
    O, L = oracle.decode(q, kc, vc, sl, 0.5)
    S = -(-Nmax // chunk)
    Op, Lp = oracle.decode_splitkv(q, kc, vc, sl, 0.5, chunk, S)
    Oc, Lc = oracle.decode_combine(Op, Lp)
    np.testing.assert_allclose(Oc, O, atol=1e-12)
    np.testing.assert_allclose(Lc, L, atol=1e-12)


# ---------------------------------------------------------------------------
# the pages' worked examples (tests/golden/smithlab_tables.json)
# ---------------------------------------------------------------------------

def _golden():
    with open(os.path.join(GOLDEN, "smithlab_tables.json")) as f:
        return json.load(f)


def test_lse_memory_table():
    g = _golden()
    h, layers = g["model"]["heads"], g["model"]["layers"]
    for n, mib in g["lse_memory_MiB"].items():
        assert oracle.lse_bytes(1, h, int(n), layers) / 2**20 == pytest.approx(mib, abs=0.5)
    for n, gib in g["eager_memory_GiB"].items():
        assert oracle.eager_softmax_bytes(1, h, int(n), int(n), layers) / 2**30 == pytest.approx(gib, abs=0.5)


def test_flop_convention_attention_share():
    """Causal forward per token = 2 N h d, training = fwd + 2.5 fwd; the page's
    attention share of training FLOPs against 6 x parameters of weight FLOPs."""
    g = _golden()
    h, hd, layers, params = (g["model"][x] for x in ("heads", "head_dim", "layers", "non_embedding_params"))
    for n, pct in g["attention_share_percent"].items():
        n = int(n)
        fwd_tok = oracle.attention_flops(1, h, n, n, hd, True) / n
        assert fwd_tok == 2 * n * h * hd
        train_tok = (fwd_tok + oracle.attention_flops(1, h, n, n, hd, True, backward=True) / n) * layers
        share = 100 * train_tok / (train_tok + 6 * params)
        # the page prints the share cut to one decimal (8.85 -> 8.8, 27.97 -> 27.9)
        assert pct <= share < pct + 0.1


def test_flop_convention_cost_table():
    g = _golden()
    h, hd, layers = (g["model"][x] for x in ("heads", "head_dim", "layers"))
    for setup, row in g["usd_per_billion_tokens"].items():
        tflops = row["tflops"][0] * row["tflops"][1]
        for n in ("2048", "8192", "32768"):
            N = int(n)
            per_tok = layers * (oracle.attention_flops(1, h, N, N, hd, True)
                                + oracle.attention_flops(1, h, N, N, hd, True, backward=True)) / N
            usd = 1e9 * per_tok / (tflops * 1e12) / 3600 * row["usd_per_hour"]
            assert usd == pytest.approx(row[n], abs=0.051), setup


# ---------------------------------------------------------------------------
# planted mistakes: a copy of the oracle with one plausible error must fail a pin
# ---------------------------------------------------------------------------

def _fwd_mutant(kind):
    def fwd(q, k, v, causal, scale):
        q, k, v = np.asarray(q, float), np.asarray(k, float), np.asarray(v, float)
        B, Nq, Hq, d = q.shape
        Nk, Hkv = k.shape[1], k.shape[2]
        G = Hq // Hkv
        if kind == "causal_offset":
            mask = (np.arange(Nk)[None, :] <= np.arange(Nq)[:, None]) if causal else np.ones((Nq, Nk), bool)
        else:
            mask = oracle.visible_mask(Nq, Nk, causal)
        O = np.zeros((B, Nq, Hq, d))
        L = np.zeros((B, Hq, Nq))
        for b in range(B):
            for h in range(Hq):
                hk = (h % Hkv) if kind == "gqa_interleaved" else h // G
                sc = 1.0 if kind == "no_scale" else scale
                S = oracle.scores(q[b, :, h], k[b, :, hk], sc, mask)
                P, lse = oracle.softmax_rows(S)
                if kind == "lse_without_max":
                    lse = np.log(np.sum(np.exp(S - np.max(S, axis=1, keepdims=True)), axis=1))
                VV = k[b, :, hk] if kind == "k_for_v" else v[b, :, hk]
                O[b, :, h] = P @ VV
                L[b, h] = lse
        return O, L
    return fwd


@pytest.mark.parametrize("kind,checks", [
    ("no_scale", [check_brute_force, check_key_shift, check_lse_direct]),
    ("causal_offset", [check_zero_q_mean, check_brute_force]),
    ("k_for_v", [check_brute_force, check_constant_v]),
    ("lse_without_max", [check_lse_direct, check_causal_row0]),
    ("gqa_interleaved", [check_brute_force]),
])
def test_planted_forward_mistakes_are_caught(kind, checks):
    mutant = _fwd_mutant(kind)
    for check in checks:
        with pytest.raises(AssertionError):
            check(mutant)


def _bwd_mutant(kind):
    def bwd(q, k, v, do, causal, scale):
        dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal, scale)
        if kind == "dk_no_scale":
            dk = dk / scale
        elif kind == "dk_first_head_only":
            # forget the sum over the group's query heads: recompute from head 0 of each group
            q_, k_, v_, do_ = (np.asarray(x, float) for x in (q, k, v, do))
            G = q_.shape[2] // k_.shape[2]
            dq2, dk2, dv2 = oracle.attention_bwd(q_[:, :, ::G], k_, v_, do_[:, :, ::G], causal, scale)
            dk, dv = dk2, dv2
        elif kind == "dv_transposed_p":
            dv = dv[:, ::-1]
        return dq, dk, dv
    return bwd


@pytest.mark.parametrize("kind", ["dk_no_scale", "dk_first_head_only", "dv_transposed_p"])
def test_planted_backward_mistakes_are_caught(kind):
    with pytest.raises(AssertionError):
        check_finite_differences(_bwd_mutant(kind))


def test_partial_backward_over_key_chunks_sums_to_the_full_backward():
    # the backward of a context-parallel ring: per-chunk contributions with the full rows' LSE and D
    rng = np.random.default_rng(31)
    q, k, v, do = (rng.standard_normal(s) for s in ((1, 96, 4, 8), (1, 96, 2, 8), (1, 96, 2, 8), (1, 96, 4, 8)))
    for causal in (False, True):
        O, L = oracle.attention_fwd(q, k, v, causal, 0.3)
        D = oracle.bwd_preprocess(O, do)
        DQ, DK, DV = oracle.attention_bwd(q, k, v, do, causal, 0.3)
        dq = np.zeros_like(DQ)
        dk = np.zeros_like(DK)
        dv = np.zeros_like(DV)
        n = 32
        for r in range(3):            # query chunk
            for c in range(3):        # key chunk
                if causal and c > r:
                    continue
                qs, ks = slice(n * r, n * (r + 1)), slice(n * c, n * (c + 1))
                a, bb, cc = oracle.attention_bwd_partial(q[:, qs], k[:, ks], v[:, ks], do[:, qs], L[:, :, qs],
                                                         D[:, :, qs], causal and c == r, 0.3)
                dq[:, qs] += a
                dk[:, ks] += bb
                dv[:, ks] += cc
        np.testing.assert_allclose(dq, DQ, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dk, DK, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dv, DV, rtol=1e-10, atol=1e-12)
