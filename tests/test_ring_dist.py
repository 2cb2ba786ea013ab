"""Host-side checks of the ring-attention driver (exact_io_aware_80_b200.ring) with
gloo ranks on the CPU.  The driver's compute steps are injected: partial
attention and the log-sum-exp merge come from the oracle, so these tests cover
the schedule, the chunk rotation and the merge order; the CUDA kernels of the
same steps are checked on the GPU by tests/test_gpu_ring.py.
"""
import datetime
import math
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class OracleOps:
    """attend = oracle attention of one chunk pair, folded into the accumulator by the
    oracle's log-sum-exp combine (the steps the CUDA kernel fuses)."""

    def __init__(self, scale):
        self.scale = scale

    def attend(self, q, k, v, causal, o_acc, lse_acc, out, lse_out, mode):
        import oracle
        o_p, l_p = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), causal, self.scale)
        if mode == 0:
            o_new, l_new = o_p, l_p
        else:
            B, n, H, d = o_p.shape
            O_parts = np.stack([o_acc.double().numpy(), o_p], axis=3)  # [B, n, H, 2, d]
            L_parts = np.stack([lse_acc.double().numpy(), l_p], axis=-1)  # [B, H, n, 2]
            O_parts = O_parts.reshape(B * n, H, 2, d)
            L_parts = L_parts.transpose(0, 2, 1, 3).reshape(B * n, H, 2)
            O, L = oracle.decode_combine(O_parts, L_parts)
            o_new = O.reshape(B, n, H, d)
            l_new = L.reshape(B, n, H).transpose(0, 2, 1)
        o_new = torch.from_numpy(np.ascontiguousarray(o_new))
        l_new = torch.from_numpy(np.ascontiguousarray(l_new))
        if mode != 2:
            o_acc.copy_(o_new)
            lse_acc.copy_(l_new)
        out.copy_(o_new)
        lse_out.copy_(l_new)


class OracleBwdOps:
    """The backward's compute from the oracle: D, per-chunk-pair partial gradients added into fp64 sums."""

    def __init__(self, scale):
        self.scale = scale

    def preprocess(self, q, k, v, o, do, lse):
        import oracle
        return torch.from_numpy(oracle.bwd_preprocess(o.numpy(), do.numpy()))

    def accumulate_bwd(self, q, k, v, do, lse, dvec, causal, dq_acc, dk_acc, dv_acc, init_q, init_kv):
        import oracle
        dq, dk, dv = (torch.from_numpy(x) for x in oracle.attention_bwd_partial(
            q.numpy(), k.numpy(), v.numpy(), do.numpy(), lse.numpy(), dvec.numpy(), causal, self.scale))
        for acc, part, init in ((dq_acc, dq, init_q), (dk_acc, dk, init_kv), (dv_acc, dv, init_kv)):
            if init:
                acc.copy_(part)
            else:
                acc.add_(part)

    def cast(self, acc, out):
        out.copy_(acc)


def _bwd_rank_main(rank, world, port, causal, layout, out):
    import torch.distributed as dist

    import oracle
    from exact_io_aware_80_b200 import ring
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, do = _bwd_inputs(world)
        O, L = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), causal, 0.25)
        c = lambda t, axis=1: _local(t, rank, world, layout, axis)  # noqa: E731
        dq, dk, dv = ring.ring_attention_bwd(c(q), c(k), c(v), c(torch.from_numpy(O)), c(do),
                                             c(torch.from_numpy(L), 2), causal=causal, scale=0.25,
                                             ops=OracleBwdOps(0.25), layout=layout)
        out[rank] = (dq.numpy(), dk.numpy(), dv.numpy())
    finally:
        dist.destroy_process_group()


def _bwd_inputs(world):
    g = torch.Generator().manual_seed(12)
    B, N, Hq, Hkv, d = 1, 40 * world, 4, 2, 8  # 40 world rows: 2 world parts of 20
    return (torch.randn(B, N, Hq, d, generator=g, dtype=torch.float64),
            torch.randn(B, N, Hkv, d, generator=g, dtype=torch.float64),
            torch.randn(B, N, Hkv, d, generator=g, dtype=torch.float64),
            torch.randn(B, N, Hq, d, generator=g, dtype=torch.float64))


@pytest.mark.parametrize("world,causal,layout", [(1, True, "contiguous"), (2, False, "contiguous"),
                                                 (2, True, "contiguous"), (3, True, "contiguous"),
                                                 (2, True, "zigzag"), (3, True, "zigzag")])
def test_ring_backward_over_gloo_ranks_is_the_full_backward(world, causal, layout):
    import torch.multiprocessing as mp

    import oracle
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_bwd_rank_main, args=(world, port, causal, layout, out), nprocs=world, join=True)
    q, k, v, do = _bwd_inputs(world)
    DQ, DK, DV = oracle.attention_bwd(q.numpy(), k.numpy(), v.numpy(), do.numpy(), causal, 0.25)
    for r in range(world):
        dq, dk, dv = out[r]
        np.testing.assert_allclose(dq, _local(DQ, r, world, layout), rtol=0, atol=1e-6)
        np.testing.assert_allclose(dk, _local(DK, r, world, layout), rtol=0, atol=1e-6)
        np.testing.assert_allclose(dv, _local(DV, r, world, layout), rtol=0, atol=1e-6)


def _local(t, rank, world, layout, axis=1):
    """This rank's parts of a whole-sequence tensor, concatenated in owned order."""
    from exact_io_aware_80_b200 import ring
    NP = ring.num_parts(world, layout)
    n = t.shape[axis] // NP
    idx = [slice(None)] * t.ndim
    parts = []
    for a in ring.owned_parts(rank, world, layout):
        idx[axis] = slice(a * n, (a + 1) * n)
        parts.append(t[tuple(idx)])
    return np.concatenate(parts, axis=axis) if isinstance(t, np.ndarray) else torch.cat(parts, dim=axis).contiguous()


def _fwd_inputs(world):
    g = torch.Generator().manual_seed(11)
    B, N, Hq, Hkv, d = 1, 48 * world, 4, 2, 16
    return (torch.randn(B, N, Hq, d, generator=g, dtype=torch.float64),
            torch.randn(B, N, Hkv, d, generator=g, dtype=torch.float64),
            torch.randn(B, N, Hkv, d, generator=g, dtype=torch.float64))


def _rank_main(rank, world, port, causal, layout, out):
    import torch.distributed as dist

    from exact_io_aware_80_b200 import ring
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v = (_local(t, rank, world, layout) for t in _fwd_inputs(world))
        o, lse = ring.ring_attention_fwd(q, k, v, causal=causal, scale=0.25, ops=OracleOps(0.25), layout=layout)
        out[rank] = (o.numpy(), lse.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal,layout", [(2, False, "contiguous"), (2, True, "contiguous"),
                                                 (3, True, "contiguous"), (2, True, "zigzag"), (3, True, "zigzag")])
def test_ring_over_gloo_ranks_is_exact_attention(world, causal, layout):
    import torch.multiprocessing as mp

    import oracle
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, port, causal, layout, out), nprocs=world, join=True)
    q, k, v = _fwd_inputs(world)
    O, L = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), causal, 0.25)
    for r in range(world):
        o, lse = out[r]
        np.testing.assert_allclose(o, _local(O, r, world, layout), rtol=0, atol=1e-5)
        np.testing.assert_allclose(lse, _local(L, r, world, layout, axis=2), rtol=0, atol=1e-5)


@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
def test_schedule_covers_every_pair_once(layout):
    from exact_io_aware_80_b200 import ring
    for world in (1, 2, 3, 5):
        for causal in (False, True):
            seen = {}
            work = []
            for r in range(world):
                mine = ring.owned_parts(r, world, layout)
                cnt = 0
                for s, c, pairs in ring.ring_schedule(r, world, causal, layout):
                    assert c == (r - s) % world
                    theirs = ring.owned_parts(c, world, layout)
                    for ia, ib, mode in pairs:
                        a, b = mine[ia], theirs[ib]
                        assert (a, b) not in seen
                        seen[(a, b)] = mode
                        assert mode == ("causal" if causal and a == b else "full")
                        cnt += 1 if mode == "full" else 0.5
                work.append(cnt)
            NP = ring.num_parts(world, layout)
            want = {(a, b) for a in range(NP) for b in range(NP) if not causal or b <= a}
            assert set(seen) == want
            if causal and layout == "zigzag":
                assert max(work) == min(work)  # every rank gets the same causal work
