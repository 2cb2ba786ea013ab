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
    """partial = oracle attention of one chunk pair; merge = oracle log-sum-exp combine."""

    def __init__(self, scale):
        self.scale = scale

    def partial(self, q, k, v, causal):
        import oracle
        O, L = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), causal, self.scale)
        return torch.from_numpy(O), torch.from_numpy(L)

    def merge(self, acc, part, last):
        import oracle
        o_acc, lse, out, first = acc
        o_p, l_p = part
        if first:
            o_new, l_new = o_p.numpy(), l_p.numpy()
        else:
            B, n, H, d = o_p.shape
            O_parts = np.stack([o_acc.double().numpy(), o_p.numpy()], axis=3)  # [B, n, H, 2, d]
            L_parts = np.stack([lse.double().numpy(), l_p.numpy()], axis=-1)   # [B, H, n, 2]
            O_parts = O_parts.reshape(B * n, H, 2, d)
            L_parts = L_parts.transpose(0, 2, 1, 3).reshape(B * n, H, 2)
            O, L = oracle.decode_combine(O_parts, L_parts)
            o_new = O.reshape(B, n, H, d)
            l_new = L.reshape(B, n, H).transpose(0, 2, 1)
        o_acc.copy_(torch.from_numpy(np.ascontiguousarray(o_new)))
        lse.copy_(torch.from_numpy(np.ascontiguousarray(l_new)))
        if last:
            out.copy_(o_acc)


class OracleBwdOps:
    """The backward's compute from the oracle: D, per-chunk-pair partial gradients, fp32 sums."""

    def __init__(self, scale):
        self.scale = scale

    def preprocess(self, q, k, v, o, do, lse):
        import oracle
        return torch.from_numpy(oracle.bwd_preprocess(o.numpy(), do.numpy()))

    def partial_bwd(self, q, k, v, o, do, lse, dvec, causal):
        import oracle
        parts = oracle.attention_bwd_partial(q.numpy(), k.numpy(), v.numpy(), do.numpy(), lse.numpy(), dvec.numpy(),
                                             causal, self.scale)
        return tuple(torch.from_numpy(x) for x in parts)

    def accumulate(self, acc, part, init):
        if init:
            acc.copy_(part)
        else:
            acc.add_(part)

    def cast(self, acc, out):
        out.copy_(acc)


def _bwd_rank_main(rank, world, port, causal, out):
    import torch.distributed as dist

    import oracle
    from exact_io_aware_80_b200 import ring
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, do = _bwd_inputs(world)
        O, L = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), causal, 0.25)
        n = q.shape[1] // world
        sl = slice(rank * n, (rank + 1) * n)
        c = lambda t: t[:, sl].contiguous()  # noqa: E731
        dq, dk, dv = ring.ring_attention_bwd(c(q), c(k), c(v), c(torch.from_numpy(O)), c(do),
                                             torch.from_numpy(L)[:, :, sl].contiguous(), causal=causal, scale=0.25,
                                             ops=OracleBwdOps(0.25))
        out[rank] = (dq.numpy(), dk.numpy(), dv.numpy())
    finally:
        dist.destroy_process_group()


def _bwd_inputs(world):
    g = torch.Generator().manual_seed(12)
    B, N, Hq, Hkv, d = 1, 40 * world, 4, 2, 8
    return (torch.randn(B, N, Hq, d, generator=g, dtype=torch.float64),
            torch.randn(B, N, Hkv, d, generator=g, dtype=torch.float64),
            torch.randn(B, N, Hkv, d, generator=g, dtype=torch.float64),
            torch.randn(B, N, Hq, d, generator=g, dtype=torch.float64))


@pytest.mark.parametrize("world,causal", [(1, True), (2, False), (2, True), (3, True)])
def test_ring_backward_over_gloo_ranks_is_the_full_backward(world, causal):
    import torch.multiprocessing as mp

    import oracle
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_bwd_rank_main, args=(world, port, causal, out), nprocs=world, join=True)
    q, k, v, do = _bwd_inputs(world)
    DQ, DK, DV = oracle.attention_bwd(q.numpy(), k.numpy(), v.numpy(), do.numpy(), causal, 0.25)
    n = q.shape[1] // world
    for r in range(world):
        dq, dk, dv = out[r]
        sl = slice(r * n, (r + 1) * n)
        np.testing.assert_allclose(dq, DQ[:, sl], rtol=0, atol=1e-6)
        np.testing.assert_allclose(dk, DK[:, sl], rtol=0, atol=1e-6)
        np.testing.assert_allclose(dv, DV[:, sl], rtol=0, atol=1e-6)


def _rank_main(rank, world, port, causal, out):
    import torch.distributed as dist

    from exact_io_aware_80_b200 import ring
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        g = torch.Generator().manual_seed(11)
        B, N, Hq, Hkv, d = 1, 48 * world, 4, 2, 16
        q = torch.randn(B, N, Hq, d, generator=g, dtype=torch.float64)
        k = torch.randn(B, N, Hkv, d, generator=g, dtype=torch.float64)
        v = torch.randn(B, N, Hkv, d, generator=g, dtype=torch.float64)
        n = N // world
        sl = slice(rank * n, (rank + 1) * n)
        o, lse = ring.ring_attention_fwd(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(),
                                         causal=causal, scale=0.25, ops=OracleOps(0.25))
        out[rank] = (o.numpy(), lse.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, False), (2, True), (3, True)])
def test_ring_over_gloo_ranks_is_exact_attention(world, causal):
    import torch.multiprocessing as mp

    import oracle
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, port, causal, out), nprocs=world, join=True)
    g = torch.Generator().manual_seed(11)
    B, N, Hq, Hkv, d = 1, 48 * world, 4, 2, 16
    q = torch.randn(B, N, Hq, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, N, Hkv, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, N, Hkv, d, generator=g, dtype=torch.float64)
    O, L = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), causal, 0.25)
    n = N // world
    for r in range(world):
        o, lse = out[r]
        np.testing.assert_allclose(o, O[:, r * n:(r + 1) * n], rtol=0, atol=1e-5)
        np.testing.assert_allclose(lse, L[:, :, r * n:(r + 1) * n], rtol=0, atol=1e-5)


def test_schedule_visits_every_chunk_once():
    from exact_io_aware_80_b200 import ring
    for world in (1, 2, 3, 5):
        for causal in (False, True):
            for r in range(world):
                sched = ring.ring_schedule(r, world, causal)
                assert sorted(c for _, c, _ in sched) == list(range(world))
                modes = {c: m for _, c, m in sched}
                if causal:
                    assert all(modes[c] == ("full" if c < r else "causal" if c == r else "skip") for c in modes)
                else:
                    assert set(modes.values()) == {"full"}
