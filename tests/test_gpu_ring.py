"""Ring attention on one GPU: the ring schedule for W virtual ranks run one
after another (no communication) with the library's forward and log-sum-exp
merge kernels must give attention over the whole sequence (oracle): O max-abs
<= 1e-2, LSE <= 1e-3; the backward schedule (per-chunk dQ / dK / dV kernels
summed in fp32) must give the full backward: relative L2 <= 2e-2."""
import math

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_io_aware_80_b200 as m
    from exact_io_aware_80_b200 import _lib
    _lib.load()
    return m


@pytest.mark.parametrize("world,causal,d,dt,layout", [(1, True, 128, torch.bfloat16, "contiguous"),
                                                      (2, False, 128, torch.bfloat16, "contiguous"),
                                                      (4, True, 128, torch.bfloat16, "contiguous"),
                                                      (3, True, 64, torch.float16, "contiguous"),
                                                      (2, True, 128, torch.bfloat16, "zigzag"),
                                                      (4, True, 64, torch.float16, "zigzag")])
def test_local_ring_is_exact_attention(fa, world, causal, d, dt, layout):
    from exact_io_aware_80_b200 import ring
    N = 192 * world
    q, k, v = workloads.make_inputs(1, 4, 2, N, N, d, dt, seed_base=9000 + world)
    o, lse = ring.ring_attention_fwd_local(q.cuda(), k.cuda(), v.cuda(), world, causal, layout=layout)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    O, L = oracle.attention_fwd(q.float().numpy(), k.float().numpy(), v.float().numpy(), causal, 1 / math.sqrt(d))
    assert np.max(np.abs(o.float().cpu().numpy() - O)) <= 1e-2
    assert np.max(np.abs(lse.cpu().numpy() - L)) <= 1e-3


def test_merge_of_key_halves(fa):
    # attention over keys [0, 256) and [256, 512) merged = attention over all 512 keys
    from exact_io_aware_80_b200 import _lib
    q, k, v = workloads.make_inputs(2, 4, 4, 128, 512, 64, torch.bfloat16, seed_base=9100)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = fa.attention_fwd(q, k[:, :256].contiguous(), v[:, :256].contiguous(), False)
    o2, l2 = fa.attention_fwd(q, k[:, 256:].contiguous(), v[:, 256:].contiguous(), False)
    acc = torch.empty(2, 128, 4, 64, device="cuda", dtype=torch.float32)
    lse = torch.empty(2, 4, 128, device="cuda", dtype=torch.float32)
    out = torch.empty_like(q)
    st = torch.cuda.current_stream().cuda_stream
    _lib.fa_lse_merge(acc.data_ptr(), lse.data_ptr(), o1.data_ptr(), l1.data_ptr(), 0, 2, 128, 4, 64, 0, 1, st)
    _lib.fa_lse_merge(acc.data_ptr(), lse.data_ptr(), o2.data_ptr(), l2.data_ptr(), out.data_ptr(), 2, 128, 4, 64, 2,
                      1, st)
    torch.cuda.synchronize()
    O, L = oracle.attention_fwd(q.float().cpu().numpy(), k.float().cpu().numpy(), v.float().cpu().numpy(), False,
                                1 / 8)
    assert np.max(np.abs(out.float().cpu().numpy() - O)) <= 1e-2
    assert np.max(np.abs(lse.cpu().numpy() - L)) <= 1e-3


@pytest.mark.parametrize("world,causal,layout", [(1, True, "contiguous"), (2, False, "contiguous"),
                                                 (4, True, "contiguous"), (2, True, "zigzag"), (3, True, "zigzag")])
def test_local_ring_backward_is_the_full_backward(fa, world, causal, layout):
    from exact_io_aware_80_b200 import ring
    N, d = 160 * world, 128
    q, k, v, do = workloads.make_inputs(1, 4, 2, N, N, d, torch.bfloat16, seed_base=9200 + world, with_do=True)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = ring.ring_attention_fwd_local(qd, kd, vd, world, causal, layout=layout)
    dq, dk, dv = ring.ring_attention_bwd_local(qd, kd, vd, o, dod, lse, world, causal, layout=layout)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    DQ, DK, DV = oracle.attention_bwd(q.float().numpy(), k.float().numpy(), v.float().numpy(), do.float().numpy(),
                                      causal, 1 / math.sqrt(d))
    for g, G in ((dq, DQ), (dk, DK), (dv, DV)):
        gg = g.float().cpu().numpy()
        assert np.linalg.norm(gg - G) / np.linalg.norm(G) <= 2e-2
