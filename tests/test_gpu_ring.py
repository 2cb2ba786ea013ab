"""Ring attention on one GPU.

* The ring schedule for W virtual ranks run one after another (no
  communication) with the library's forward-with-merge kernel must give
  attention over the whole sequence (oracle): O max-abs <= 1e-2, LSE <= 1e-3;
  the backward schedule (per-chunk dQ / dK / dV kernels adding into fp32)
  must give the full backward: relative L2 <= 2e-2.
* The fused entry points themselves: fa_fwd_merge over a partition of the keys
  equals attention over all keys, and over one chunk equals fa_fwd bit for bit;
  fa_bwd_accumulate over a partition equals the full backward, and over one
  chunk (then cast) equals fa_bwd bit for bit.
* The process-group driver itself (ring_attention_fwd / _bwd with the CUDA
  kernels) through a one-rank NCCL group on this GPU.
"""
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


def _fwd_merge(fa, q, k, v, acc_o, acc_lse, out, lse, mode, causal):
    from exact_io_aware_80_b200 import _lib
    B, N, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    _lib.fa_fwd_merge(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), acc_o.data_ptr(),
                      acc_lse.data_ptr(), mode, B, Hq, Hkv, N, Nk, d, causal, 1 / math.sqrt(d),
                      _lib.FA_BF16 if q.dtype == torch.bfloat16 else _lib.FA_FP16,
                      torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("d,dt,Nq,cuts", [(128, torch.bfloat16, 300, [0, 128, 333, 700]),
                                          (64, torch.float16, 129, [0, 1, 256, 257])])
def test_fwd_merge_over_key_chunks(fa, d, dt, Nq, cuts):
    """Modes 0, 1, ..., 2 over a partition of the keys = attention over all of them; the
    single-chunk mode 0 output = fa_fwd bit for bit."""
    Nk = cuts[-1]
    q, k, v = workloads.make_inputs(2, 4, 2, Nq, Nk, d, dt, seed_base=9300 + Nq)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    acc_o = torch.full((2, Nq, 4, d), float("nan"), device="cuda")
    acc_l = torch.full((2, 4, Nq), float("nan"), device="cuda")
    out, lse = torch.empty_like(q), torch.empty(2, 4, Nq, device="cuda")
    n = len(cuts) - 1
    for i in range(n):
        kc, vc = k[:, cuts[i]:cuts[i + 1]].contiguous(), v[:, cuts[i]:cuts[i + 1]].contiguous()
        _fwd_merge(fa, q, kc, vc, acc_o, acc_l, out, lse, 0 if i == 0 else (2 if i == n - 1 else 1), False)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    O, L = oracle.attention_fwd(q.float().cpu().numpy(), k.float().cpu().numpy(), v.float().cpu().numpy(), False,
                                1 / math.sqrt(d))
    assert np.max(np.abs(out.float().cpu().numpy() - O)) <= 1e-2
    assert np.max(np.abs(lse.cpu().numpy() - L)) <= 1e-3
    # one chunk, mode 0: the plain forward's result, and the accumulator holds it in fp32
    o1, l1 = fa.attention_fwd(q, k, v, True)
    _fwd_merge(fa, q, k, v, acc_o, acc_l, out, lse, 0, True)
    torch.cuda.synchronize()
    assert torch.equal(out, o1) and torch.equal(lse, l1)
    assert torch.equal(acc_o.to(q.dtype), o1) and torch.equal(acc_l, l1)


def test_bwd_accumulate_over_key_chunks(fa):
    """fa_bwd_accumulate over three key chunks (init on the first) = the full backward; over
    one chunk, cast to 16 bits = fa_bwd bit for bit."""
    from exact_io_aware_80_b200 import _lib
    B, Hq, Hkv, N, d = 1, 4, 2, 333, 128
    q, k, v, do = workloads.make_inputs(B, Hq, Hkv, N, N, d, torch.bfloat16, seed_base=9400, with_do=True)
    q, k, v, do = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.attention_fwd(q, k, v, False)
    st = torch.cuda.current_stream().cuda_stream
    ws = torch.empty(_lib.fa_bwd_workspace_bytes(B, Hq, N), device="cuda", dtype=torch.uint8)
    _lib.fa_bwd_preprocess(0, 0, 0, o.data_ptr(), do.data_ptr(), 0, 0, 0, 0, ws.data_ptr(), B, Hq, Hkv, N, N, d, 0,
                           1.0, _lib.FA_BF16, st)
    dq = torch.full((B, N, Hq, d), float("nan"), device="cuda")
    dk = torch.full((B, N, Hkv, d), float("nan"), device="cuda")
    dv = torch.full((B, N, Hkv, d), float("nan"), device="cuda")
    cuts = [0, 100, 256, N]
    for i in range(3):
        a, b = cuts[i], cuts[i + 1]
        kc, vc = k[:, a:b].contiguous(), v[:, a:b].contiguous()
        dkc = torch.full((B, b - a, Hkv, d), float("nan"), device="cuda")
        dvc = torch.full((B, b - a, Hkv, d), float("nan"), device="cuda")
        _lib.fa_bwd_accumulate(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), do.data_ptr(), lse.data_ptr(),
                               ws.data_ptr(), dq.data_ptr(), dkc.data_ptr(), dvc.data_ptr(), 3 if i == 0 else 2,
                               B, Hq, Hkv, N, b - a, d, False, 1 / math.sqrt(d), _lib.FA_BF16, st)
        dk[:, a:b] = dkc
        dv[:, a:b] = dvc
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    DQ, DK, DV = oracle.attention_bwd(q.float().cpu().numpy(), k.float().cpu().numpy(), v.float().cpu().numpy(),
                                      do.float().cpu().numpy(), False, 1 / math.sqrt(d))
    for g, G in ((dq, DQ), (dk, DK), (dv, DV)):
        gg = g.cpu().numpy().astype(np.float64)
        assert np.linalg.norm(gg - G) / np.linalg.norm(G) <= 2e-2
    # one chunk: cast to bf16 = the plain backward
    _lib.fa_bwd_accumulate(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(), lse.data_ptr(), ws.data_ptr(),
                           dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), 3, B, Hq, Hkv, N, N, d, True,
                           1 / math.sqrt(d), _lib.FA_BF16, st)
    g16 = fa.attention_bwd(q, k, v, o, do, lse, True)
    torch.cuda.synchronize()
    for acc, ref in zip((dq, dk, dv), g16):
        cast = torch.empty_like(ref)
        _lib.fa_cast_f32(acc.data_ptr(), cast.data_ptr(), cast.numel(), _lib.FA_BF16, st)
        torch.cuda.synchronize()
        assert torch.equal(cast, ref)


def test_process_group_driver_with_cuda_kernels(fa):
    """ring_attention_fwd / _bwd with the library's kernels through a one-rank NCCL process group."""
    import datetime
    import os
    import socket

    import torch.distributed as dist

    from exact_io_aware_80_b200 import ring
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        N, d = 640, 128
        q, k, v, do = workloads.make_inputs(1, 4, 2, N, N, d, torch.bfloat16, seed_base=9500, with_do=True)
        qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
        for causal in (False, True):
            o, lse = ring.ring_attention_fwd(qd, kd, vd, causal)
            dq, dk, dv = ring.ring_attention_bwd(qd, kd, vd, o, dod, lse, causal)
            torch.cuda.synchronize()
            assert fa.device_status() == 0
            O, L = oracle.attention_fwd(q.float().numpy(), k.float().numpy(), v.float().numpy(), causal,
                                        1 / math.sqrt(d))
            assert np.max(np.abs(o.float().cpu().numpy() - O)) <= 1e-2
            assert np.max(np.abs(lse.cpu().numpy() - L)) <= 1e-3
            DQ, DK, DV = oracle.attention_bwd(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                              do.float().numpy(), causal, 1 / math.sqrt(d))
            for g, G in ((dq, DQ), (dk, DK), (dv, DV)):
                gg = g.float().cpu().numpy()
                assert np.linalg.norm(gg - G) / np.linalg.norm(G) <= 2e-2
    finally:
        dist.destroy_process_group()


@pytest.mark.slow
def test_local_ring_eight_ranks_long_context_sampled(fa):
    """W = 8 virtual ranks (zigzag, 16 parts of 1024) over the long-context shape B=1,
    Hq=32, Hkv=8, N=16384, d=128, causal: sampled forward and dQ rows of three heads and
    dK/dV rows of one KV head against the oracle."""
    from exact_io_aware_80_b200 import ring
    w = workloads.get(4)
    q, k, v, do = workloads.workload_inputs(w)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = ring.ring_attention_fwd_local(qd, kd, vd, 8, True, layout="zigzag")
    dq, dk, dv = ring.ring_attention_bwd_local(qd, kd, vd, o, dod, lse, 8, True, layout="zigzag")
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    qn, kn, vn, don = (t.float().numpy().astype(np.float64) for t in (q, k, v, do))
    o64, lse64 = o.float().cpu().numpy(), lse.cpu().numpy()
    dq64, dk64, dv64 = (t.float().cpu().numpy() for t in (dq, dk, dv))
    rows = [0, 1, 1023, 1024, 5000, 8191, 8192, 15359, 16383]
    for h in (0, 17, 31):
        Or, Lr = oracle.attention_fwd_rows(qn, kn, vn, True, w.scale, 0, h, rows)
        assert np.abs(o64[0, rows, h] - Or).max() <= 1e-2
        assert np.abs(lse64[0, h, rows] - Lr).max() <= 1e-3
        dQr = oracle.attention_bwd_dq_rows(qn, kn, vn, don, True, w.scale, 0, h, rows)
        assert np.linalg.norm(dq64[0, rows, h] - dQr) / np.linalg.norm(dQr) <= 2e-2
    keys = [0, 1, 1023, 1024, 9000, 16383]
    dKr, dVr = oracle.attention_bwd_kv_rows(qn, kn, vn, don, True, w.scale, 0, 5, keys)
    assert np.linalg.norm(dk64[0, keys, 5] - dKr) / np.linalg.norm(dKr) <= 2e-2
    assert np.linalg.norm(dv64[0, keys, 5] - dVr) / np.linalg.norm(dVr) <= 2e-2
