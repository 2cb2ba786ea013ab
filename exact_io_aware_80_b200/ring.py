"""Context parallelism: ring attention across ranks (forward and backward).

The sequence is split into equal contiguous chunks, one per rank: rank r holds
queries, keys and values of positions [r n, (r + 1) n).  In step s = 0 .. W-1
rank r holds the key/value chunk c = (r - s) mod W, attends its queries to it
(causal: c < r all keys, c == r the causal diagonal, c > r nothing) with the
16-bit forward kernel, and folds the partial (O, LSE) into an fp32 accumulator
with the log-sum-exp merge kernel; meanwhile it sends its chunk to rank r + 1
and receives the next from rank r - 1 (point-to-point sends over the process
group, NCCL between GPUs).  After W steps every rank holds exact attention of
its queries over the whole sequence ("FlashAttention 심층 분석", "Flash-Decoding":
attention over disjoint key ranges merges exactly by log-sum-exp; the
koritips note names ring attention for context lengths past one GPU).

Backward: with the rows' LSE (from the forward) and D = rowsum(dO * O), each
(query chunk, key chunk) pair contributes exact partial gradients (the dQ and
dK/dV kernels on that pair); dQ partials are summed in fp32 on the query's
rank, and the fp32 dK/dV sums of a key chunk travel around the ring with its
keys and values and reach their owner after one last hop.

`ring_schedule` is the pure schedule; `ring_attention_fwd` / `ring_attention_bwd`
run it over a process group with the library's kernels (or, for host-side
tests, with the compute functions a caller passes in); the `_local` variants
run the same schedule for W virtual ranks on one device, one after another,
without communication.
"""
from __future__ import annotations

import math

from . import _lib

__all__ = ["ring_schedule", "ring_attention_fwd", "ring_attention_fwd_local", "ring_attention_bwd",
           "ring_attention_bwd_local"]


def ring_schedule(rank: int, world: int, causal: bool):
    """[(step, chunk, mode)] for one rank; mode "full", "causal" (diagonal chunk) or "skip"."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    out = []
    for s in range(world):
        c = (rank - s) % world
        if not causal or c < rank:
            mode = "full"
        elif c == rank:
            mode = "causal"
        else:
            mode = "skip"
        out.append((s, c, mode))
    return out


class _CudaOps:
    """The library's kernels: partial attention (fa_fwd) and the log-sum-exp merge (fa_lse_merge)."""

    def __init__(self, torch, scale):
        self.torch, self.scale = torch, scale

    def partial(self, q, k, v, causal):
        torch = self.torch
        B, N, Hq, d = q.shape
        _, Nk, Hkv, _ = k.shape
        o = torch.empty_like(q)
        lse = torch.empty(B, Hq, N, device=q.device, dtype=torch.float32)
        _lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, Nk, d,
                    causal, self.scale, _dtype(torch, q), torch.cuda.current_stream(q.device).cuda_stream)
        return o, lse

    def merge(self, acc, part, last):
        torch = self.torch
        o_acc, lse_acc, out, first = acc
        o_p, lse_p = part
        B, N, H, d = o_p.shape
        mode = 0 if first else (2 if last else 1)
        if mode == 0 and last:  # a single chunk: its partial is the answer
            out.copy_(o_p)
            lse_acc.copy_(lse_p)
            return
        _lib.fa_lse_merge(o_acc.data_ptr(), lse_acc.data_ptr(), o_p.data_ptr(), lse_p.data_ptr(),
                          out.data_ptr() if mode == 2 else 0, B, N, H, d, mode, _dtype(torch, o_p),
                          torch.cuda.current_stream(o_p.device).cuda_stream)


    # ----------------------------------------------------------------- backward
    def preprocess(self, q, k, v, o, do, lse):
        """D = rowsum(dO * O) of this rank's rows, in a workspace the backward kernels read."""
        torch = self.torch
        B, N, Hq, d = q.shape
        ws = torch.empty(_lib.fa_bwd_workspace_bytes(B, Hq, N), device=q.device, dtype=torch.uint8)
        _lib.fa_bwd_preprocess(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                               0, 0, 0, ws.data_ptr(), B, Hq, k.shape[2], N, k.shape[1], d, False, self.scale,
                               _dtype(torch, q), torch.cuda.current_stream(q.device).cuda_stream)
        return ws

    def partial_bwd(self, q, k, v, o, do, lse, ws, causal):
        """dQ, dK, dV contributions (16-bit) of one chunk pair, with the rows' LSE and D."""
        torch = self.torch
        B, N, Hq, d = q.shape
        _, Nk, Hkv, _ = k.shape
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(), dq.data_ptr(),
                dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), B, Hq, Hkv, N, Nk, d, causal, self.scale,
                _dtype(torch, q), torch.cuda.current_stream(q.device).cuda_stream)
        _lib.fa_bwd_dkdv(*args)
        _lib.fa_bwd_dq(*args)
        return dq, dk, dv

    def accumulate(self, acc, part, init):
        torch = self.torch
        _lib.fa_accumulate(acc.data_ptr(), part.data_ptr(), part.numel(), init, _dtype(torch, part),
                           torch.cuda.current_stream(part.device).cuda_stream)

    def cast(self, acc, out):
        torch = self.torch
        _lib.fa_cast_f32(acc.data_ptr(), out.data_ptr(), out.numel(), _dtype(torch, out),
                         torch.cuda.current_stream(out.device).cuda_stream)


def _dtype(torch, t):
    return _lib.FA_BF16 if t.dtype == torch.bfloat16 else _lib.FA_FP16


def _run_schedule(sched, q, get_kv, ops, out, lse, o_acc, torch):
    """Partial attention per non-skipped step, merged in step order into (o_acc, lse) -> out."""
    work = [(s, c, m) for s, c, m in sched if m != "skip"]
    first = True
    for i, (s, c, mode) in enumerate(work):
        k, v = get_kv(s)
        part = ops.partial(q, k, v, mode == "causal")
        ops.merge((o_acc, lse, out, first), part, i == len(work) - 1)
        first = False
    return out, lse


def ring_attention_fwd_local(q, k, v, world: int, causal: bool = False, scale: float | None = None):
    """The ring schedule for `world` virtual ranks on one device (no communication).

    q [B, N, Hq, d], k/v [B, N, Hkv, d] with N divisible by `world`; returns O, LSE of the whole sequence.
    """
    import torch
    B, N, Hq, d = q.shape
    if N % world:
        raise ValueError("sequence length must be a multiple of the number of ranks")
    n = N // world
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    ops = _CudaOps(torch, scale)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, N, device=q.device, dtype=torch.float32)
    for r in range(world):
        qr = q[:, r * n:(r + 1) * n].contiguous()
        o_acc = torch.empty(B, n, Hq, d, device=q.device, dtype=torch.float32)
        lse_r = torch.empty(B, Hq, n, device=q.device, dtype=torch.float32)
        out_r = torch.empty_like(qr)
        chunks = {c: (k[:, c * n:(c + 1) * n].contiguous(), v[:, c * n:(c + 1) * n].contiguous()) for c in range(world)}
        sched = ring_schedule(r, world, causal)
        _run_schedule(sched, qr, lambda s: chunks[sched[s][1]], ops, out_r, lse_r, o_acc, torch)
        out[:, r * n:(r + 1) * n] = out_r
        lse[:, :, r * n:(r + 1) * n] = lse_r
    return out, lse


def ring_attention_fwd(q, k, v, causal: bool = False, scale: float | None = None, group=None, ops=None):
    """Ring attention over a process group; q, k, v are this rank's chunk ([B, n, H, d]).

    Returns this rank's O [B, n, Hq, d] and LSE [B, Hq, n].  `ops` (partial, merge) defaults to the
    library's CUDA kernels; the sends and receives of the K/V chunks overlap the compute of each step.
    """
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, n, Hq, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    ops = ops or _CudaOps(torch, scale)
    acc_dtype = torch.float32
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, n, device=q.device, dtype=torch.float32)
    o_acc = torch.empty(B, n, Hq, d, device=q.device, dtype=acc_dtype)
    sched = ring_schedule(rank, world, causal)
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    nxt_g = dist.get_global_rank(group, nxt) if group is not None else nxt
    prv_g = dist.get_global_rank(group, prv) if group is not None else prv
    cur = (k.contiguous(), v.contiguous())
    bufs = [cur, (torch.empty_like(cur[0]), torch.empty_like(cur[1]))]
    # step s computes on bufs[s % 2] while the chunk for step s + 1 travels into bufs[(s + 1) % 2]
    work = [(s, c, m) for s, c, m in sched if m != "skip"]
    first = True
    done = 0
    for s in range(world):
        reqs = []
        if s + 1 < world:
            src, dst = bufs[s % 2], bufs[(s + 1) % 2]
            ops_p2p = [dist.P2POp(dist.isend, src[0], nxt_g, group), dist.P2POp(dist.isend, src[1], nxt_g, group),
                       dist.P2POp(dist.irecv, dst[0], prv_g, group), dist.P2POp(dist.irecv, dst[1], prv_g, group)]
            reqs = dist.batch_isend_irecv(ops_p2p)
        _, c, mode = sched[s]
        if mode != "skip":
            kc, vc = bufs[s % 2]
            part = ops.partial(q, kc, vc, mode == "causal")
            done += 1
            ops.merge((o_acc, lse, out, first), part, done == len(work))
            first = False
        for r in reqs:
            r.wait()
    if not work:  # every key chunk is after this rank's queries (cannot happen for causal rank order)
        out.zero_()
        lse.fill_(-math.inf)
    return out, lse


def ring_attention_bwd_local(q, k, v, o, do, lse, world: int, causal: bool = False, scale: float | None = None):
    """The backward ring schedule for `world` virtual ranks on one device (no communication).

    q, o, do [B, N, Hq, d], k/v [B, N, Hkv, d], lse [B, Hq, N] of the whole sequence (N divisible by
    `world`); returns dQ, dK, dV.
    """
    import torch
    B, N, Hq, d = q.shape
    if N % world:
        raise ValueError("sequence length must be a multiple of the number of ranks")
    n = N // world
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    ops = _CudaOps(torch, scale)
    sl = [slice(r * n, (r + 1) * n) for r in range(world)]
    ch = lambda t, r: t[:, sl[r]].contiguous()  # noqa: E731
    dk_acc = [torch.empty(B, n, k.shape[2], d, device=q.device, dtype=torch.float32) for _ in range(world)]
    dv_acc = [torch.empty(B, n, k.shape[2], d, device=q.device, dtype=torch.float32) for _ in range(world)]
    kv_init = [True] * world
    dq = torch.empty_like(q)
    for r in range(world):
        qr, orr, dor = ch(q, r), ch(o, r), ch(do, r)
        lr = lse[:, :, sl[r]].contiguous()
        ws = ops.preprocess(qr, ch(k, r), ch(v, r), orr, dor, lr)
        dq_acc = torch.empty(B, n, Hq, d, device=q.device, dtype=torch.float32)
        first = True
        for s_, c, mode in ring_schedule(r, world, causal):
            if mode == "skip":
                continue
            dq_p, dk_p, dv_p = ops.partial_bwd(qr, ch(k, c), ch(v, c), orr, dor, lr, ws, mode == "causal")
            ops.accumulate(dq_acc, dq_p, first)
            ops.accumulate(dk_acc[c], dk_p, kv_init[c])
            ops.accumulate(dv_acc[c], dv_p, kv_init[c])
            first = False
            kv_init[c] = False
        dq_r = torch.empty_like(qr)
        ops.cast(dq_acc, dq_r)
        dq[:, sl[r]] = dq_r
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    for c in range(world):
        if kv_init[c]:  # no query attends to this chunk (cannot happen for these schedules)
            dk[:, sl[c]] = 0
            dv[:, sl[c]] = 0
            continue
        t = torch.empty_like(ch(k, c))
        ops.cast(dk_acc[c], t)
        dk[:, sl[c]] = t
        ops.cast(dv_acc[c], t)
        dv[:, sl[c]] = t
    return dq, dk, dv


def ring_attention_bwd(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None, group=None,
                       ops=None):
    """Backward of ring_attention_fwd over a process group: this rank's dQ, dK, dV.

    q, o, do [B, n, Hq, d], k/v [B, n, Hkv, d] and lse [B, Hq, n] are this rank's chunk (lse as returned
    by ring_attention_fwd: over the whole sequence).  Keys and values travel as in the forward, now with
    their fp32 dK / dV sums; after the last step the sums take one more hop to their owner.
    """
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, n, Hq, d = q.shape
    Hkv = k.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    ops = ops or _CudaOps(torch, scale)
    sched = ring_schedule(rank, world, causal)
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    nxt_g = dist.get_global_rank(group, nxt) if group is not None else nxt
    prv_g = dist.get_global_rank(group, prv) if group is not None else prv
    ws = ops.preprocess(q, k, v, o, do, lse)
    dq_acc = torch.empty(B, n, Hq, d, device=q.device, dtype=torch.float32)
    zeros = lambda: torch.zeros(B, n, Hkv, d, device=q.device, dtype=torch.float32)  # noqa: E731
    kv = [(k.contiguous(), v.contiguous()), (torch.empty_like(k), torch.empty_like(v))]
    acc = [(zeros(), zeros()), (zeros(), zeros())]

    def exchange(send, recv):
        ops_p2p = [dist.P2POp(dist.isend, t, nxt_g, group) for t in send] + \
                  [dist.P2POp(dist.irecv, t, prv_g, group) for t in recv]
        return dist.batch_isend_irecv(ops_p2p)

    first = True
    for s in range(world):
        cur, nx = s % 2, (s + 1) % 2
        # keys and values of the next step travel while this step computes
        reqs = exchange(kv[cur], kv[nx]) if s + 1 < world else []
        _, c, mode = sched[s]
        if mode != "skip":
            dq_p, dk_p, dv_p = ops.partial_bwd(q, kv[cur][0], kv[cur][1], o, do, lse, ws, mode == "causal")
            ops.accumulate(dq_acc, dq_p, first)
            ops.accumulate(acc[cur][0], dk_p, False)
            ops.accumulate(acc[cur][1], dv_p, False)
            first = False
        for r_ in reqs:
            r_.wait()
        # this chunk's gradient sums move on with it (after this step's contribution)
        if s + 1 < world:
            for r_ in exchange(acc[cur], acc[nx]):
                r_.wait()
            acc[cur] = (zeros(), zeros())
    # the sums now held belong to the next rank's chunk: one last hop to their owners
    last = (world - 1) % 2
    if world == 1:
        own = acc[last]
    else:
        own = (zeros(), zeros())
        for r_ in exchange(acc[last], own):
            r_.wait()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if first:
        dq.zero_()
    else:
        ops.cast(dq_acc, dq)
    ops.cast(own[0], dk)
    ops.cast(own[1], dv)
    return dq, dk, dv
