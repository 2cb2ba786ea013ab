"""Context parallelism: ring attention across ranks (forward and backward).

The sequence is split into parts: W equal contiguous parts, rank r owning part
r ("contiguous"), or 2W parts with rank r owning parts r and 2W - 1 - r
("zigzag", which gives every rank the same causal work).  A rank holds the
queries, keys and values of its parts, concatenated in that order.  In step
s = 0 .. W-1 rank r holds the keys and values of rank c = (r - s) mod W and
attends each of its query parts a to each held key part b (causal: b < a all
keys, b == a the causal diagonal, b > a nothing) with the forward kernel, whose
epilogue folds the chunk's result into that query part's fp32 accumulator by
log-sum-exp (fa_fwd_merge: no 16-bit rounding of partial results); meanwhile
it sends the keys and values it holds to rank r + 1 and receives the next from
rank r - 1 (point-to-point sends over the process group, NCCL between GPUs).  After W steps every rank holds
exact attention of its queries over the whole sequence ("FlashAttention 심층
분석", "Flash-Decoding": attention over disjoint key ranges merges exactly by
log-sum-exp; the koritips note names ring attention for context lengths past
one GPU).

Backward: with the rows' LSE (from the forward) and D = rowsum(dO * O), each
(query part, key part) pair contributes exact partial gradients, which the dQ
and dK/dV kernels add straight into fp32 accumulators (fa_bwd_accumulate);
dQ sums stay on the query's rank, and the fp32 dK/dV sums of the held key
parts travel around the ring with their keys and values and reach their owner
after one last hop.  Only the final results are rounded to 16 bits.

`ring_schedule` is the pure schedule; `ring_attention_fwd` / `ring_attention_bwd`
run it over a process group with the library's kernels (or, for host-side
tests, with the compute functions a caller passes in); the `_local` variants
run the same schedule for W virtual ranks on one device, one after another,
without communication, taking and returning whole-sequence tensors.
"""
from __future__ import annotations

import math

from . import _lib

__all__ = ["owned_parts", "num_parts", "ring_schedule", "ring_attention_fwd", "ring_attention_fwd_local",
           "ring_attention_bwd", "ring_attention_bwd_local"]

LAYOUTS = ("contiguous", "zigzag")


def num_parts(world: int, layout: str) -> int:
    """Number of sequence parts: W (contiguous) or 2W (zigzag)."""
    if layout not in LAYOUTS:
        raise ValueError(f"layout must be one of {LAYOUTS}")
    return world if layout == "contiguous" else 2 * world


def owned_parts(rank: int, world: int, layout: str = "contiguous"):
    """Global part indices rank `rank` holds, in the order its local tensors concatenate them."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return [rank] if num_parts(world, layout) == world else [rank, 2 * world - 1 - rank]


def ring_schedule(rank: int, world: int, causal: bool, layout: str = "contiguous"):
    """[(step, held rank, [(own part idx, held part idx, mode)])]; mode "full" or "causal", skipped pairs left out."""
    mine = owned_parts(rank, world, layout)
    out = []
    for s in range(world):
        c = (rank - s) % world
        pairs = []
        for ia, a in enumerate(mine):
            for ib, b in enumerate(owned_parts(c, world, layout)):
                if not causal or b < a:
                    pairs.append((ia, ib, "full"))
                elif b == a:
                    pairs.append((ia, ib, "causal"))
        out.append((s, c, pairs))
    return out


class _CudaOps:
    """The library's kernels: the forward with its fp32 log-sum-exp merge (fa_fwd_merge), the
    backward preprocess, the backward adding into fp32 accumulators (fa_bwd_accumulate) and the
    final casts."""

    def __init__(self, torch, scale):
        self.torch, self.scale = torch, scale

    def attend(self, q, k, v, causal, o_acc, lse_acc, out, lse_out, mode):
        """Attention of q over one key chunk, merged into (o_acc, lse_acc) by log-sum-exp.

        mode 0: the accumulator takes this chunk's result; 1: merge and keep; 2: merge into
        out, lse_out (the last chunk).  out, lse_out are written in every mode."""
        torch = self.torch
        B, N, Hq, d = q.shape
        _, Nk, Hkv, _ = k.shape
        _lib.fa_fwd_merge(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_out.data_ptr(),
                          o_acc.data_ptr(), lse_acc.data_ptr(), mode, B, Hq, Hkv, N, Nk, d, causal, self.scale,
                          _dtype(torch, q), torch.cuda.current_stream(q.device).cuda_stream)

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

    def accumulate_bwd(self, q, k, v, do, lse, ws, causal, dq_acc, dk_acc, dv_acc, init_q, init_kv):
        """The dQ, dK, dV contributions of one chunk pair added into fp32 accumulators (or set, per init flag)."""
        torch = self.torch
        B, N, Hq, d = q.shape
        _, Nk, Hkv, _ = k.shape
        _lib.fa_bwd_accumulate(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(), lse.data_ptr(), ws.data_ptr(),
                               dq_acc.data_ptr(), dk_acc.data_ptr(), dv_acc.data_ptr(),
                               (1 if init_q else 0) | (2 if init_kv else 0), B, Hq, Hkv, N, Nk, d, causal,
                               self.scale, _dtype(torch, q), torch.cuda.current_stream(q.device).cuda_stream)

    def cast(self, acc, out):
        torch = self.torch
        _lib.fa_cast_f32(acc.data_ptr(), out.data_ptr(), out.numel(), _dtype(torch, out),
                         torch.cuda.current_stream(out.device).cuda_stream)


def _dtype(torch, t):
    return _lib.FA_BF16 if t.dtype == torch.bfloat16 else _lib.FA_FP16


def _split(t, P):
    """P contiguous parts of t along the sequence axis (dim 1)."""
    n = t.shape[1] // P
    return [t[:, i * n:(i + 1) * n].contiguous() for i in range(P)]


def _split_lse(t, P):
    n = t.shape[2] // P
    return [t[:, :, i * n:(i + 1) * n].contiguous() for i in range(P)]


def _fwd_rank(torch, ops, sched, q_parts, held_kv):
    """Forward of one rank: every scheduled (query part, key part) pair attended and merged per query part.

    held_kv(step) -> list of (k, v) parts held at that step.  Returns lists of O and LSE per own part.
    """
    P = len(q_parts)
    remaining = [0] * P
    for _, _, pairs in sched:
        for ia, _, _ in pairs:
            remaining[ia] += 1
    B, n, Hq, d = q_parts[0].shape
    outs = [torch.empty_like(qp) for qp in q_parts]
    lses = [torch.empty(B, Hq, n, device=qp.device, dtype=torch.float32) for qp in q_parts]
    accs = [torch.empty(B, n, Hq, d, device=qp.device, dtype=torch.float32) for qp in q_parts]
    acc_lses = [torch.empty(B, Hq, n, device=qp.device, dtype=torch.float32) for qp in q_parts]
    first = [True] * P
    for s, _, pairs in sched:
        kv = held_kv(s)
        for ia, ib, mode in pairs:
            remaining[ia] -= 1
            m = 0 if first[ia] else (2 if remaining[ia] == 0 else 1)
            ops.attend(q_parts[ia], kv[ib][0], kv[ib][1], mode == "causal", accs[ia], acc_lses[ia], outs[ia],
                       lses[ia], m)
            first[ia] = False
    for ia in range(P):
        if first[ia]:  # no key part attends to these queries (cannot happen for these schedules)
            outs[ia].zero_()
            lses[ia].fill_(-math.inf)
    return outs, lses


def ring_attention_fwd_local(q, k, v, world: int, causal: bool = False, scale: float | None = None,
                             layout: str = "contiguous"):
    """The ring schedule for `world` virtual ranks on one device (no communication).

    q [B, N, Hq, d], k/v [B, N, Hkv, d] of the whole sequence, N divisible by the number of parts;
    returns O, LSE of the whole sequence.
    """
    import torch
    B, N, Hq, d = q.shape
    NP = num_parts(world, layout)
    if N % NP:
        raise ValueError("sequence length must be a multiple of the number of parts")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    ops = _CudaOps(torch, scale)
    qg, kg, vg = _split(q, NP), _split(k, NP), _split(v, NP)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, N, device=q.device, dtype=torch.float32)
    n = N // NP
    for r in range(world):
        mine = owned_parts(r, world, layout)
        sched = ring_schedule(r, world, causal, layout)
        held = lambda s, sched=sched: [(kg[b], vg[b]) for b in owned_parts(sched[s][1], world, layout)]  # noqa: E731
        outs, lses = _fwd_rank(torch, ops, sched, [qg[a] for a in mine], held)
        for ia, a in enumerate(mine):
            out[:, a * n:(a + 1) * n] = outs[ia]
            lse[:, :, a * n:(a + 1) * n] = lses[ia]
    return out, lse


def _p2p(dist, group, nxt, prv, send, recv):
    ops_p2p = [dist.P2POp(dist.isend, t, nxt, group) for t in send] + \
              [dist.P2POp(dist.irecv, t, prv, group) for t in recv]
    return dist.batch_isend_irecv(ops_p2p) if ops_p2p else []


def _neighbours(dist, group, rank, world):
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    if group is not None:
        nxt, prv = dist.get_global_rank(group, nxt), dist.get_global_rank(group, prv)
    return nxt, prv


def ring_attention_fwd(q, k, v, causal: bool = False, scale: float | None = None, group=None, ops=None,
                       layout: str = "contiguous"):
    """Ring attention over a process group; q, k, v are this rank's parts concatenated ([B, n, H, d]).

    Returns this rank's O [B, n, Hq, d] and LSE [B, Hq, n].  `ops` (attend) defaults to the
    library's CUDA kernels; the sends and receives of the keys and values overlap each step's compute.
    """
    import torch
    import torch.distributed as dist
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    P = len(owned_parts(rank, world, layout))
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    ops = ops or _CudaOps(torch, scale)
    sched = ring_schedule(rank, world, causal, layout)
    nxt, prv = _neighbours(dist, group, rank, world)
    q_parts = _split(q, P)
    bufs = [list(zip(_split(k, P), _split(v, P))), [(torch.empty_like(kk), torch.empty_like(vv))
                                                    for kk, vv in zip(_split(k, P), _split(v, P))]]
    pending = {}

    def held(s):
        # the keys and values of step s + 1 start travelling before step s computes
        for r_ in pending.pop(s, []):
            r_.wait()
        if s + 1 < world:
            src, dst = bufs[s % 2], bufs[(s + 1) % 2]
            pending[s + 1] = _p2p(dist, group, nxt, prv, [t for kv in src for t in kv], [t for kv in dst for t in kv])
        return bufs[s % 2]

    outs, lses = _fwd_rank(torch, ops, sched, q_parts, held)
    for reqs in pending.values():
        for r_ in reqs:
            r_.wait()
    return torch.cat(outs, dim=1), torch.cat(lses, dim=2)


def _bwd_rank(torch, ops, sched, qp, op, dop, lp, held, kv_acc):
    """Backward of one rank: dQ sums per own part; the dK/dV contributions of held part ib at step s are
    added into kv_acc(s, ib) -> (dk_acc, dv_acc, init)."""
    P = len(qp)
    wss = [ops.preprocess(qp[i], qp[i], qp[i], op[i], dop[i], lp[i]) for i in range(P)]
    B, n, Hq, d = qp[0].shape
    dq_acc = [torch.empty(B, n, Hq, d, device=qp[0].device, dtype=torch.float32) for _ in range(P)]
    first = [True] * P
    for s, _, pairs in sched:
        kv = held(s)
        for ia, ib, mode in pairs:
            dk_acc, dv_acc, init_kv = kv_acc(s, ib)
            ops.accumulate_bwd(qp[ia], kv[ib][0], kv[ib][1], dop[ia], lp[ia], wss[ia], mode == "causal",
                               dq_acc[ia], dk_acc, dv_acc, first[ia], init_kv)
            first[ia] = False
    dq = [torch.empty_like(x) for x in qp]
    for i in range(P):
        if first[i]:
            dq[i].zero_()
        else:
            ops.cast(dq_acc[i], dq[i])
    return dq


def ring_attention_bwd_local(q, k, v, o, do, lse, world: int, causal: bool = False, scale: float | None = None,
                             layout: str = "contiguous"):
    """The backward ring schedule for `world` virtual ranks on one device (no communication).

    Whole-sequence q, o, do [B, N, Hq, d], k/v [B, N, Hkv, d], lse [B, Hq, N]; returns dQ, dK, dV.
    """
    import torch
    B, N, Hq, d = q.shape
    NP = num_parts(world, layout)
    if N % NP:
        raise ValueError("sequence length must be a multiple of the number of parts")
    n = N // NP
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    ops = _CudaOps(torch, scale)
    qg, kg, vg, og, dog, lg = _split(q, NP), _split(k, NP), _split(v, NP), _split(o, NP), _split(do, NP), \
        _split_lse(lse, NP)
    Hkv = k.shape[2]
    dk_acc = [torch.empty(B, n, Hkv, d, device=q.device, dtype=torch.float32) for _ in range(NP)]
    dv_acc = [torch.empty(B, n, Hkv, d, device=q.device, dtype=torch.float32) for _ in range(NP)]
    kv_first = [True] * NP
    dq = torch.empty_like(q)
    for r in range(world):
        mine = owned_parts(r, world, layout)
        sched = ring_schedule(r, world, causal, layout)

        def held(s, sched=sched):
            return [(kg[b], vg[b]) for b in owned_parts(sched[s][1], world, layout)]

        def kv_acc(s, ib, sched=sched):
            b = owned_parts(sched[s][1], world, layout)[ib]
            init = kv_first[b]
            kv_first[b] = False
            return dk_acc[b], dv_acc[b], init

        dqs = _bwd_rank(torch, ops, sched, [qg[a] for a in mine], [og[a] for a in mine], [dog[a] for a in mine],
                        [lg[a] for a in mine], held, kv_acc)
        for ia, a in enumerate(mine):
            dq[:, a * n:(a + 1) * n] = dqs[ia]
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    for b in range(NP):
        t = torch.empty_like(kg[b])
        if kv_first[b]:
            t.zero_()
            dk[:, b * n:(b + 1) * n] = t
            dv[:, b * n:(b + 1) * n] = t
            continue
        ops.cast(dk_acc[b], t)
        dk[:, b * n:(b + 1) * n] = t
        ops.cast(dv_acc[b], t)
        dv[:, b * n:(b + 1) * n] = t
    return dq, dk, dv


def ring_attention_bwd(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None, group=None,
                       ops=None, layout: str = "contiguous"):
    """Backward of ring_attention_fwd over a process group: this rank's dQ, dK, dV.

    q, o, do [B, n, Hq, d], k/v [B, n, Hkv, d] and lse [B, Hq, n] are this rank's parts (lse as returned by
    ring_attention_fwd: over the whole sequence).  Keys and values travel as in the forward, with the fp32
    dK / dV sums of their parts; after the last step the sums take one more hop to their owner.
    """
    import torch
    import torch.distributed as dist
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    P = len(owned_parts(rank, world, layout))
    B, n, Hq, d = q.shape
    Hkv = k.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    ops = ops or _CudaOps(torch, scale)
    sched = ring_schedule(rank, world, causal, layout)
    nxt, prv = _neighbours(dist, group, rank, world)
    np_ = n // P
    zeros = lambda: torch.zeros(B, np_, Hkv, d, device=q.device, dtype=torch.float32)  # noqa: E731
    kv = [list(zip(_split(k, P), _split(v, P))), [(torch.empty_like(kk), torch.empty_like(vv))
                                                  for kk, vv in zip(_split(k, P), _split(v, P))]]
    acc = [[(zeros(), zeros()) for _ in range(P)], [(zeros(), zeros()) for _ in range(P)]]
    qp, op, dop, lp = _split(q, P), _split(o, P), _split(do, P), _split_lse(lse, P)
    wss = [ops.preprocess(qp[i], qp[i], qp[i], op[i], dop[i], lp[i]) for i in range(P)]
    dq_acc = [torch.empty(B, np_, Hq, d, device=q.device, dtype=torch.float32) for _ in range(P)]
    first = [True] * P
    pending = []
    for s, _, pairs in sched:
        for r_ in pending:
            r_.wait()
        pending = []
        cur_kv = kv[s % 2]
        if s + 1 < world:  # the keys and values of the next step travel while this step computes
            pending = _p2p(dist, group, nxt, prv, [t for x in cur_kv for t in x], [t for x in kv[(s + 1) % 2] for t in x])
        for ia, ib, mode in pairs:
            ops.accumulate_bwd(qp[ia], cur_kv[ib][0], cur_kv[ib][1], dop[ia], lp[ia], wss[ia], mode == "causal",
                               dq_acc[ia], acc[s % 2][ib][0], acc[s % 2][ib][1], first[ia], False)
            first[ia] = False
        if s + 1 < world:
            # the held parts' gradient sums move on with them, after this step's contributions
            for r_ in _p2p(dist, group, nxt, prv, [t for x in acc[s % 2] for t in x],
                           [t for x in acc[(s + 1) % 2] for t in x]):
                r_.wait()
            acc[s % 2] = [(zeros(), zeros()) for _ in range(P)]
    for r_ in pending:
        r_.wait()
    # the sums now held belong to the next rank's parts: one last hop to their owners
    last = acc[(world - 1) % 2]
    if world == 1:
        own = last
    else:
        own = [(zeros(), zeros()) for _ in range(P)]
        for r_ in _p2p(dist, group, nxt, prv, [t for x in last for t in x], [t for x in own for t in x]):
            r_.wait()
    dq_parts = [torch.empty_like(x) for x in qp]
    for i in range(P):
        if first[i]:
            dq_parts[i].zero_()
        else:
            ops.cast(dq_acc[i], dq_parts[i])
    dk_parts = [torch.empty(B, np_, Hkv, d, device=q.device, dtype=k.dtype) for _ in range(P)]
    dv_parts = [torch.empty(B, np_, Hkv, d, device=q.device, dtype=v.dtype) for _ in range(P)]
    for i in range(P):
        ops.cast(own[i][0], dk_parts[i])
        ops.cast(own[i][1], dv_parts[i])
    return torch.cat(dq_parts, dim=1), torch.cat(dk_parts, dim=1), torch.cat(dv_parts, dim=1)
