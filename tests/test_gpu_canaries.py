"""Bounds evidence for the output writes, with no sanitizer: guard canaries.

Every output a kernel writes is placed inside a larger device buffer whose
other bytes hold a sentinel pattern; after the call the sentinel bytes before
and after the output must be intact (a ragged-tail store that ran past the end
of O, LSE, dQ, dK, dV, the decode partials, the FP8 codes or the fp32
accumulators would overwrite them).  The cases are the ragged ones: Nq, Nk not
multiples of 128, a single query row, block-sparse tables with empty rows of
blocks (whose O rows the kernel writes directly), GQA groups, d = 64 and 128.
Inputs get sentinels too, so a stray write into an input is also caught.
Every call goes through the C ABI with pointers into the guarded buffers.
"""
import math

import pytest

import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GUARD = 64 * 1024  # bytes of sentinel on each side of every tensor
SENTINEL = 0xA5


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_io_aware_80_b200 import _lib
    _lib.load()
    return _lib


class Guarded:
    """A tensor of `shape` / `dtype` living at byte GUARD of a sentinel-filled buffer."""

    def __init__(self, shape, dtype, fill=None):
        n = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
        self.nbytes = n
        self.buf = torch.full((GUARD + (n + 15) // 16 * 16 + GUARD,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.t = self.buf[GUARD:GUARD + n].view(dtype).view(shape)
        if fill is not None:
            self.t.copy_(fill)

    def ptr(self):
        return self.t.data_ptr()

    def intact(self):
        torch.cuda.synchronize()
        pad = self.buf[GUARD + self.nbytes:]
        return bool((self.buf[:GUARD] == SENTINEL).all()) and bool((pad == SENTINEL).all())


def _dt(lib, t):
    return lib.FA_BF16 if t.dtype == torch.bfloat16 else lib.FA_FP16


def _stream():
    return torch.cuda.current_stream().cuda_stream


FWD_CASES = [
    # B, Hq, Hkv, Nq, Nk, d, dtype, causal
    (1, 2, 1, 1, 77, 128, torch.bfloat16, True),
    (2, 4, 2, 333, 451, 128, torch.bfloat16, False),
    (1, 4, 4, 129, 129, 64, torch.float16, True),
    (3, 6, 3, 65, 300, 64, torch.bfloat16, False),
    (1, 8, 2, 700, 700, 128, torch.float16, True),
]


def _inputs(B, Hq, Hkv, Nq, Nk, d, dt, seed):
    q, k, v, do = workloads.make_inputs(B, Hq, Hkv, Nq, Nk, d, dt, seed_base=seed, with_do=True)
    return (Guarded(q.shape, dt, q.cuda()), Guarded(k.shape, dt, k.cuda()), Guarded(v.shape, dt, v.cuda()),
            Guarded(do.shape, dt, do.cuda()))


@pytest.mark.parametrize("case", FWD_CASES)
def test_forward_and_backward_stay_inside_their_outputs(lib, case):
    B, Hq, Hkv, Nq, Nk, d, dt, causal = case
    q, k, v, do = _inputs(B, Hq, Hkv, Nq, Nk, d, dt, 17 * Nq + Nk)
    o = Guarded((B, Nq, Hq, d), dt)
    lse = Guarded((B, Hq, Nq), torch.float32)
    s = 1 / math.sqrt(d)
    lib.fa_fwd(q.ptr(), k.ptr(), v.ptr(), o.ptr(), lse.ptr(), B, Hq, Hkv, Nq, Nk, d, causal, s, _dt(lib, q.t),
               _stream())
    dq, dk, dv = Guarded((B, Nq, Hq, d), dt), Guarded((B, Nk, Hkv, d), dt), Guarded((B, Nk, Hkv, d), dt)
    ws = Guarded((B * Hq * Nq,), torch.float32)
    lib.fa_bwd(q.ptr(), k.ptr(), v.ptr(), o.ptr(), do.ptr(), lse.ptr(), dq.ptr(), dk.ptr(), dv.ptr(), ws.ptr(), B, Hq,
               Hkv, Nq, Nk, d, causal, s, _dt(lib, q.t), _stream())
    assert lib.fa_get_device_status(_stream()) == 0
    for name, g in (("q", q), ("k", k), ("v", v), ("do", do), ("o", o), ("lse", lse), ("dq", dq), ("dk", dk),
                    ("dv", dv), ("D", ws)):
        assert g.intact(), name
    assert torch.isfinite(o.t.float()).all() and torch.isfinite(dq.t.float()).all()


@pytest.mark.parametrize("case", FWD_CASES[:3])
def test_dropout_stays_inside_its_outputs(lib, case):
    B, Hq, Hkv, Nq, Nk, d, dt, causal = case
    q, k, v, do = _inputs(B, Hq, Hkv, Nq, Nk, d, dt, 23 * Nq + Nk)
    o, lse = Guarded((B, Nq, Hq, d), dt), Guarded((B, Hq, Nq), torch.float32)
    s = 1 / math.sqrt(d)
    lib.fa_fwd_dropout(q.ptr(), k.ptr(), v.ptr(), o.ptr(), lse.ptr(), B, Hq, Hkv, Nq, Nk, d, causal, s, 0.2, 99, 1,
                       _dt(lib, q.t), _stream())
    dq, dk, dv = Guarded((B, Nq, Hq, d), dt), Guarded((B, Nk, Hkv, d), dt), Guarded((B, Nk, Hkv, d), dt)
    ws = Guarded((B * Hq * Nq,), torch.float32)
    lib.fa_bwd_dropout(q.ptr(), k.ptr(), v.ptr(), o.ptr(), do.ptr(), lse.ptr(), dq.ptr(), dk.ptr(), dv.ptr(), ws.ptr(),
                       B, Hq, Hkv, Nq, Nk, d, causal, s, 0.2, 99, 1, _dt(lib, q.t), _stream())
    assert lib.fa_get_device_status(_stream()) == 0
    for name, g in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv), ("D", ws)):
        assert g.intact(), name


@pytest.mark.parametrize("Nq,Nk,causal,density", [(333, 451, False, 0.4), (300, 300, True, 0.5), (1, 200, True, 1.0),
                                                  (520, 129, False, 0.0)])
def test_blocksparse_empty_rows_stay_inside_their_outputs(lib, Nq, Nk, causal, density):
    """Query tiles with no marked block take the direct-write path for O and LSE."""
    B, Hq, Hkv, d, dt = 2, 4, 2, 128, torch.bfloat16
    q, k, v, _ = _inputs(B, Hq, Hkv, Nq, Nk, d, dt, 29 * Nq + Nk)
    nqb, nkb = -(-Nq // 128), -(-Nk // 128)
    mask = workloads.block_mask_random(B, Hq, nqb, nkb, density, seed=Nq + Nk)
    mask[:, :, 0] = 0  # the first query tile of every head sees nothing
    bm = Guarded(mask.shape, torch.uint8, mask.cuda())
    o, lse = Guarded((B, Nq, Hq, d), dt), Guarded((B, Hq, Nq), torch.float32)
    lib.fa_fwd_blocksparse(q.ptr(), k.ptr(), v.ptr(), o.ptr(), lse.ptr(), bm.ptr(), B, Hq, Hkv, Nq, Nk, d, causal,
                           1 / math.sqrt(d), _dt(lib, q.t), _stream())
    assert lib.fa_get_device_status(_stream()) == 0
    for name, g in (("o", o), ("lse", lse), ("mask", bm), ("q", q)):
        assert g.intact(), name
    assert (o.t[:, :min(Nq, 128)] == 0).all()


@pytest.mark.parametrize("splits", [1, 5, 0])
def test_decode_stays_inside_partials_and_outputs(lib, splits):
    B, Hq, Hkv, N, d = 5, 8, 2, 1000, 128
    qc, kc, vc, _ = workloads.make_decode_inputs(B, Hq, Hkv, N, d, torch.bfloat16, seed_base=31)
    q, k, v = (Guarded(t.shape, torch.bfloat16, t.cuda()) for t in (qc, kc, vc))
    sl = Guarded((B,), torch.int32, torch.tensor([1000, 1, 0, 999, 64], dtype=torch.int32).cuda())
    S = splits if splits > 0 else lib.fa_decode_num_splits(B, Hkv, N, d, 0)
    ws = Guarded((lib.fa_decode_workspace_bytes(B, Hq, S, d),), torch.uint8)
    o, lse = Guarded((B, 1, Hq, d), torch.bfloat16), Guarded((B, Hq, 1), torch.float32)
    lib.fa_decode_splitkv(q.ptr(), k.ptr(), v.ptr(), sl.ptr(), B, Hq, Hkv, N, d, d ** -0.5, S, ws.ptr(), lib.FA_BF16,
                          _stream())
    lib.fa_decode_combine(ws.ptr(), o.ptr(), lse.ptr(), sl.ptr(), B, Hq, S, d, lib.FA_BF16, _stream())
    assert lib.fa_get_device_status(_stream()) == 0
    for name, g in (("ws", ws), ("o", o), ("lse", lse), ("k", k), ("sl", sl)):
        assert g.intact(), name


@pytest.mark.parametrize("d,Nq,Nk", [(128, 300, 77), (64, 1, 129)])
def test_fp8_quantizers_stay_inside_codes_and_scales(lib, d, Nq, Nk):
    B, Hq, Hkv = 2, 4, 2
    q, k, v, _ = _inputs(B, Hq, Hkv, Nq, Nk, d, torch.bfloat16, 37 * Nq + Nk)
    signs = Guarded((d,), torch.float32, workloads.rotation_signs(d, 5).cuda())
    npad = (Nk + 15) // 16 * 16
    q8, k8, v8t = Guarded((B, Nq, Hq, d), torch.uint8), Guarded((B, Nk, Hkv, d), torch.uint8), \
        Guarded((B, Hkv, d, npad), torch.uint8)
    qs, ks, vs = Guarded((B, Hq, -(-Nq // 128)), torch.float32), Guarded((B, Hkv, -(-Nk // 128)), torch.float32), \
        Guarded((B, Hkv), torch.float32)
    ws = Guarded((lib.fa_fp8_v_workspace_bytes(B, Hkv, Nk),), torch.uint8)
    lib.fa_fp8_quantize_qkv(q.ptr(), k.ptr(), v.ptr(), q8.ptr(), k8.ptr(), v8t.ptr(), qs.ptr(), ks.ptr(), vs.ptr(),
                            signs.ptr(), ws.ptr(), B, Hq, Hkv, Nq, Nk, d, lib.FA_BF16, _stream())
    assert lib.fa_get_device_status(_stream()) == 0
    for name, g in (("q8", q8), ("k8", k8), ("v8t", v8t), ("qs", qs), ("ks", ks), ("vs", vs), ("ws", ws),
                    ("v", v)):
        assert g.intact(), name


def test_fp32_accumulator_paths_stay_inside(lib):
    B, Hq, Hkv, Nq, Nk, d, dt = 1, 4, 2, 200, 333, 128, torch.bfloat16
    q, k, v, do = _inputs(B, Hq, Hkv, Nq, Nk, d, dt, 41)
    s = 1 / math.sqrt(d)
    o, lse = Guarded((B, Nq, Hq, d), dt), Guarded((B, Hq, Nq), torch.float32)
    acc_o, acc_l = Guarded((B, Nq, Hq, d), torch.float32), Guarded((B, Hq, Nq), torch.float32)
    for mode in (0, 1, 2):
        lib.fa_fwd_merge(q.ptr(), k.ptr(), v.ptr(), o.ptr(), lse.ptr(), acc_o.ptr(), acc_l.ptr(), mode, B, Hq, Hkv,
                         Nq, Nk, d, True, s, lib.FA_BF16, _stream())
    ws = Guarded((B * Hq * Nq,), torch.float32)
    lib.fa_bwd_preprocess(0, 0, 0, o.ptr(), do.ptr(), 0, 0, 0, 0, ws.ptr(), B, Hq, Hkv, Nq, Nk, d, 0, 1.0,
                          lib.FA_BF16, _stream())
    dq = Guarded((B, Nq, Hq, d), torch.float32)
    dk, dv = Guarded((B, Nk, Hkv, d), torch.float32), Guarded((B, Nk, Hkv, d), torch.float32)
    for init in (3, 0):
        lib.fa_bwd_accumulate(q.ptr(), k.ptr(), v.ptr(), do.ptr(), lse.ptr(), ws.ptr(), dq.ptr(), dk.ptr(), dv.ptr(),
                              init, B, Hq, Hkv, Nq, Nk, d, True, s, lib.FA_BF16, _stream())
    assert lib.fa_get_device_status(_stream()) == 0
    for name, g in (("o", o), ("lse", lse), ("acc_o", acc_o), ("acc_l", acc_l), ("dq", dq), ("dk", dk), ("dv", dv),
                    ("ws", ws)):
        assert g.intact(), name
