"""Host-side checks of libfa.so that need no GPU: the library loads, exports
every entry point include/fa.h declares, and validation rejects bad
arguments before anything is launched (so fake pointers are never touched)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module")
def lib():
    from exact_io_aware_80_b200 import build, _lib
    build.build()
    return _lib.load()


def declared_functions():
    with open(HEADER) as fh:
        src = fh.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(fa_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("fa_fwd", "fa_bwd", "fa_decode_splitkv", "fa_decode_combine", "fa_get_device_status"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    from exact_io_aware_80_b200 import _lib
    for n in declared_functions():
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, f"binding lacks {n}"


def test_checking_build_exports_the_same_boundary():
    """libfa_checks.so (FA_CHECKS: device-side index checks) has every entry point too."""
    from exact_io_aware_80_b200 import build
    path = build.build(checks=True)
    chk = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(chk, n), n
    chk.fa_status_string.restype = ctypes.c_char_p
    assert chk.fa_status_string(-6) == b"device-side index check failed"


def test_status_strings_and_version(lib):
    from exact_io_aware_80_b200 import _lib
    assert _lib.fa_version() >= 1
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert _lib.status_string(code)
        assert _lib.status_string(code) != "unknown status"


def test_workspace_sizes(lib):
    from exact_io_aware_80_b200 import _lib
    assert _lib.fa_bwd_workspace_bytes(1, 32, 8192) == 32 * 8192 * 4
    ws = _lib.fa_decode_workspace_bytes(64, 32, 16, 128)
    assert ws >= 64 * 32 * 16 * 128 * 4 + 64 * 32 * 16 * 4
    assert ws % 16 == 0


def test_decode_chunk_and_splits(lib):
    from exact_io_aware_80_b200 import _lib
    assert _lib.fa_decode_chunk(32768, 16) == 2048
    assert _lib.fa_decode_chunk(1000, 3) == 384
    for B, Hkv, N in ((64, 8, 32768), (1, 1, 1), (1, 8, 100000), (256, 8, 512)):
        s = _lib.fa_decode_num_splits(B, Hkv, N, 128, 148)
        assert 1 <= s <= -(-N // 64)
        # the last split must not start past the cache
        assert (s - 1) * _lib.fa_decode_chunk(N, s) < N or s == 1


FAKE = 0x10000  # never dereferenced: validation fails first


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), -1),
    (dict(Hq=6, Hkv=4), -1),
    (dict(causal=1, Nq=10, Nk=5), -1),
    (dict(d=96), -2),
    (dict(d=256), -2),
    (dict(dt=7), -2),
    (dict(B=0), -1),
    (dict(Nq=0), -1),
    (dict(Nk=0), -1),
    (dict(Hkv=0), -1),
    (dict(Nq=(1 << 30) + 1, Nk=(1 << 30) + 1), -2),
    (dict(B=65536), -2),
    (dict(q=FAKE + 8), -3),
])
def test_fwd_rejects_bad_arguments(lib, kw, code):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=4, Hkv=2, Nq=8, Nk=8, d=128, causal=0,
             scale=0.1, dt=1, stream=None)
    a.update(kw)
    rc = lib.fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"],
                    a["d"], a["causal"], a["scale"], a["dt"], a["stream"])
    assert rc == code


def test_bwd_rejects_bad_arguments(lib):
    # only invalid argument lists are passed: a valid one would launch on fake pointers
    args = [FAKE] * 10 + [1, 4, 2, 8, 8, 128, 0, 0.1, 1, None]
    bad = list(args)
    bad[9] = None  # workspace
    assert lib.fa_bwd(*bad) == -1
    bad = list(args)
    bad[15] = 80  # d
    assert lib.fa_bwd(*bad) == -2
    bad = list(args)
    bad[3] = FAKE + 4  # o misaligned
    assert lib.fa_bwd(*bad) == -3


def test_decode_rejects_bad_arguments(lib):
    # q, kc, vc, seqlens, B, Hq, Hkv, Nk_max, d, scale, splits, ws, dt, stream
    base = [FAKE, FAKE, FAKE, FAKE, 2, 32, 8, 1024, 128, 0.1, 4, FAKE, 1, None]
    bad = list(base)
    bad[5] = 33  # Hq % Hkv
    assert lib.fa_decode_splitkv(*bad) == -1
    bad = list(base)
    bad[5], bad[6] = 64, 2  # group of 32 > 16
    assert lib.fa_decode_splitkv(*bad) == -2
    bad = list(base)
    bad[10] = 17  # more splits than 64-key tiles
    assert lib.fa_decode_splitkv(*bad) == -1
    bad = list(base)
    bad[3] = FAKE + 2  # seqlens misaligned
    assert lib.fa_decode_splitkv(*bad) == -3
    assert lib.fa_decode_combine(FAKE, FAKE, FAKE, FAKE, 2, 32, 0, 128, 1, None) == -1
    assert lib.fa_decode_combine(FAKE, FAKE, FAKE, FAKE, 2, 32, 4, 72, 1, None) == -2


def test_binding_without_gpu_fails_loudly():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    import exact_io_aware_80_b200 as fa
    q = torch.zeros(1, 8, 2, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        fa.attention_fwd(q, q, q)


def test_fp8_entry_points_reject_bad_arguments(lib):
    from exact_io_aware_80_b200 import _lib
    assert _lib.fa_fp8_v_workspace_bytes(2, 8, 300) == 2 * 8 * 3 * 4
    assert _lib.fa_fp8_v_workspace_bytes(0, 8, 300) == 0
    # x, x8, scales, signs, B, H, N, d, dt, stream
    assert lib.fa_fp8_quantize_qk(0, FAKE, FAKE, 0, 1, 2, 8, 128, 1, None) == -1
    assert lib.fa_fp8_quantize_qk(FAKE, FAKE, FAKE, 0, 1, 2, 8, 96, 1, None) == -2
    assert lib.fa_fp8_quantize_qk(FAKE + 8, FAKE, FAKE, 0, 1, 2, 8, 128, 1, None) == -3
    assert lib.fa_fp8_quantize_qk(FAKE, FAKE, FAKE, FAKE + 2, 1, 2, 8, 128, 1, None) == -3
    assert lib.fa_fp8_quantize_v(FAKE, FAKE, FAKE, 0, 1, 2, 8, 128, 1, None) == -1
    assert lib.fa_fp8_quantize_v(FAKE, FAKE, FAKE, FAKE, 1, 2, 0, 128, 1, None) == -1
    # q, k, v, q8, k8, v8t, qs, ks, vs, signs, ws, B, Hq, Hkv, Nq, Nk, d, dt, stream
    qkv = [FAKE] * 9 + [0, FAKE, 1, 4, 2, 8, 8, 128, 1, None]
    for idx, val, code in ((0, 0, -1), (10, 0, -1), (12, 5, -1), (16, 96, -2), (17, 7, -2), (3, FAKE + 8, -3),
                           (6, FAKE + 2, -3), (9, FAKE + 2, -3), (14, 0, -1)):
        bad = list(qkv)
        bad[idx] = val
        assert lib.fa_fp8_quantize_qkv(*bad) == code, (idx, val)
    # q8, qs, k8, ks, v8t, vs, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, rotated, dt, stream
    base = [FAKE] * 8 + [1, 4, 2, 8, 8, 128, 0, 0.1, 0, 1, None]
    bad = list(base)
    bad[13] = 64  # the FP8 forward takes d = 128 only
    assert lib.fa_fwd_fp8(*bad) == -2
    bad = list(base)
    bad[9] = 5  # Hq % Hkv
    assert lib.fa_fwd_fp8(*bad) == -1
    bad = list(base)
    bad[1] = 0  # q_scale
    assert lib.fa_fwd_fp8(*bad) == -1
    bad = list(base)
    bad[4] = FAKE + 4  # v8t misaligned
    assert lib.fa_fwd_fp8(*bad) == -3


def test_blocksparse_rejects_bad_arguments(lib):
    # q, k, v, o, lse, mask, B, Hq, Hkv, Nq, Nk, d, causal, scale, dt, stream
    base = [FAKE] * 6 + [1, 4, 2, 8, 8, 128, 0, 0.1, 1, None]
    bad = list(base)
    bad[5] = 0  # no mask
    assert lib.fa_fwd_blocksparse(*bad) == -1
    bad = list(base)
    bad[11] = 80
    assert lib.fa_fwd_blocksparse(*bad) == -2
    bad = list(base)
    bad[0] = FAKE + 2
    assert lib.fa_fwd_blocksparse(*bad) == -3


def test_dropout_rejects_bad_arguments(lib):
    # q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, p, seed, offset, dt, stream
    base = [FAKE] * 5 + [1, 4, 2, 8, 8, 128, 0, 0.1, 0.25, 7, 0, 1, None]
    for p in (1.0, -0.1, float("nan")):
        bad = list(base)
        bad[13] = p
        assert lib.fa_fwd_dropout(*bad) == -1
    bad = list(base)
    bad[10] = 96
    assert lib.fa_fwd_dropout(*bad) == -2
    bwd = [FAKE] * 10 + [1, 4, 2, 8, 8, 128, 0, 0.1, 1.5, 7, 0, 1, None]
    assert lib.fa_bwd_dropout(*bwd) == -1
    bwd[18] = 0.2
    bwd[9] = None  # workspace
    assert lib.fa_bwd_dropout(*bwd) == -1


def test_lse_merge_rejects_bad_arguments(lib):
    # o_acc, lse_acc, o_part, lse_part, o_out, B, N, H, d, mode, dt, stream
    assert lib.fa_lse_merge(FAKE, FAKE, FAKE, FAKE, 0, 1, 8, 2, 128, 2, 1, None) == -1  # mode 2 needs o_out
    assert lib.fa_lse_merge(FAKE, FAKE, FAKE, FAKE, 0, 1, 8, 2, 128, 3, 1, None) == -1
    assert lib.fa_lse_merge(FAKE, FAKE, FAKE, FAKE, 0, 1, 8, 2, 96, 1, 1, None) == -2
    assert lib.fa_lse_merge(FAKE + 4, FAKE, FAKE, FAKE, 0, 1, 8, 2, 128, 1, 1, None) == -3


def test_accumulate_and_cast_reject_bad_arguments(lib):
    assert lib.fa_accumulate(FAKE, FAKE, 12, 1, 1, None) == -1      # n not a multiple of 8
    assert lib.fa_accumulate(0, FAKE, 16, 1, 1, None) == -1
    assert lib.fa_accumulate(FAKE + 4, FAKE, 16, 1, 1, None) == -3
    assert lib.fa_cast_f32(FAKE, FAKE, 16, 5, None) == -2
    assert lib.fa_cast_f32(FAKE, FAKE + 2, 16, 1, None) == -3
