"""ctypes binding of libfa.so -- argument marshalling only.

Every function here has the name of the C entry point it calls (declared in
include/fa.h) and forwards plain pointers, sizes and a CUDA stream handle.
There is no fallback: if libfa.so is missing or fails to load, every call
raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# FA_LIBRARY selects another build of the same ABI, e.g. libfa_checks.so (device-side
# index checks): a file name inside this package or an absolute path.
LIB_PATH = os.path.join(_HERE, os.environ.get("FA_LIBRARY", "libfa.so"))

FA_OK = 0
FA_ERR_INVALID = -1
FA_ERR_UNSUPPORTED = -2
FA_ERR_ALIGN = -3
FA_ERR_CUDA = -4
FA_ERR_TIMEOUT = -5
FA_ERR_BOUNDS = -6
FA_FP16 = 0
FA_BF16 = 1

# name -> (restype, argtypes), mirroring include/fa.h
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
SIGNATURES = {
    "fa_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_bwd_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I]),
    "fa_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_bwd_preprocess": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_bwd_dkdv": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_bwd_dq": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_decode_num_splits": (_I, [_I, _I, _I, _I, _I]),
    "fa_decode_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "fa_decode_splitkv": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P, _I, _P]),
    "fa_decode_combine": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "fa_decode_chunk": (_I, [_I, _I]),
    "fa_decode_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "fa_fwd_blocksparse": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_fwd_dropout": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F, ctypes.c_uint64, ctypes.c_uint32,
                            _I, _P]),
    "fa_bwd_dropout": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F,
                            ctypes.c_uint64, ctypes.c_uint32, _I, _P]),
    "fa_fp8_quantize_qk": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "fa_fp8_v_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I]),
    "fa_fp8_quantize_v": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "fa_fp8_quantize_qkv": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P]),
    "fa_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "fa_fwd_merge": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_bwd_accumulate": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_lse_merge": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "fa_accumulate": (_I, [_P, _P, ctypes.c_longlong, _I, _I, _P]),
    "fa_cast_f32": (_I, [_P, _P, ctypes.c_longlong, _I, _P]),
    "fa_get_device_status": (_I, [_P]),
    "fa_watchdog_selftest": (_I, [_I, _P]),
    "fa_status_string": (ctypes.c_char_p, [_I]),
    "fa_version": (_I, []),
}

_lib = None


class FAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfa.so (once) and attach the signatures.  Raises if it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(f"{path} is not built: run `python -m exact_io_aware_80_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def status_string(code: int) -> str:
    return load().fa_status_string(code).decode()


def _check(fn: str, code: int) -> int:
    if code != FA_OK:
        raise FAError(fn, code)
    return code


def fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, dt, stream):
    return _check("fa_fwd", load().fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, int(causal), scale, dt, stream))


def fa_bwd_workspace_bytes(B, Hq, Nq):
    return load().fa_bwd_workspace_bytes(B, Hq, Nq)


def fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, causal, scale, dt, stream):
    return _check("fa_bwd", load().fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d,
                                          int(causal), scale, dt, stream))


def fa_bwd_preprocess(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, causal, scale, dt,
                      stream):
    return _check("fa_bwd_preprocess", load().fa_bwd_preprocess(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq,
                                                                Hkv, Nq, Nk, d, int(causal), scale, dt, stream))


def fa_bwd_dkdv(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, causal, scale, dt, stream):
    return _check("fa_bwd_dkdv", load().fa_bwd_dkdv(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq,
                                                    Nk, d, int(causal), scale, dt, stream))


def fa_bwd_dq(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, causal, scale, dt, stream):
    return _check("fa_bwd_dq", load().fa_bwd_dq(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk,
                                                d, int(causal), scale, dt, stream))


def fa_decode_num_splits(B, Hkv, Nk_max, d, num_sms=0):
    return load().fa_decode_num_splits(B, Hkv, Nk_max, d, num_sms)


def fa_decode_workspace_bytes(B, Hq, num_splits, d):
    return load().fa_decode_workspace_bytes(B, Hq, num_splits, d)


def fa_decode_chunk(Nk_max, num_splits):
    return load().fa_decode_chunk(Nk_max, num_splits)


def fa_decode_splitkv(q, k_cache, v_cache, seqlens_k, B, Hq, Hkv, Nk_max, d, scale, num_splits, workspace, dt,
                      stream):
    return _check("fa_decode_splitkv", load().fa_decode_splitkv(q, k_cache, v_cache, seqlens_k, B, Hq, Hkv, Nk_max,
                                                                d, scale, num_splits, workspace, dt, stream))


def fa_decode_combine(workspace, o, lse, seqlens_k, B, Hq, num_splits, d, dt, stream):
    return _check("fa_decode_combine", load().fa_decode_combine(workspace, o, lse, seqlens_k, B, Hq, num_splits, d,
                                                                dt, stream))


def fa_fwd_dropout(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, p_drop, seed, offset, dt, stream):
    return _check("fa_fwd_dropout", load().fa_fwd_dropout(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, int(causal), scale,
                                                          p_drop, seed, offset, dt, stream))


def fa_bwd_dropout(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, causal, scale, p_drop, seed,
                   offset, dt, stream):
    return _check("fa_bwd_dropout", load().fa_bwd_dropout(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq,
                                                          Nk, d, int(causal), scale, p_drop, seed, offset, dt,
                                                          stream))


def fa_fwd_blocksparse(q, k, v, o, lse, block_mask, B, Hq, Hkv, Nq, Nk, d, causal, scale, dt, stream):
    return _check("fa_fwd_blocksparse", load().fa_fwd_blocksparse(q, k, v, o, lse, block_mask, B, Hq, Hkv, Nq, Nk, d,
                                                                  int(causal), scale, dt, stream))


def fa_fp8_quantize_qk(x, x8, scales, signs, B, H, N, d, dt, stream):
    return _check("fa_fp8_quantize_qk", load().fa_fp8_quantize_qk(x, x8, scales, signs, B, H, N, d, dt, stream))


def fa_fp8_v_workspace_bytes(B, Hkv, Nk):
    return load().fa_fp8_v_workspace_bytes(B, Hkv, Nk)


def fa_fp8_quantize_v(v, v8t, scale, workspace, B, Hkv, Nk, d, dt, stream):
    return _check("fa_fp8_quantize_v", load().fa_fp8_quantize_v(v, v8t, scale, workspace, B, Hkv, Nk, d, dt, stream))


def fa_fp8_quantize_qkv(q, k, v, q8, k8, v8t, q_scale, k_scale, v_scale, signs, workspace, B, Hq, Hkv, Nq, Nk, d, dt,
                        stream):
    return _check("fa_fp8_quantize_qkv", load().fa_fp8_quantize_qkv(q, k, v, q8, k8, v8t, q_scale, k_scale, v_scale,
                                                                    signs, workspace, B, Hq, Hkv, Nq, Nk, d, dt,
                                                                    stream))


def fa_fwd_fp8(q8, q_scale, k8, k_scale, v8t, v_scale, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, rotated, dt,
               stream):
    return _check("fa_fwd_fp8", load().fa_fwd_fp8(q8, q_scale, k8, k_scale, v8t, v_scale, o, lse, B, Hq, Hkv, Nq, Nk,
                                                  d, int(causal), scale, int(rotated), dt, stream))


def fa_fwd_merge(q, k, v, o, lse, acc_o, acc_lse, mode, B, Hq, Hkv, Nq, Nk, d, causal, scale, dt, stream):
    return _check("fa_fwd_merge", load().fa_fwd_merge(q, k, v, o, lse, acc_o, acc_lse, mode, B, Hq, Hkv, Nq, Nk, d,
                                                      int(causal), scale, dt, stream))


def fa_bwd_accumulate(q, k, v, dout, lse, workspace, dq_acc, dk_acc, dv_acc, init, B, Hq, Hkv, Nq, Nk, d, causal,
                      scale, dt, stream):
    return _check("fa_bwd_accumulate", load().fa_bwd_accumulate(q, k, v, dout, lse, workspace, dq_acc, dk_acc, dv_acc,
                                                                init, B, Hq, Hkv, Nq, Nk, d, int(causal), scale, dt,
                                                                stream))


def fa_lse_merge(o_acc, lse_acc, o_part, lse_part, o_out, B, N, H, d, mode, dt, stream):
    return _check("fa_lse_merge", load().fa_lse_merge(o_acc, lse_acc, o_part, lse_part, o_out, B, N, H, d, mode, dt,
                                                      stream))


def fa_accumulate(acc, part, n, init, dt, stream):
    return _check("fa_accumulate", load().fa_accumulate(acc, part, n, int(init), dt, stream))


def fa_cast_f32(acc, out, n, dt, stream):
    return _check("fa_cast_f32", load().fa_cast_f32(acc, out, n, dt, stream))


def fa_watchdog_selftest(limit_us, stream):
    return _check("fa_watchdog_selftest", load().fa_watchdog_selftest(limit_us, stream))


def fa_get_device_status(stream):
    return load().fa_get_device_status(stream)


def fa_version():
    return load().fa_version()
