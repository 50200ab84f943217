"""ctypes binding of liblsh.so: the C ABI of ``include/lsh.h``, same names.

Argument marshalling only: every step of the computation runs in the CUDA
library. Tensor arguments may be torch tensors (their ``data_ptr()`` is
passed) or raw integer device addresses. A missing library raises
``LshLibraryMissing``; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "liblsh.so")

LSH_F32, LSH_BF16 = 0, 1
STATUS_NAMES = {
    0: "LSH_OK", 1: "LSH_ERR_INVALID_ARG", 2: "LSH_ERR_UNSUPPORTED", 3: "LSH_ERR_WORKSPACE",
    4: "LSH_ERR_CUDA", 5: "LSH_ERR_TIMEOUT", 6: "LSH_ERR_DEVICE_CHECK", 7: "LSH_ERR_RANGE",
}
# Every symbol include/lsh.h declares.
EXPORTS = ("lsh_hash", "lsh_sort_workspace_size", "lsh_sort", "lsh_fwd_workspace_size",
           "lsh_attn_fwd", "lsh_bwd_workspace_size", "lsh_attn_bwd", "lsh_device_status",
           "lsh_status_string", "lsh_launch_count", "lsh_sort_noalloc", "lsh_check_wait_timeout",
           "lsh_local_fwd_workspace_size", "lsh_local_attn_fwd", "lsh_local_bwd_workspace_size",
           "lsh_local_attn_bwd", "lsh_ff_workspace_size", "lsh_ff_fwd", "lsh_ff_bwd",
           "lsh_rev_fwd_workspace_size", "lsh_rev_fwd", "lsh_rev_bwd_workspace_size",
           "lsh_rev_bwd")
# Size of the library-owned scratch used by lsh_sort_noalloc (matches lsh.h).
SORT_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


class LshLibraryMissing(RuntimeError):
    pass


class LshError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)} ({status_string(code)})")


class lsh_problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("L", ctypes.c_int32),
                ("d", ctypes.c_int32), ("n_buckets", ctypes.c_int32),
                ("n_rounds", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("causal", ctypes.c_int32), ("scale", ctypes.c_float), ("dtype", ctypes.c_int32)]


class lsh_ff_problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("L", ctypes.c_int32),
                ("d_ff", ctypes.c_int32), ("ff_chunk", ctypes.c_int32)]


def make_ff_problem(B, H, L, d_ff, ff_chunk) -> lsh_ff_problem:
    return lsh_ff_problem(int(B), int(H), int(L), int(d_ff), int(ff_chunk))


def make_problem(B, H, L, d, n_buckets, n_rounds, chunk, causal, scale, dtype) -> lsh_problem:
    if isinstance(dtype, str):
        dtype = {"f32": LSH_F32, "bf16": LSH_BF16}[dtype]
    return lsh_problem(int(B), int(H), int(L), int(d), int(n_buckets), int(n_rounds), int(chunk),
                       int(bool(causal)), float(scale), int(dtype))


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise LshLibraryMissing(
                f"{LIB_PATH} is missing: build it with `python -m efficient_transformer_lsh_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(lsh_problem)
        F = ctypes.POINTER(lsh_ff_problem)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
        sig = {
            "lsh_hash": ([P, vp, vp, vp, vp], ctypes.c_int),
            "lsh_sort_workspace_size": ([P], sz),
            "lsh_sort": ([P, vp, vp, vp, sz, vp], ctypes.c_int),
            "lsh_fwd_workspace_size": ([P], sz),
            "lsh_attn_fwd": ([P, vp, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
            "lsh_bwd_workspace_size": ([P], sz),
            "lsh_attn_bwd": ([P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
            "lsh_device_status": ([vp], ctypes.c_int),
            "lsh_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "lsh_launch_count": ([], ctypes.c_uint64),
            "lsh_sort_noalloc": ([P, vp, vp, vp], ctypes.c_int),
            "lsh_check_wait_timeout": ([ctypes.c_uint64, vp], ctypes.c_int),
            "lsh_local_fwd_workspace_size": ([P, i32, i32], sz),
            "lsh_local_attn_fwd": ([P, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
            "lsh_local_bwd_workspace_size": ([P, i32, i32], sz),
            "lsh_local_attn_bwd": ([P, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
                                   ctypes.c_int),
            "lsh_ff_workspace_size": ([F], sz),
            "lsh_ff_fwd": ([F] + [vp] * 8 + [sz, vp], ctypes.c_int),
            "lsh_ff_bwd": ([F] + [vp] * 15 + [sz, vp], ctypes.c_int),
            "lsh_rev_fwd_workspace_size": ([P, F], sz),
            "lsh_rev_fwd": ([P, F] + [vp] * 11 + [sz, vp], ctypes.c_int),
            "lsh_rev_bwd_workspace_size": ([P, F], sz),
            "lsh_rev_bwd": ([P, F] + [vp] * 18 + [sz, vp], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(code: int, where: str):
    if code != 0:
        raise LshError(code, where)


def status_string(code: int) -> str:
    return lib().lsh_status_string(int(code)).decode()


def lsh_hash(p: lsh_problem, qk, R, bucket, stream=None):
    _check(lib().lsh_hash(ctypes.byref(p), _ptr(qk), _ptr(R), _ptr(bucket), _stream(stream)),
           "lsh_hash")


def lsh_sort_workspace_size(p: lsh_problem) -> int:
    return int(lib().lsh_sort_workspace_size(ctypes.byref(p)))


def lsh_sort(p: lsh_problem, bucket, perm, ws, ws_bytes: int, stream=None):
    _check(lib().lsh_sort(ctypes.byref(p), _ptr(bucket), _ptr(perm), _ptr(ws), int(ws_bytes),
                          _stream(stream)), "lsh_sort")


def lsh_sort_noalloc(p: lsh_problem, bucket, perm, stream=None):
    """lsh_sort for callers that cannot provide a workspace (library-owned scratch)."""
    _check(lib().lsh_sort_noalloc(ctypes.byref(p), _ptr(bucket), _ptr(perm), _stream(stream)),
           "lsh_sort_noalloc")


def lsh_fwd_workspace_size(p: lsh_problem) -> int:
    return int(lib().lsh_fwd_workspace_size(ctypes.byref(p)))


def lsh_attn_fwd(p: lsh_problem, qk, v, perm, out, out_lo, lse, ws, ws_bytes: int, stream=None):
    _check(lib().lsh_attn_fwd(ctypes.byref(p), _ptr(qk), _ptr(v), _ptr(perm), _ptr(out),
                              _ptr(out_lo), _ptr(lse), _ptr(ws), int(ws_bytes), _stream(stream)),
           "lsh_attn_fwd")


def lsh_bwd_workspace_size(p: lsh_problem) -> int:
    return int(lib().lsh_bwd_workspace_size(ctypes.byref(p)))


def lsh_attn_bwd(p: lsh_problem, qk, v, perm, out, out_lo, lse, dout, dqk, dv, ws, ws_bytes: int,
                 stream=None):
    _check(lib().lsh_attn_bwd(ctypes.byref(p), _ptr(qk), _ptr(v), _ptr(perm), _ptr(out),
                              _ptr(out_lo), _ptr(lse), _ptr(dout), _ptr(dqk), _ptr(dv), _ptr(ws),
                              int(ws_bytes), _stream(stream)), "lsh_attn_bwd")


def lsh_local_fwd_workspace_size(p: lsh_problem, n_back: int, n_fwd: int) -> int:
    return int(lib().lsh_local_fwd_workspace_size(ctypes.byref(p), int(n_back), int(n_fwd)))


def lsh_local_attn_fwd(p: lsh_problem, n_back, n_fwd, qk, v, out, out_lo, lse, ws, ws_bytes: int,
                       stream=None):
    _check(lib().lsh_local_attn_fwd(ctypes.byref(p), int(n_back), int(n_fwd), _ptr(qk), _ptr(v),
                                    _ptr(out), _ptr(out_lo), _ptr(lse), _ptr(ws), int(ws_bytes),
                                    _stream(stream)), "lsh_local_attn_fwd")


def lsh_local_bwd_workspace_size(p: lsh_problem, n_back: int, n_fwd: int) -> int:
    return int(lib().lsh_local_bwd_workspace_size(ctypes.byref(p), int(n_back), int(n_fwd)))


def lsh_local_attn_bwd(p: lsh_problem, n_back, n_fwd, qk, v, out, out_lo, lse, dout, dqk, dv, ws,
                       ws_bytes: int, stream=None):
    _check(lib().lsh_local_attn_bwd(ctypes.byref(p), int(n_back), int(n_fwd), _ptr(qk), _ptr(v),
                                    _ptr(out), _ptr(out_lo), _ptr(lse), _ptr(dout), _ptr(dqk),
                                    _ptr(dv), _ptr(ws), int(ws_bytes), _stream(stream)),
           "lsh_local_attn_bwd")


def lsh_ff_workspace_size(f: lsh_ff_problem) -> int:
    return int(lib().lsh_ff_workspace_size(ctypes.byref(f)))


def lsh_ff_fwd(f: lsh_ff_problem, x, W1, b1, W2, b2, res, y, ws, ws_bytes: int, stream=None):
    _check(lib().lsh_ff_fwd(ctypes.byref(f), _ptr(x), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2),
                            _ptr(res), _ptr(y), _ptr(ws), int(ws_bytes), _stream(stream)),
           "lsh_ff_fwd")


def lsh_ff_bwd(f: lsh_ff_problem, x, W1, b1, W2, b2, dy, dres, y_in, rec, dx, dW1, db1, dW2, db2,
               ws, ws_bytes: int, stream=None):
    _check(lib().lsh_ff_bwd(ctypes.byref(f), _ptr(x), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2),
                            _ptr(dy), _ptr(dres), _ptr(y_in), _ptr(rec), _ptr(dx), _ptr(dW1),
                            _ptr(db1), _ptr(dW2), _ptr(db2), _ptr(ws), int(ws_bytes),
                            _stream(stream)), "lsh_ff_bwd")


def lsh_rev_fwd_workspace_size(p: lsh_problem, f: lsh_ff_problem) -> int:
    return int(lib().lsh_rev_fwd_workspace_size(ctypes.byref(p), ctypes.byref(f)))


def lsh_rev_fwd(p: lsh_problem, f: lsh_ff_problem, x1, x2, R, W1, b1, W2, b2, y1, y2, perm, ws,
                ws_bytes: int, stream=None):
    _check(lib().lsh_rev_fwd(ctypes.byref(p), ctypes.byref(f), _ptr(x1), _ptr(x2), _ptr(R),
                             _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), _ptr(y1), _ptr(y2),
                             _ptr(perm), _ptr(ws), int(ws_bytes), _stream(stream)), "lsh_rev_fwd")


def lsh_rev_bwd_workspace_size(p: lsh_problem, f: lsh_ff_problem) -> int:
    return int(lib().lsh_rev_bwd_workspace_size(ctypes.byref(p), ctypes.byref(f)))


def lsh_rev_bwd(p: lsh_problem, f: lsh_ff_problem, y1, y2, dy1, dy2, perm, W1, b1, W2, b2, x1, x2,
                dx1, dx2, dW1, db1, dW2, db2, ws, ws_bytes: int, stream=None):
    _check(lib().lsh_rev_bwd(ctypes.byref(p), ctypes.byref(f), _ptr(y1), _ptr(y2), _ptr(dy1),
                             _ptr(dy2), _ptr(perm), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2),
                             _ptr(x1), _ptr(x2), _ptr(dx1), _ptr(dx2), _ptr(dW1), _ptr(db1),
                             _ptr(dW2), _ptr(db2), _ptr(ws), int(ws_bytes), _stream(stream)),
           "lsh_rev_bwd")


def lsh_device_status(stream=None) -> int:
    return int(lib().lsh_device_status(_stream(stream)))


def lsh_check_wait_timeout(limit_ns: int, stream=None):
    """Runs the bounded-wait failure path once (see lsh.h); read the result
    with lsh_device_status()."""
    _check(lib().lsh_check_wait_timeout(int(limit_ns), _stream(stream)), "lsh_check_wait_timeout")


def lsh_launch_count() -> int:
    return int(lib().lsh_launch_count())
