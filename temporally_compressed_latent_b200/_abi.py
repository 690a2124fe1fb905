"""ctypes binding of libmtla.so: the C ABI of include/mtla.h, same names.

Arguments are torch tensors (their device pointer is passed), plain integers
(taken as raw pointers) or None (NULL).  Nothing here computes any part of the
method; every call goes straight to the library, asynchronously on the current
CUDA stream unless ``stream`` is given.
"""
from __future__ import annotations

import ctypes
import os
import re

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmtla.so")
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "mtla.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is not built; run `python temporally_compressed_latent_b200/build_lib.py` "
        "(the MTLA hot path has no fallback)")

lib = ctypes.CDLL(LIB_PATH)

MTLA_F32, MTLA_BF16 = 0, 1
WS_DECODE = 0
PROJ_IN, PROJ_OUT = 1, 2
TRAIN_ATTN_BWD, TRAIN_KV_BWD, TRAIN_MERGE_BWD = 1, 2, 3  # MTLA_TRAIN_*
DECODE_STATIC_SCRATCH_BYTES = 24 << 20  # MTLA_DECODE_STATIC_SCRATCH_BYTES
MAX_NEW_TOKENS = 16  # MTLA_MAX_NEW_TOKENS
DEVERR_PE_RANGE, DEVERR_CAPACITY, DEVERR_EMPTY, DEVERR_TIMEOUT = 1, 2, 4, 8
_c = ctypes


class _Dims(_c.Structure):
    _fields_ = [("H", _c.c_int32), ("d_h", _c.c_int32), ("r", _c.c_int32), ("d_R", _c.c_int32),
                ("s", _c.c_int32), ("dtype", _c.c_int32)]


class _Merge(_c.Structure):
    _fields_ = [("c_new", _c.c_void_p), ("kR_new", _c.c_void_p), ("W_c", _c.c_void_p), ("b_c", _c.c_void_p),
                ("P", _c.c_void_p), ("J_max", _c.c_int32)]


_P = _c.c_void_p
_I32, _I64, _SZ = _c.c_int32, _c.c_int64, _c.c_size_t
_DIMS_P, _MERGE_P = _c.POINTER(_Dims), _c.POINTER(_Merge)

lib.mtla_merge_append.restype = _c.c_int
lib.mtla_merge_append.argtypes = [_DIMS_P, _I32, _MERGE_P, _P, _I64, _I64, _P, _P, _P, _P, _P, _P]
lib.mtla_decode_attn.restype = _c.c_int
lib.mtla_decode_attn.argtypes = [_DIMS_P, _I32, _P, _P, _MERGE_P, _P, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _SZ,
                                 _P, _P]
lib.mtla_decode_attn_static.restype = _c.c_int
lib.mtla_decode_attn_static.argtypes = [_DIMS_P, _I32, _P, _P, _MERGE_P, _P, _I64, _I64, _P, _P, _P, _P, _P, _P, _P,
                                        _P]
lib.mtla_prefill_masked_attn.restype = _c.c_int
lib.mtla_prefill_masked_attn.argtypes = [_DIMS_P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _P, _P, _P]
lib.mtla_workspace_bytes.restype = _SZ
lib.mtla_workspace_bytes.argtypes = [_DIMS_P, _I32, _I32]
lib.mtla_status_string.restype = _c.c_char_p
lib.mtla_status_string.argtypes = [_c.c_int]
lib.mtla_debug_stride_mask.restype = _c.c_int
lib.mtla_debug_stride_mask.argtypes = [_I32, _I32, _P]
lib.mtla_cache_length.restype = _I64
lib.mtla_cache_length.argtypes = [_I64, _I32]
lib.mtla_decode_attn_multi.restype = _c.c_int
lib.mtla_decode_attn_multi.argtypes = [_DIMS_P, _I32, _I32, _P, _P, _MERGE_P, _P, _I64, _I64, _P, _P, _P, _P, _P,
                                       _P, _P, _SZ, _P, _P]
lib.mtla_decode_multi_workspace_bytes.restype = _SZ
lib.mtla_decode_multi_workspace_bytes.argtypes = [_DIMS_P, _I32, _I32]
lib.mtla_prefill_kv.restype = _c.c_int
lib.mtla_prefill_kv.argtypes = [_DIMS_P, _I32, _I32, _P, _P, _P, _P, _P, _P]
lib.mtla_prefill_unabsorbed_attn.restype = _c.c_int
lib.mtla_prefill_unabsorbed_attn.argtypes = [_DIMS_P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P]
lib.mtla_project_in.restype = _c.c_int
lib.mtla_project_in.argtypes = [_DIMS_P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _P]
lib.mtla_project_out.restype = _c.c_int
lib.mtla_project_out.argtypes = [_DIMS_P, _I32, _I32, _P, _P, _P, _P, _SZ, _P, _P]
lib.mtla_project_workspace_bytes.restype = _SZ
lib.mtla_project_workspace_bytes.argtypes = [_DIMS_P, _I32, _I32, _I32]
lib.mtla_train_attn_fwd.restype = _c.c_int
lib.mtla_train_attn_fwd.argtypes = [_DIMS_P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _P]
lib.mtla_train_workspace_bytes.restype = _SZ
lib.mtla_train_workspace_bytes.argtypes = [_DIMS_P, _I32, _I32, _I32]
lib.mtla_train_attn_bwd.restype = _c.c_int
lib.mtla_train_attn_bwd.argtypes = [_DIMS_P, _I32, _I32] + [_P] * 14 + [_SZ, _P, _P]
lib.mtla_train_kv_bwd.restype = _c.c_int
lib.mtla_train_kv_bwd.argtypes = [_DIMS_P, _I32, _I32, _P, _P, _P, _P, _P, _SZ, _P, _P]
lib.mtla_train_merge_bwd.restype = _c.c_int
lib.mtla_train_merge_bwd.argtypes = [_DIMS_P, _I32, _I32, _P, _P, _P, _P, _I32, _P, _P, _P, _P, _P, _P, _SZ, _P,
                                     _P]


class MtlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {mtla_status_string(status)} (status {status})")


def mtla_status_string(status: int) -> str:
    return lib.mtla_status_string(int(status)).decode()


def dims(H: int, d_h: int, r: int, d_R: int, s: int, dtype) -> _Dims:
    if isinstance(dtype, str):
        dtype = {"f32": MTLA_F32, "bf16": MTLA_BF16}[dtype]
    return _Dims(H, d_h, r, d_R, s, int(dtype))


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


_MERGE_CACHE: dict = {}


def _merge(m):
    """The merge-argument struct for `m`; the structs of the last few distinct
    argument sets are kept, so a decode loop does not rebuild one per call."""
    if m is None:
        return None
    key = (_ptr(m["c_new"]), _ptr(m["kR_new"]), _ptr(m["W_c"]), _ptr(m["b_c"]), _ptr(m["P"]), int(m["J_max"]))
    st = _MERGE_CACHE.get(key)
    if st is None:
        if len(_MERGE_CACHE) >= 64:
            _MERGE_CACHE.clear()
        st = _MERGE_CACHE[key] = _Merge(*key)
    return _c.byref(st)


def _check(status: int, where: str):
    if status != 0:
        raise MtlaError(status, where)


def mtla_merge_append(d, B, merge, cache, cache_rows, row_stride, seq_offset, seq_capacity, t_processed,
                      cache_len, dev_err, stream=None):
    _check(lib.mtla_merge_append(_c.byref(d), B, _merge(merge), _ptr(cache), cache_rows, row_stride,
                                 _ptr(seq_offset), _ptr(seq_capacity), _ptr(t_processed), _ptr(cache_len),
                                 _ptr(dev_err), _stream(stream)), "mtla_merge_append")


def mtla_decode_attn(d, B, q_abs, q_rope, merge, cache, cache_rows, row_stride, seq_offset, seq_capacity,
                     t_processed, cache_len, out, lse, workspace, workspace_bytes, dev_err, stream=None):
    _check(lib.mtla_decode_attn(_c.byref(d), B, _ptr(q_abs), _ptr(q_rope), _merge(merge), _ptr(cache), cache_rows,
                                row_stride, _ptr(seq_offset), _ptr(seq_capacity), _ptr(t_processed),
                                _ptr(cache_len), _ptr(out), _ptr(lse), _ptr(workspace), workspace_bytes,
                                _ptr(dev_err), _stream(stream)), "mtla_decode_attn")


def mtla_decode_attn_static(d, B, q_abs, q_rope, merge, cache, cache_rows, row_stride, seq_offset, seq_capacity,
                            t_processed, cache_len, out, lse, dev_err, stream=None):
    _check(lib.mtla_decode_attn_static(_c.byref(d), B, _ptr(q_abs), _ptr(q_rope), _merge(merge), _ptr(cache),
                                       cache_rows, row_stride, _ptr(seq_offset), _ptr(seq_capacity),
                                       _ptr(t_processed), _ptr(cache_len), _ptr(out), _ptr(lse), _ptr(dev_err),
                                       _stream(stream)), "mtla_decode_attn_static")


def mtla_prefill_masked_attn(d, B, T, q_abs, q_rope, c, kR, W_c, b_c, P, J_max, c_partial, cache_out, out,
                             dev_err, stream=None):
    _check(lib.mtla_prefill_masked_attn(_c.byref(d), B, T, _ptr(q_abs), _ptr(q_rope), _ptr(c), _ptr(kR),
                                        _ptr(W_c), _ptr(b_c), _ptr(P), J_max, _ptr(c_partial), _ptr(cache_out),
                                        _ptr(out), _ptr(dev_err), _stream(stream)), "mtla_prefill_masked_attn")


def mtla_decode_attn_multi(d, B, n, q_abs, q_rope, merge, cache, cache_rows, row_stride, seq_offset, seq_capacity,
                           t_processed, cache_len, out, lse, workspace, workspace_bytes, dev_err, stream=None):
    _check(lib.mtla_decode_attn_multi(_c.byref(d), B, n, _ptr(q_abs), _ptr(q_rope), _merge(merge), _ptr(cache),
                                      cache_rows, row_stride, _ptr(seq_offset), _ptr(seq_capacity),
                                      _ptr(t_processed), _ptr(cache_len), _ptr(out), _ptr(lse), _ptr(workspace),
                                      workspace_bytes, _ptr(dev_err), _stream(stream)), "mtla_decode_attn_multi")


def mtla_decode_multi_workspace_bytes(d, B, n) -> int:
    return int(lib.mtla_decode_multi_workspace_bytes(_c.byref(d), B, n))


def mtla_prefill_kv(d, B, T, c_partial, W_kv, k, v, dev_err, stream=None):
    _check(lib.mtla_prefill_kv(_c.byref(d), B, T, _ptr(c_partial), _ptr(W_kv), _ptr(k), _ptr(v), _ptr(dev_err),
                               _stream(stream)), "mtla_prefill_kv")


def mtla_prefill_unabsorbed_attn(d, B, T, q, q_rope, k, v, c_partial, out, dev_err, stream=None):
    _check(lib.mtla_prefill_unabsorbed_attn(_c.byref(d), B, T, _ptr(q), _ptr(q_rope), _ptr(k), _ptr(v),
                                            _ptr(c_partial), _ptr(out), _ptr(dev_err), _stream(stream)),
           "mtla_prefill_unabsorbed_attn")


def mtla_train_attn_fwd(d, B, T, q, q_rope, k, v, kR, out, lse, dev_err, stream=None):
    _check(lib.mtla_train_attn_fwd(_c.byref(d), B, T, _ptr(q), _ptr(q_rope), _ptr(k), _ptr(v), _ptr(kR), _ptr(out),
                                   _ptr(lse), _ptr(dev_err), _stream(stream)), "mtla_train_attn_fwd")


def mtla_train_workspace_bytes(d, B, T, which) -> int:
    return int(lib.mtla_train_workspace_bytes(_c.byref(d), B, T, which))


def mtla_train_attn_bwd(d, B, T, q, q_rope, k, v, kR, out, lse, d_out, dq, dq_rope, dk, dv, dkR, workspace,
                        workspace_bytes, dev_err, stream=None):
    _check(lib.mtla_train_attn_bwd(_c.byref(d), B, T, _ptr(q), _ptr(q_rope), _ptr(k), _ptr(v), _ptr(kR), _ptr(out),
                                   _ptr(lse), _ptr(d_out), _ptr(dq), _ptr(dq_rope), _ptr(dk), _ptr(dv), _ptr(dkR),
                                   _ptr(workspace), workspace_bytes, _ptr(dev_err), _stream(stream)),
           "mtla_train_attn_bwd")


def mtla_train_kv_bwd(d, B, T, dk, dv, W_kv, dC, workspace, workspace_bytes, dev_err, stream=None):
    _check(lib.mtla_train_kv_bwd(_c.byref(d), B, T, _ptr(dk), _ptr(dv), _ptr(W_kv), _ptr(dC), _ptr(workspace),
                                 workspace_bytes, _ptr(dev_err), _stream(stream)), "mtla_train_kv_bwd")


def mtla_train_merge_bwd(d, B, T, c, W_c, b_c, P, J_max, dC, dc, dW_c, db_c, dP, workspace, workspace_bytes, dev_err,
                         stream=None):
    _check(lib.mtla_train_merge_bwd(_c.byref(d), B, T, _ptr(c), _ptr(W_c), _ptr(b_c), _ptr(P), J_max, _ptr(dC),
                                    _ptr(dc), _ptr(dW_c), _ptr(db_c), _ptr(dP), _ptr(workspace), workspace_bytes,
                                    _ptr(dev_err), _stream(stream)), "mtla_train_merge_bwd")


def mtla_project_in(d, B, dm, x, W_in, pos, q_abs, q_rope, c_new, kR_new, workspace, workspace_bytes, dev_err,
                    stream=None):
    _check(lib.mtla_project_in(_c.byref(d), B, dm, _ptr(x), _ptr(W_in), _ptr(pos), _ptr(q_abs), _ptr(q_rope),
                               _ptr(c_new), _ptr(kR_new), _ptr(workspace), workspace_bytes, _ptr(dev_err),
                               _stream(stream)), "mtla_project_in")


def mtla_project_out(d, B, dm, o, W_out, y, workspace, workspace_bytes, dev_err, stream=None):
    _check(lib.mtla_project_out(_c.byref(d), B, dm, _ptr(o), _ptr(W_out), _ptr(y), _ptr(workspace),
                                workspace_bytes, _ptr(dev_err), _stream(stream)), "mtla_project_out")


def mtla_project_workspace_bytes(d, B, dm, which) -> int:
    return int(lib.mtla_project_workspace_bytes(_c.byref(d), B, dm, which))


def mtla_workspace_bytes(d, B, which=WS_DECODE) -> int:
    return int(lib.mtla_workspace_bytes(_c.byref(d), B, which))


def mtla_debug_stride_mask(s: int, T: int):
    import numpy as np
    out = np.zeros((T, T), dtype=np.uint8)
    _check(lib.mtla_debug_stride_mask(s, T, out.ctypes.data if T else None), "mtla_debug_stride_mask")
    return out


def mtla_cache_length(t: int, s: int) -> int:
    return int(lib.mtla_cache_length(t, s))


def exported_symbols():
    """Function names declared in include/mtla.h (the ABI's entry points)."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(mtla_\w+)\s*\(", text, flags=re.M)))
