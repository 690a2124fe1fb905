"""The C ABI library without a GPU: it loads, exports every entry point that
include/mtla.h declares, and its host-side logic (status codes, argument
checks, the mask and cache-length rules) behaves as documented."""
import ctypes

import numpy as np
import pytest

import oracle
import temporally_compressed_latent_b200 as mtla


def test_library_exports_every_declared_symbol():
    names = mtla.exported_symbols()
    assert {"mtla_merge_append", "mtla_decode_attn", "mtla_prefill_masked_attn", "mtla_workspace_bytes",
            "mtla_status_string", "mtla_debug_stride_mask", "mtla_cache_length"} <= set(names)
    for n in names:
        assert hasattr(mtla.lib, n), n


def test_status_strings():
    for code in range(5):
        assert mtla.mtla_status_string(code)
    assert mtla.mtla_status_string(99) == "unknown status"


@pytest.mark.parametrize("s", [1, 2, 3, 4, 8, 13])
def test_mask_and_lengths_bit_exact(s):
    for T in (0, 1, 5, 33):
        got = mtla.mtla_debug_stride_mask(s, T)
        if T:
            np.testing.assert_array_equal(got.astype(bool), oracle.stride_mask(T, s))
    for t in range(0, 200):
        assert mtla.mtla_cache_length(t, s) == oracle.cache_length(t, s)


def _fake(n=1 << 12):
    # host memory stands in for device pointers: only argument checks run
    buf = (ctypes.c_uint8 * (n + 64))()
    base = (ctypes.addressof(buf) + 63) & ~63
    return buf, base


def test_host_argument_errors_need_no_gpu():
    keep, p = _fake()
    d = mtla.dims(8, 64, 256, 32, 2, "bf16")
    bad_dims = mtla.dims(8, 64, 256, 32, 0, "bf16")
    huge = mtla.dims(32, 64, 256, 32, 2, "bf16")
    L = mtla.lib
    # s < 1
    assert L.mtla_decode_attn(ctypes.byref(bad_dims), 1, p, p, None, p, 10, 288, p, p, p, p, p, p, p, 1 << 20,
                              p, None) == 1
    # H beyond the supported range
    assert L.mtla_decode_attn(ctypes.byref(huge), 1, p, p, None, p, 10, 288, p, p, p, p, p, p, p, 1 << 20,
                              p, None) == 2
    # null cache
    assert L.mtla_decode_attn(ctypes.byref(d), 1, p, p, None, None, 10, 288, p, p, p, p, p, p, p, 1 << 20,
                              p, None) == 1
    # misaligned query
    assert L.mtla_decode_attn(ctypes.byref(d), 1, p + 2, p, None, p, 10, 288, p, p, p, p, p, p, p, 1 << 20,
                              p, None) == 1
    # row stride below D, and not a multiple of 16 bytes
    assert L.mtla_decode_attn(ctypes.byref(d), 1, p, p, None, p, 10, 280, p, p, p, p, p, p, p, 1 << 20,
                              p, None) == 1
    assert L.mtla_decode_attn(ctypes.byref(d), 1, p, p, None, p, 10, 292, p, p, p, p, p, p, p, 1 << 20,
                              p, None) == 1
    # B == 0 is a valid no-op and launches nothing
    assert L.mtla_decode_attn(ctypes.byref(d), 0, p, p, None, p, 10, 288, p, p, p, p, p, p, p, 0, p, None) == 0
    # prefill: P table shorter than ceil(T/s)
    assert L.mtla_prefill_masked_attn(ctypes.byref(d), 1, 10, p, p, p, p, p, p, p, 4, p, None, p, p, None) == 1
    assert L.mtla_prefill_masked_attn(ctypes.byref(d), 0, 10, p, p, p, p, p, p, p, 4, p, None, p, p, None) == 0
    # prefill: C_hat' or the cache rows off a 16-byte boundary (the running
    # merge's TMA maps and stores need it) are refused before any launch
    assert L.mtla_prefill_masked_attn(ctypes.byref(d), 1, 10, None, None, p, p, p, p, p, 8, p + 2, p, None, p,
                                      None) == 1
    assert L.mtla_prefill_masked_attn(ctypes.byref(d), 1, 10, None, None, p, p, p, p, p, 8, p, p + 2, None, p,
                                      None) == 1
    # merge arguments: J_max must be positive
    m = mtla._abi._Merge(p, p, p, p, p, 0)
    assert L.mtla_merge_append(ctypes.byref(d), 1, ctypes.byref(m), p, 10, 288, p, p, p, p, p, None) == 1


def test_binding_raises_on_error_status():
    keep, p = _fake()
    d = mtla.dims(8, 64, 256, 32, 0, "bf16")
    with pytest.raises(mtla.MtlaError) as ei:
        mtla.mtla_merge_append(d, 1, {"c_new": p, "kR_new": p, "W_c": p, "b_c": p, "P": p, "J_max": 3},
                               p, 10, 288, p, p, p, p, p, stream=0)
    assert ei.value.status == 1


def test_training_calls_check_arguments_on_the_host():
    keep, p = _fake()
    d = mtla.dims(8, 64, 256, 32, 2, "bf16")
    other = mtla.dims(8, 32, 256, 32, 2, "bf16")  # d_h = 32: no training kernels
    L = mtla.lib
    ws = mtla.mtla_train_workspace_bytes(d, 2, 100, mtla.TRAIN_ATTN_BWD)
    # two fp32 [B, H, T] arrays and the per-head RoPE key gradients
    assert ws >= 2 * 2 * 8 * 100 * 4 + 2 * 100 * 8 * 32 * 4
    assert mtla.mtla_train_workspace_bytes(d, 2, 100, mtla.TRAIN_KV_BWD) == 0  # W_kv is read as stored
    assert mtla.mtla_train_workspace_bytes(d, 2, 100, mtla.TRAIN_MERGE_BWD) > 2 * 100 * 256 * 4
    assert mtla.mtla_train_workspace_bytes(other, 2, 100, mtla.TRAIN_ATTN_BWD) == 0
    assert mtla.mtla_train_workspace_bytes(d, 2, 100, 9) == 0
    bwd = lambda dims, B, T, wsb: L.mtla_train_attn_bwd(ctypes.byref(dims), B, T, *([p] * 13), p, wsb, p, None)
    assert bwd(other, 2, 100, ws) == 2                      # unsupported dims
    assert bwd(d, 2, 100, ws - 1) == 3                      # workspace too small
    assert bwd(d, 0, 100, 0) == 0                           # empty batch: nothing to do
    assert L.mtla_train_attn_bwd(ctypes.byref(d), 2, 100, *([p] * 12), None, p, ws, p, None) == 1  # null dkR
    # merge backward: the P table must cover ceil(T / s) groups
    wm = mtla.mtla_train_workspace_bytes(d, 2, 100, mtla.TRAIN_MERGE_BWD)
    assert L.mtla_train_merge_bwd(ctypes.byref(d), 2, 100, p, p, p, p, 49, p, p, p, p, p, p, wm, p, None) == 1
    assert L.mtla_train_merge_bwd(ctypes.byref(d), 2, 100, p, p, p, p, 50, p, p, p, p, p, p, wm - 1, p, None) == 3
    assert L.mtla_train_kv_bwd(ctypes.byref(other), 2, 100, p, p, p, p, None, 0, p, None) == 2
    assert L.mtla_train_attn_fwd(ctypes.byref(other), 2, 100, p, p, p, p, p, p, p, p, None) == 2
