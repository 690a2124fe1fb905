"""mtla_merge_append (the merge of one new token per sequence, alone) through
the C ABI vs the oracle's merge_weight / merge_step.

MTLA paper notes, "Key designs: hyper-network temporal merging": the new
token's gate w = sigmoid(Linear(c_t) * Linear(pe_j)) scales [c_t ; k^R_t],
which opens row j = ceil(t/s) when (t-1) mod s == 0 and is added in place to
the tail row otherwise (Figure 2(a) of the abstract page).  Lengths and the
rows the call must not touch are compared bit for bit."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import mtla_synth as synth
import oracle
import temporally_compressed_latent_b200 as mtla
from gpu_harness import DecodeRun, assert_close, dev, host, oracle_P

pytestmark = pytest.mark.gpu


def _merge_call(run: DecodeRun, c_new, kR_new, cache_len=True):
    run._c = dev(c_new, run.dtype)
    run._k = dev(kR_new, run.dtype)
    merge = {"c_new": run._c, "kR_new": run._k, "W_c": run.W_c, "b_c": run.b_c, "P": run.P, "J_max": run.J_max}
    mtla.mtla_merge_append(run.md, run.B, merge, run.cache.buf, run.cache.cache_rows, run.cache.row_stride,
                           run.cache.offset, run.cache.capacity, run.t, run.cache_len if cache_len else None,
                           run.err)
    torch.cuda.synchronize()


def _check_merge(case: synth.DecodeCase, run: DecodeRun, what: str):
    """One merge step on `run` (state = case) against the oracle, element by element."""
    d = case.dims
    before = host(run.cache.buf).copy()
    _merge_call(run, case.c_new, case.kR_new)
    assert int(run.err.item()) == 0, f"{what}: device error {int(run.err.item())}"
    P = oracle_P(case.lin, run.J_max)
    t_new = [int(t) + 1 for t in case.t_prev]
    assert run.t.cpu().tolist() == t_new
    assert run.cache_len.cpu().tolist() == [oracle.cache_length(t, d.s) for t in t_new]
    after = host(run.cache.buf)
    touched = np.zeros(after.shape[0], dtype=bool)
    for b in range(case.B):
        t = t_new[b]
        j = oracle.group_index(t, d.s)
        w = oracle.merge_weight(case.c_new[b], P[j - 1], case.lin["W_c"], case.lin["b_c"])
        rows_ref = oracle.merge_step(list(case.rows[b]), t, d.s, case.c_new[b], case.kR_new[b], w)
        tail = run.cache.offs[b] + j - 1
        touched[tail] = True
        assert_close(after[tail, :d.D], rows_ref[-1], case.dtype, f"{what} tail row b={b} t={t}")
        # the rows before the tail are the oracle's too, and unchanged bit for bit
        n_keep = j - 1
        np.testing.assert_array_equal(after[run.cache.offs[b]:run.cache.offs[b] + n_keep, :d.D],
                                      np.asarray(case.rows[b][:n_keep], dtype=np.float64))
    # nothing else in the buffer moved (NaN gaps compare equal as NaN)
    np.testing.assert_array_equal(after[~touched], before[~touched])
    # the row-stride padding of the tail rows is untouched as well
    if run.cache.row_stride > d.D:
        np.testing.assert_array_equal(after[touched, d.D:], before[touched, d.D:])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("s", [1, 2, 3, 8, 64])
def test_merge_append_both_branches(dtype, s):
    """t_prev spans an empty cache (t = 1), each side of a group boundary
    (append when (t-1) mod s == 0, in place otherwise) and ragged lengths, on
    a paged cache with gaps between sequences."""
    dims = dataclasses.replace(synth.MAIN if dtype == "bf16" else synth.TINY, s=s)
    rng = np.random.default_rng(800 + s)
    t_prev = np.concatenate([[0, 1, s - 1, s, s + 1, 2 * s, 5 * s + 2], rng.integers(0, 300, size=7)])
    t_prev = np.maximum(t_prev, 0)
    case = synth.decode_case(dims, t_prev, seed=810 + s, dtype=dtype)
    run = DecodeRun(case, gap=2, extra_capacity=2)
    _check_merge(case, run, f"{dtype} s={s}")


def test_merge_append_padded_stride_and_null_cache_len():
    """A row stride of 304 elements (16 spare per row) and cache_len = NULL:
    t_processed still advances, the padding is never written."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=2)
    case = synth.decode_case(dims, [0, 5, 6, 130, 999], seed=820, dtype="bf16")
    run = DecodeRun(case, row_stride=304, gap=1, extra_capacity=1)
    before_len = run.cache_len.clone()
    before = host(run.cache.buf).copy()
    _merge_call(run, case.c_new, case.kR_new, cache_len=False)
    assert int(run.err.item()) == 0
    assert run.t.cpu().tolist() == [int(t) + 1 for t in case.t_prev]
    assert torch.equal(run.cache_len, before_len)
    after = host(run.cache.buf)
    np.testing.assert_array_equal(after[:, 288:], before[:, 288:])


def test_merge_append_consecutive_steps():
    """Seven merges in a row (s = 3 crosses two group boundaries) against the
    oracle stepping the same tokens."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=3)
    case = synth.decode_case(dims, [0, 1, 2, 3, 40], seed=830, dtype="bf16")
    run = DecodeRun(case, extra_capacity=4)
    P = oracle_P(case.lin, run.J_max)
    rows = [list(np.asarray(r, np.float64)) for r in case.rows]
    t_prev = case.t_prev.copy()
    rng = np.random.default_rng(831)
    for step in range(7):
        cn = synth.cast(rng.standard_normal((case.B, 256)), "bf16")
        kn = synth.cast(rng.standard_normal((case.B, 32)), "bf16")
        _merge_call(run, cn, kn)
        t_prev = t_prev + 1
        for b in range(case.B):
            t = int(t_prev[b])
            w = oracle.merge_weight(cn[b], P[oracle.group_index(t, 3) - 1], case.lin["W_c"], case.lin["b_c"])
            rows[b] = oracle.merge_step(rows[b], t, 3, cn[b], kn[b], w)
            # the device cache holds bf16 rows: the oracle continues from them
            got = run.cache.rows(b, len(rows[b]))
            assert_close(got[-1], rows[b][-1], "bf16", f"step {step} b={b}")
            rows[b] = [r for r in got]
        assert run.t.cpu().tolist() == t_prev.tolist()
        assert run.cache_len.cpu().tolist() == [math.ceil(int(t) / 3) for t in t_prev]
    assert int(run.err.item()) == 0


def test_merge_append_device_errors():
    """A full sequence (CAPACITY) and a group beyond the P table (PE_RANGE)
    skip their merge and leave t_processed; the other sequences merge."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=2)
    # b=0: 8 tokens in 4 rows, capacity 4 -> token 9 needs row 5: CAPACITY
    # b=1: 7 tokens, token 8 fills row 4 in place: fine
    case = synth.decode_case(dims, [8, 7], seed=840, dtype="bf16")
    run = DecodeRun(case, extra_capacity=0)
    before = host(run.cache.buf).copy()
    _merge_call(run, case.c_new, case.kR_new)
    assert int(run.err.item()) & mtla.DEVERR_CAPACITY
    assert run.t.cpu().tolist() == [8, 8]
    np.testing.assert_array_equal(host(run.cache.buf)[:4], before[:4])
    # P table of 4 rows: token 9 of b=0 (group 5) is out of range, token 8 of b=1 (group 4) is not
    case2 = synth.decode_case(dims, [8, 7], seed=841, dtype="bf16")
    run2 = DecodeRun(case2, extra_capacity=2)
    run2.J_max = 4
    _merge_call(run2, case2.c_new, case2.kR_new)
    assert int(run2.err.item()) == mtla.DEVERR_PE_RANGE
    assert run2.t.cpu().tolist() == [8, 8]
