"""Decode step (merge/append + absorbed attention) through the C ABI vs the oracle."""
import math

import numpy as np
import pytest
import torch

import mtla_synth as synth
import oracle
from gpu_harness import (DecodeRun, assert_close, expected_lengths, host, oracle_decode, rel_err)

pytestmark = pytest.mark.gpu


def _check_step(run: DecodeRun, merge=True, what=""):
    case = run.case
    d = case.dims
    out, lse = run.step(case.q_abs, case.q_rope, case.c_new if merge else None, case.kR_new if merge else None)
    o_ref, l_ref, rows_ref = oracle_decode(case, run.J_max, merge=merge)
    B = case.B
    assert_close(out, np.stack([o_ref[b] for b in range(B)]), case.dtype, f"{what} out")
    # lse is compared as an absolute error relative to its own scale
    assert_close(lse, np.stack([l_ref[b] for b in range(B)]), case.dtype, f"{what} lse")
    # integer state: bit-exact
    L = expected_lengths(case.t_prev, d.s, merge)
    assert run.cache_len.cpu().tolist() == L
    assert run.t.cpu().tolist() == [int(t) + (1 if merge else 0) for t in case.t_prev]
    assert int(run.err.item()) == 0
    # the cache: rows before the tail untouched (bit-exact), tail row as the oracle
    for b in range(B):
        got = run.cache.rows(b, L[b])
        n_keep = len(case.rows[b]) - (0 if (not merge or oracle.opens_new_row(int(case.t_prev[b]) + 1, d.s)) else 1)
        np.testing.assert_array_equal(got[:n_keep], case.rows[b][:n_keep].astype(np.float64))
        if merge:
            assert_close(got[-1], rows_ref[b][-1], case.dtype, f"{what} tail row b={b}")
    return out


def test_decode_uniform_b32():
    """B=32, 4096/4095 processed tokens (append in even, in-place in odd sequences), s=2."""
    _check_step(DecodeRun(synth.decode_uniform()), what="uniform")


def test_decode_ragged_b128():
    """B=128, processed lengths uniform in [512, 8192], paged contiguous cache."""
    _check_step(DecodeRun(synth.decode_ragged(), gap=3), what="ragged")


@pytest.mark.parametrize("s", [1, 2, 3, 4, 8, 16, 64])
@pytest.mark.parametrize("merge", [True, False])
def test_decode_small_ragged(s, merge):
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=s)
    rng = np.random.default_rng(100 + s)
    t_prev = np.concatenate([[1, 2, s, s + 1, 63 * s, 64 * s, 64 * s + 1, 129 * s - 1],
                             rng.integers(1, 700, size=9)])
    if not merge:
        t_prev = np.maximum(t_prev, 1)
    case = synth.decode_case(dims, t_prev, seed=200 + s, dtype="bf16")
    _check_step(DecodeRun(case, gap=1, extra_capacity=3), merge=merge, what=f"s={s}")


def test_decode_padded_row_stride():
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=2)
    case = synth.decode_case(dims, [5, 130, 1000, 3], seed=7, dtype="bf16")
    _check_step(DecodeRun(case, row_stride=304, gap=2), what="stride 304")


def test_decode_single_sequence_long():
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=2)
    case = synth.decode_case(dims, [40001], seed=8, dtype="bf16")
    _check_step(DecodeRun(case), what="B=1 long")


def test_decode_many_short_sequences():
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=3)
    rng = np.random.default_rng(9)
    case = synth.decode_case(dims, rng.integers(1, 12, size=700), seed=9, dtype="bf16")
    _check_step(DecodeRun(case, extra_capacity=1), what="B=700 short")


@pytest.mark.parametrize("B", [1024, 1025])
def test_decode_batch_limit(B):
    """The largest batch the tensor-core decode takes (1024 sequences) and one
    more (the generic kernel): short ragged sequences, merge at every step."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=2)
    rng = np.random.default_rng(15 + B)
    case = synth.decode_case(dims, rng.integers(1, 40, size=B), seed=16 + B, dtype="bf16")
    _check_step(DecodeRun(case, extra_capacity=1), what=f"B={B}")


def test_decode_consecutive_steps():
    """Five decode steps in a row, state kept on the device, vs the oracle stepping."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=3)
    case = synth.decode_case(dims, [1, 2, 3, 200, 301, 77], seed=10, dtype="bf16")
    run = DecodeRun(case)
    rng = np.random.default_rng(11)
    rows = [list(r.astype(np.float64)) for r in case.rows]
    t_prev = case.t_prev.copy()
    for step in range(5):
        qa = synth.cast(rng.standard_normal((case.B, 8, 256)), "bf16")
        qr = synth.cast(rng.standard_normal((case.B, 8, 32)), "bf16")
        cn = synth.cast(rng.standard_normal((case.B, 256)), "bf16")
        kn = synth.cast(rng.standard_normal((case.B, 32)), "bf16")
        out, _ = run.step(qa, qr, cn, kn)
        o_ref, _, r_ref = oracle_decode(case, run.J_max, q_abs=qa, q_rope=qr, c_new=cn, kR_new=kn, rows=rows,
                                        t_prev=t_prev)
        assert_close(out, np.stack([o_ref[b] for b in range(case.B)]), "bf16", f"step {step}")
        rows = [list(r_ref[b]) for b in range(case.B)]
        t_prev = t_prev + 1
        assert run.t.cpu().tolist() == t_prev.tolist()
        assert run.cache_len.cpu().tolist() == [math.ceil(t / 3) for t in t_prev]


def test_decode_tiny_fp32():
    """fp32 path (one block per sequence), tiny dims, 1e-5 tolerance."""
    case = synth.decode_case(synth.TINY, [1, 2, 3, 40, 41, 64], seed=12, dtype="f32")
    _check_step(DecodeRun(case, gap=1), what="tiny fp32")
    _check_step(DecodeRun(case, gap=1), merge=False, what="tiny fp32 no merge")


def test_decode_workspace_reused_many_calls():
    """One workspace serves 20 calls in a row: results stay bit-identical."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=2)
    case = synth.decode_case(dims, [3000, 17, 5000, 2500], seed=13, dtype="bf16")
    run = DecodeRun(case)
    first, _ = run.step(case.q_abs, case.q_rope)
    for _ in range(19):
        again, _ = run.step(case.q_abs, case.q_rope)
        np.testing.assert_array_equal(again, first)



def test_decode_workspace_needs_no_zeroing():
    """A workspace full of NaN bytes: short sequences leave some blocks of the
    split-L grid with empty shares inside a split sequence's block range."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=2)
    # fewer cost positions (rows, plus the merge weight of a merged sequence)
    # than the grid's blocks: one merged sequence, then three without merge
    for t_prev, merge in (([180], True), ([180, 3, 61], False)):
        case = synth.decode_case(dims, t_prev, seed=17, dtype="bf16")
        run = DecodeRun(case)
        run.ws.fill_(0xFF)
        _check_step(run, merge=merge, what=f"NaN workspace {t_prev}")


def test_decode_device_errors():
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=2)
    case = synth.decode_case(dims, [8, 9, 0], seed=14, dtype="bf16")
    # sequence 1 needs a 6th row but owns 5; sequence 2 is empty without a merge
    run = DecodeRun(case, extra_capacity=0)
    run.step(case.q_abs, case.q_rope, case.c_new, case.kR_new)
    err = int(run.err.item())
    assert err & 2, "capacity overflow must be reported"
    run2 = DecodeRun(case)
    run2.step(case.q_abs, case.q_rope)
    assert int(run2.err.item()) & 4, "attention over an empty cache must be reported"
    assert np.isfinite(host(run2.out)).all()
    # P table too short for the new token's group
    run3 = DecodeRun(case, J_extra=0)
    run3.J_max = 4
    run3.step(case.q_abs, case.q_rope, case.c_new, case.kR_new)
    assert int(run3.err.item()) & 1


def test_decode_host_errors():
    import temporally_compressed_latent_b200 as mtla
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=2)
    case = synth.decode_case(dims, [8, 9], seed=15, dtype="bf16")
    run = DecodeRun(case)
    with pytest.raises(mtla.MtlaError) as ei:
        mtla.mtla_decode_attn(run.md, 2, run.cache.buf, run.cache.buf, None, run.cache.buf, run.cache.cache_rows,
                              288, run.cache.offset, run.cache.capacity, run.t, run.cache_len, run.out, run.lse,
                              run.ws, 16, run.err)
    assert ei.value.status == 3
