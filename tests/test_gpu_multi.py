"""Several new tokens per sequence in one decode call (mtla_decode_attn_multi)
through the C ABI: against the oracle stepping the same tokens one at a time
(MTLA paper notes, "Key designs: hyper-network temporal merging"; abstract
page, Figure 2(a)), and bit for bit against as many single-token calls on
the device for the cache it leaves."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import mtla_synth as synth
import oracle
import temporally_compressed_latent_b200 as mtla
from gpu_harness import DeviceCache, DecodeRun, assert_close, dev, host, oracle_P

pytestmark = pytest.mark.gpu


def _tokens(case, n, seed):
    """n new tokens per sequence: queries, latents and RoPE keys ~ N(0,1)."""
    d = case.dims
    rng = np.random.default_rng(seed)
    cast = lambda a: synth.cast(a, case.dtype)
    return (cast(rng.standard_normal((case.B, n, d.H, d.r))), cast(rng.standard_normal((case.B, n, d.H, d.d_R))),
            cast(rng.standard_normal((case.B, n, d.r))), cast(rng.standard_normal((case.B, n, d.d_R))))


def _multi_call(run: DecodeRun, n, qa, qr, cn, kn):
    d, B = run.dims, run.B
    run._mq = [dev(a, run.dtype) for a in (qa, qr, cn, kn)]
    ws_bytes = mtla.mtla_decode_multi_workspace_bytes(run.md, B, n)
    run._mws = torch.full((ws_bytes,), 0xFF, dtype=torch.uint8, device="cuda")  # needs no initialisation
    out = torch.full((B, n, d.H, d.r), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((B, n, d.H), float("nan"), dtype=torch.float32, device="cuda")
    merge = {"c_new": run._mq[2], "kR_new": run._mq[3], "W_c": run.W_c, "b_c": run.b_c, "P": run.P,
             "J_max": run.J_max}
    mtla.mtla_decode_attn_multi(run.md, B, n, run._mq[0], run._mq[1], merge, run.cache.buf, run.cache.cache_rows,
                                run.cache.row_stride, run.cache.offset, run.cache.capacity, run.t, run.cache_len,
                                out, lse, run._mws, ws_bytes, run.err)
    torch.cuda.synchronize()
    return host(out), host(lse)


def _oracle_multi(case, J, n, qa, qr, cn, kn, seqs=None):
    d = case.dims
    P = oracle_P(case.lin, J)
    seqs = range(case.B) if seqs is None else seqs
    o_ref, l_ref, rows_ref = {}, {}, {}
    for b in seqs:
        rows = list(np.asarray(case.rows[b], np.float64))
        t = int(case.t_prev[b])
        outs, lses = [], []
        for i in range(n):
            rows, o, lse = oracle.decode_step(rows, t, d.s, cn[b, i], kn[b, i], qa[b, i], qr[b, i],
                                              case.lin["W_c"], case.lin["b_c"], P, d.d_h)
            t += 1
            outs.append(o)
            lses.append(lse)
        o_ref[b], l_ref[b], rows_ref[b] = np.stack(outs), np.stack(lses), np.stack(rows)
    return o_ref, l_ref, rows_ref


@pytest.mark.parametrize("s,n", [(1, 3), (2, 1), (2, 4), (3, 7), (8, 16), (2, 16)])
def test_multi_vs_oracle(s, n):
    """Ragged lengths (0 included), n tokens crossing group boundaries."""
    dims = dataclasses.replace(synth.MAIN, s=s)
    rng = np.random.default_rng(1600 + 10 * s + n)
    t_prev = np.concatenate([[0, 1, s - 1, s, 2 * s + 1], rng.integers(0, 900, size=11)])
    case = synth.decode_case(dims, t_prev, seed=1610 + s + n, dtype="bf16")
    run = DecodeRun(case, extra_capacity=n // s + 2, gap=2)
    toks = _tokens(case, n, 1620 + s + n)
    out, lse = _multi_call(run, n, *toks)
    assert int(run.err.item()) == 0
    o_ref, l_ref, rows_ref = _oracle_multi(case, run.J_max, n, *toks)
    B = case.B
    assert_close(out, np.stack([o_ref[b] for b in range(B)]), "bf16", f"out s={s} n={n}")
    assert_close(lse, np.stack([l_ref[b] for b in range(B)]), "bf16", f"lse s={s} n={n}")
    assert run.t.cpu().tolist() == [int(t) + n for t in t_prev]
    assert run.cache_len.cpu().tolist() == [math.ceil((int(t) + n) / s) for t in t_prev]
    for b in range(B):
        L = len(rows_ref[b])
        assert_close(run.cache.rows(b, L), rows_ref[b], "bf16", f"rows b={b}")


def test_multi_b32_4096_tokens_n4():
    """The B=32 decode shapes (4096 / 4095 processed tokens, s = 2) with four
    new tokens per sequence."""
    case = synth.decode_uniform()
    n = 4
    run = DecodeRun(case, extra_capacity=4)
    toks = _tokens(case, n, 1700)
    out, _ = _multi_call(run, n, *toks)
    assert int(run.err.item()) == 0
    o_ref, _, rows_ref = _oracle_multi(case, run.J_max, n, *toks)
    assert_close(out, np.stack([o_ref[b] for b in range(case.B)]), "bf16", "out")
    for b in (0, 1, 30, 31):
        L = len(rows_ref[b])
        assert_close(run.cache.rows(b, L)[-3:], rows_ref[b][-3:], "bf16", f"tail rows b={b}")


def test_multi_equals_single_steps_bit_exact():
    """The cache, lengths and processed counts a multi-token call leaves are
    bit for bit those of n single-token calls on the same state (the tokens
    are merged in the same order and rounded after each one); the outputs
    agree within the tolerance (the row shares differ)."""
    dims = dataclasses.replace(synth.MAIN, s=3)
    rng = np.random.default_rng(1800)
    t_prev = rng.integers(0, 3000, size=40)
    case = synth.decode_case(dims, t_prev, seed=1801, dtype="bf16")
    n = 5
    toks = _tokens(case, n, 1802)
    multi = DecodeRun(case, extra_capacity=3)
    single = DecodeRun(case, extra_capacity=3)
    out_m, _ = _multi_call(multi, n, *toks)
    outs = []
    for i in range(n):
        o, _ = single.step(toks[0][:, i], toks[1][:, i], toks[2][:, i], toks[3][:, i])
        outs.append(o)
    assert torch.equal(multi.cache.buf.view(torch.int16), single.cache.buf.view(torch.int16))
    assert torch.equal(multi.t, single.t) and torch.equal(multi.cache_len, single.cache_len)
    assert_close(out_m, np.stack(outs, axis=1), "bf16", "multi vs single-token calls")


def test_multi_tiny_fp32():
    case = synth.decode_case(dataclasses.replace(synth.TINY, s=3), [0, 1, 2, 40, 41, 64], seed=1900, dtype="f32")
    n = 5
    run = DecodeRun(case, extra_capacity=3, gap=1)
    toks = _tokens(case, n, 1901)
    out, lse = _multi_call(run, n, *toks)
    assert int(run.err.item()) == 0
    o_ref, l_ref, _ = _oracle_multi(case, run.J_max, n, *toks)
    assert_close(out, np.stack([o_ref[b] for b in range(case.B)]), "f32", "out fp32")
    assert_close(lse, np.stack([l_ref[b] for b in range(case.B)]), "f32", "lse fp32")


def test_multi_generic_path_beyond_1024_queries():
    """B n = 1200 per-query sequences: the one-block-per-query kernel."""
    dims = synth.MAIN
    rng = np.random.default_rng(2000)
    case = synth.decode_case(dims, rng.integers(0, 60, size=300), seed=2001, dtype="bf16")
    n = 4
    run = DecodeRun(case, extra_capacity=3)
    toks = _tokens(case, n, 2002)
    out, _ = _multi_call(run, n, *toks)
    assert int(run.err.item()) == 0
    seqs = [0, 1, 150, 299]
    o_ref, _, _ = _oracle_multi(case, run.J_max, n, *toks, seqs=seqs)
    assert_close(out[seqs], np.stack([o_ref[b] for b in seqs]), "bf16", "out")
    assert run.t.cpu().tolist() == [int(t) + n for t in case.t_prev]


def test_multi_device_errors():
    """A sequence whose tokens overflow its capacity merges none of them and
    its queries attend its cache as it stands; the others merge."""
    dims = synth.MAIN
    case = synth.decode_case(dims, [8, 7, 20], seed=2100, dtype="bf16")
    n = 3
    run = DecodeRun(case, extra_capacity=1)  # b=0: 4 rows + 1 spare, tokens 9..11 need 6 rows
    toks = _tokens(case, n, 2101)
    out, _ = _multi_call(run, n, *toks)
    assert int(run.err.item()) & mtla.DEVERR_CAPACITY
    assert run.t.cpu().tolist() == [8, 10, 20]
    o_att = [oracle.decode_attention(toks[0][0, i], toks[1][0, i], case.rows[0], dims.d_h)[0] for i in range(n)]
    assert_close(out[0], np.stack(o_att), "bf16", "unmerged sequence attends its cache")
    o_ref, _, _ = _oracle_multi(case, run.J_max, n, *toks, seqs=[1])
    assert_close(out[1], o_ref[1], "bf16", "b=1")
