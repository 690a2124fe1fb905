"""Masked parallel forward (running merge + stride-aware attention) through the
C ABI vs the oracle, and parallel == per-step decode on the GPU."""
import math

import numpy as np
import pytest
import torch

import mtla_synth as synth
import oracle
import temporally_compressed_latent_b200 as mtla
from gpu_harness import DecodeRun, TDT, assert_close, dev, host, mdims
from temporally_compressed_latent_b200 import glue

pytestmark = pytest.mark.gpu


class PrefillRun:
    def __init__(self, dims, dtype, q_abs, q_rope, c, kR, lin, with_out=True):
        self.dims, self.dtype = dims, dtype
        B, T = c.shape[0], c.shape[1]
        self.B, self.T = B, T
        self.J = synth.ceil_div(T, dims.s) + 2
        self.P = glue.pe_table(self.J, torch.from_numpy(lin["W_p"]).cuda(), torch.from_numpy(lin["b_p"]).cuda())
        self.W_c = torch.from_numpy(lin["W_c"]).cuda()
        self.b_c = torch.from_numpy(lin["b_c"]).cuda()
        self.qa = q_abs if q_abs is None or torch.is_tensor(q_abs) else dev(q_abs, dtype)
        self.qr = q_rope if q_rope is None or torch.is_tensor(q_rope) else dev(q_rope, dtype)
        self.c = c if torch.is_tensor(c) else dev(c, dtype)
        self.kR = kR if torch.is_tensor(kR) else dev(kR, dtype)
        D = dims.D
        self.cp = torch.full((B, T, D), float("nan"), dtype=TDT[dtype], device="cuda")
        self.cache = torch.full((B, synth.ceil_div(T, dims.s), D), float("nan"), dtype=TDT[dtype], device="cuda")
        self.out = (torch.full((B, T, dims.H, dims.r), float("nan"), dtype=TDT[dtype], device="cuda")
                    if with_out else None)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run(self):
        mtla.mtla_prefill_masked_attn(mdims(self.dims, self.dtype), self.B, self.T, self.qa, self.qr, self.c,
                                      self.kR, self.W_c, self.b_c, self.P, self.J, self.cp, self.cache, self.out,
                                      self.err)
        torch.cuda.synchronize()
        assert int(self.err.item()) == 0
        return self


def _oracle_seq(case_lin, c, kR, qa, qr, dims, with_out=True):
    P = oracle.pe_table(synth.ceil_div(c.shape[0], dims.s) + 2, case_lin["W_p"], case_lin["b_p"])
    Cp = oracle.partial_merge_sequence(c, kR, case_lin["W_c"], case_lin["b_c"], P, dims.s)
    o = oracle.masked_forward(qa, qr, Cp, dims.s, dims.d_h)[0] if with_out else None
    return Cp, o


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("s,T", [(1, 33), (2, 1), (2, 64), (3, 130), (5, 47), (8, 80), (70, 100)])
def test_prefill_small(dtype, s, T):
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=s) if dtype == "bf16" else \
        synth.Dims(H=4, d_h=16, r=64, d_R=8, s=s)
    case = synth.token_case(dims, B=2, T=T, seed=300 + s + T, dtype=dtype)
    run = PrefillRun(dims, dtype, case.q_abs, case.q_rope, case.c, case.kR, case.lin).run()
    for b in range(2):
        Cp, o = _oracle_seq(case.lin, case.c[b], case.kR[b], case.q_abs[b], case.q_rope[b], dims)
        assert_close(host(run.cp[b]), Cp, dtype, "C_hat'")
        assert_close(host(run.cache[b]), oracle.compressed_cache(Cp, s), dtype, "cache_out")
        assert_close(host(run.out[b]), o, dtype, "out")


def test_tiny_end_to_end_fp32():
    """B=1, H=4, d_h=16, r=64, d_R=8, s=2: prompt of 64 tokens then 16 decode steps.

    x and every weight from seed 0; the GPU side projects with torch fp32, the
    oracle with its own float64 glue."""
    mc = synth.tiny_e2e(0)
    dims = mc.dims
    T0, T = 64, 80
    W = {k: torch.from_numpy(v).cuda() for k, v in mc.W.items()}
    qa, qr, c, kR = glue.project(torch.from_numpy(mc.x).cuda(), W)
    # oracle: its own projections, the masked forward over the prompt, the decode loop over all 80
    q_abs_o, q_rope_o, c_o, kR_o = oracle.project_inputs(mc.x[0], mc.W)
    P_o = oracle.pe_table(synth.ceil_div(T, 2) + 2, mc.lin["W_p"], mc.lin["b_p"])
    Cp_o = oracle.partial_merge_sequence(c_o[:T0], kR_o[:T0], mc.lin["W_c"], mc.lin["b_c"], P_o, 2)
    o_par, _ = oracle.masked_forward(q_abs_o[:T0], q_rope_o[:T0], Cp_o, 2, dims.d_h)
    loop = oracle.decode_loop(c_o, kR_o, q_abs_o, q_rope_o, mc.lin["W_c"], mc.lin["b_c"], P_o, 2, dims.d_h)
    np.testing.assert_allclose(o_par, loop["o"][:T0], rtol=1e-11, atol=1e-12)

    run = PrefillRun(dims, "f32", qa[:, :T0].contiguous(), qr[:, :T0].contiguous(), c[:, :T0].contiguous(),
                     kR[:, :T0].contiguous(), mc.lin)
    run.J = synth.ceil_div(T, 2) + 2
    run.P = glue.pe_table(run.J, torch.from_numpy(mc.lin["W_p"]).cuda(), torch.from_numpy(mc.lin["b_p"]).cuda())
    run.run()
    assert_close(host(run.out[0]), o_par, "f32", "prompt outputs")
    assert_close(host(run.cache[0]), oracle.compressed_cache(Cp_o, 2), "f32", "prompt cache")

    # decode t = 65..80 from the prompt's cache
    L0 = T0 // 2
    rows0 = host(run.cache[0])
    case = synth.DecodeCase(dims, "f32", np.array([T0]), [rows0.astype(np.float32)], None, None, None, None, mc.lin)
    drun = DecodeRun(case, extra_capacity=10)
    drun.J_max, drun.P = run.J, run.P
    outs = []
    for t in range(T0 + 1, T + 1):
        o, _ = drun.step(host(qa[:, t - 1]).astype(np.float32), host(qr[:, t - 1]).astype(np.float32),
                         host(c[:, t - 1]).astype(np.float32), host(kR[:, t - 1]).astype(np.float32))
        outs.append(o[0])
    assert_close(np.stack(outs), loop["o"][T0:], "f32", "decode steps 65..80")
    assert drun.cache_len.cpu().tolist() == [40]

    # GPU parallel forward over all 80 tokens == GPU prompt + per-step decode
    full = PrefillRun(dims, "f32", qa, qr, c, kR, mc.lin)
    full.J, full.P = run.J, run.P
    full.run()
    gpu_seq = np.concatenate([host(run.out[0]), np.stack(outs)])
    assert_close(host(full.out[0]), gpu_seq, "f32", "parallel vs incremental (GPU)")
    assert_close(host(full.out[0]), loop["o"], "f32", "parallel (GPU) vs oracle decode loop")


def test_prefill_b8_t4096_sampled():
    """B=8, T=4096, d=512, s=2, bf16: x and weights from seed 5 through the
    layer glue; the running merge and the cache of every sequence in full,
    and sampled queries of three sequences (the last included), vs the
    oracle."""
    mc = synth.prefill_model()
    dims = mc.dims
    W = {k: torch.from_numpy(v).cuda() for k, v in mc.W.items()}
    x = torch.from_numpy(mc.x).cuda()
    qa, qr, c, kR = (t.to(torch.bfloat16).contiguous() for t in glue.project(x, W))
    run = PrefillRun(dims, "bf16", qa, qr, c, kR, mc.lin).run()
    rng = np.random.default_rng(55)
    P_o = oracle.pe_table(run.J, mc.lin["W_p"], mc.lin["b_p"])
    for b in range(mc.x.shape[0]):
        qa_o, qr_o, c_o, kR_o = oracle.project_inputs(mc.x[b], mc.W)
        Cp = oracle.partial_merge_sequence(c_o, kR_o, mc.lin["W_c"], mc.lin["b_c"], P_o, 2)
        # the running merge and the cache in full, every sequence
        assert_close(host(run.cp[b]), Cp, "bf16", f"C_hat' b={b}")
        assert_close(host(run.cache[b]), oracle.compressed_cache(Cp, 2), "bf16", f"cache b={b}")
        if b not in (0, 5, 7):
            continue
        # the attention at sampled queries of the first, a middle and the last sequence
        ms = sorted(set([1, 2, 3, 4, 127, 128, 129, 4095, 4096] + rng.integers(1, 4097, size=24).tolist()))
        got = host(run.out[b])
        ref = np.stack([oracle.masked_forward_query(m, qa_o[m - 1], qr_o[m - 1], Cp, 2, dims.d_h)[0] for m in ms])
        assert_close(got[np.array(ms) - 1], ref, "bf16", f"out b={b}")


def test_prefill_equals_gpu_decode_steps():
    """One sequence of the B=8, T=4096 workload: the GPU masked forward at every
    position equals the GPU incremental decode of the same tokens."""
    mc = synth.prefill_model(B=1)
    dims = mc.dims
    W = {k: torch.from_numpy(v).cuda() for k, v in mc.W.items()}
    qa, qr, c, kR = (t.to(torch.bfloat16).contiguous() for t in glue.project(torch.from_numpy(mc.x).cuda(), W))
    T = qa.shape[1]
    run = PrefillRun(dims, "bf16", qa, qr, c, kR, mc.lin).run()
    case = synth.DecodeCase(dims, "bf16", np.array([0]), [np.zeros((0, dims.D), np.float32)], None, None, None,
                            None, mc.lin)
    drun = DecodeRun(case, extra_capacity=T // 2 + 1)
    drun.J_max, drun.P = run.J, run.P
    outs = torch.empty(T, dims.H, dims.r, dtype=torch.float32, device="cuda")
    for t in range(T):
        merge = {"c_new": c[0, t], "kR_new": kR[0, t], "W_c": drun.W_c, "b_c": drun.b_c, "P": drun.P,
                 "J_max": drun.J_max}
        mtla.mtla_decode_attn(drun.md, 1, qa[0, t], qr[0, t], merge, drun.cache.buf, drun.cache.cache_rows,
                              drun.cache.row_stride, drun.cache.offset, drun.cache.capacity, drun.t, drun.cache_len,
                              outs[t], None, drun.ws, drun.ws_bytes, drun.err)
    torch.cuda.synchronize()
    assert int(drun.err.item()) == 0
    assert drun.t.cpu().tolist() == [T] and drun.cache_len.cpu().tolist() == [T // 2]
    # same gates; decode rounds the stored tail row after each token, the
    # prefill only once per stored state: equal within the bf16 tolerance
    assert_close(drun.cache.rows(0, T // 2), host(run.cache[0]), "bf16", "decode-built vs prefill cache")
    assert_close(host(run.out[0]), host(outs), "bf16", "parallel vs incremental (GPU)")


def test_prefill_cache_only_mode():
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=3)
    case = synth.token_case(dims, B=3, T=100, seed=31, dtype="bf16", with_queries=False)
    run = PrefillRun(dims, "bf16", None, None, case.c, case.kR, case.lin, with_out=False).run()
    for b in range(3):
        Cp, _ = _oracle_seq(case.lin, case.c[b], case.kR[b], None, None, dims, with_out=False)
        assert_close(host(run.cache[b]), oracle.compressed_cache(Cp, 3), "bf16", "cache")


def test_stride_mask_matches_oracle_bit_exact():
    for s in (1, 2, 3, 4, 7, 8):
        for T in (1, 9, 64):
            np.testing.assert_array_equal(mtla.mtla_debug_stride_mask(s, T).astype(bool), oracle.stride_mask(T, s))


@pytest.mark.parametrize("s,T", [(1, 256), (2, 96), (3, 400), (4, 128), (5, 80), (8, 1024), (70, 112)])
def test_prefill_tensor_core_path(s, T):
    """bf16 (H, r, d_R) = (8, 256, 32) with T a multiple of 16 runs the tcgen05
    kernel: several key tiles, ragged staircases, queries with no completed group."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=s)
    case = synth.token_case(dims, B=3, T=T, seed=400 + s, dtype="bf16")
    run = PrefillRun(dims, "bf16", case.q_abs, case.q_rope, case.c, case.kR, case.lin).run()
    for b in range(3):
        Cp, o = _oracle_seq(case.lin, case.c[b], case.kR[b], case.q_abs[b], case.q_rope[b], dims)
        assert_close(host(run.out[b]), o, "bf16", f"out s={s} T={T} b={b}")


def test_prefill_tensor_core_repeatable():
    """Two calls give bit-identical outputs (no race between the warp roles)."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=2)
    case = synth.token_case(dims, B=4, T=512, seed=77, dtype="bf16")
    run = PrefillRun(dims, "bf16", case.q_abs, case.q_rope, case.c, case.kR, case.lin).run()
    first = run.out.clone()
    run.run()
    assert torch.equal(first, run.out)


@pytest.mark.parametrize("s,T", [(1, 512), (4, 1024)])
def test_prefill_tensor_core_rising_scores(s, T):
    """Key magnitudes that ramp up along the sequence and larger queries on odd
    heads: the running max jumps at later key tiles for some rows of a warp and
    not others, so the rescale of O in TMEM runs, and runs for part of a warp."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=s)
    case = synth.token_case(dims, B=2, T=T, seed=500 + s, dtype="bf16")
    ramp = (1.0 + 5.0 * np.arange(T) / T)[None, :, None]
    c = synth.cast(case.c * ramp, "bf16")
    kR = synth.cast(case.kR * ramp, "bf16")
    head = np.where(np.arange(8) % 2 == 1, 3.0, 1.0)[None, None, :, None]
    qa = synth.cast(case.q_abs * head, "bf16")
    qr = synth.cast(case.q_rope * head, "bf16")
    run = PrefillRun(dims, "bf16", qa, qr, c, kR, case.lin).run()
    # the bf16 running merge takes W_c at bf16 (fp32 sums), so the C_hat' it
    # stores is the oracle's for the bf16-rounded weights
    lin16 = dict(case.lin, W_c=synth.round_to_bf16(case.lin["W_c"]))
    for b in range(2):
        Cp, _ = _oracle_seq(lin16, c[b], kR[b], qa[b], qr[b], dims, with_out=False)
        # scores reach ~50 here, so the bf16 storage of C_hat' alone moves the
        # fp64 answer by ~4e-2 of its range; the oracle therefore attends over
        # its own C_hat' rounded to the cache's storage type
        o = oracle.masked_forward(qa[b], qr[b], synth.round_to_bf16(Cp), s, dims.d_h)[0]
        assert_close(host(run.out[b]), o, "bf16", f"out s={s} T={T} b={b}")


@pytest.mark.parametrize("s,T", [(1, 300), (2, 1000), (3, 97), (4, 4096), (7, 333), (16, 160), (31, 100), (32, 97),
                                 (33, 70)])
def test_running_merge_strides(s, T):
    """The running merge and the compressed cache alone (cache-only call) for
    strides up to 32 (tensor-core kernel: warp blocks of floor(32/s)*s tokens)
    and 33 (generic kernel), ragged prompt ends included."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=s)
    case = synth.token_case(dims, B=3, T=T, seed=600 + s, dtype="bf16", with_queries=False)
    run = PrefillRun(dims, "bf16", None, None, case.c, case.kR, case.lin, with_out=False).run()
    for b in range(3):
        Cp, _ = _oracle_seq(case.lin, case.c[b], case.kR[b], None, None, dims, with_out=False)
        assert_close(host(run.cp[b]), Cp, "bf16", f"C_hat' s={s} T={T} b={b}")
        assert_close(host(run.cache[b]), oracle.compressed_cache(Cp, s), "bf16", f"cache s={s} T={T} b={b}")


@pytest.mark.parametrize("B,s,T", [(1, 1, 16), (5, 2, 16), (1, 3, 48), (2, 16, 4096), (2, 64, 4096),
                                   (1, 128, 4096)])
def test_prefill_tensor_core_edges(B, s, T):
    """Shapes of the tcgen05 kernel the other cases miss: one 16-token query
    tile per sequence, a single sequence, and long prompts at large strides
    (most query tiles then see one or two key tiles).  Sampled queries around
    the group and tile boundaries vs the oracle, every stored row checked."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=s)
    case = synth.token_case(dims, B=B, T=T, seed=700 + 7 * s + B, dtype="bf16")
    run = PrefillRun(dims, "bf16", case.q_abs, case.q_rope, case.c, case.kR, case.lin).run()
    rng = np.random.default_rng(s + T)
    edges = [1, 2, s - 1, s, s + 1, 2 * s, 2 * s + 1, 16, 17, 64, 65, 128, 129, T - s, T - 1, T]
    ms = sorted(set(m for m in edges + rng.integers(1, T + 1, size=16).tolist() if 1 <= m <= T))
    idx = np.array(ms) - 1
    P = oracle.pe_table(run.J, case.lin["W_p"], case.lin["b_p"])
    for b in range(B):
        Cp = oracle.partial_merge_sequence(case.c[b], case.kR[b], case.lin["W_c"], case.lin["b_c"], P, s)
        ref = np.stack([oracle.masked_forward_query(m, case.q_abs[b, m - 1], case.q_rope[b, m - 1], Cp, s,
                                                    dims.d_h)[0] for m in ms])
        assert_close(host(run.out[b])[idx], ref, "bf16", f"out B={B} s={s} T={T} b={b}")
        assert_close(host(run.cp[b]), Cp, "bf16", f"C_hat' b={b}")
        assert_close(host(run.cache[b]), oracle.compressed_cache(Cp, s), "bf16", f"cache b={b}")


@pytest.mark.parametrize("B,s,T", [(2, 2, 17), (3, 3, 33), (2, 1, 23), (2, 2, 5), (1, 8, 1), (1, 2, 4095),
                                   (1, 2, 4097), (2, 5, 1000)])
def test_prefill_tensor_core_ragged_prompt(B, s, T):
    """Prompt lengths that are not a multiple of the 16-query tile stay on the
    tcgen05 kernel: the last query tile of every sequence is ragged, its rows
    past T read the next sequence's rows (or the fill past the last one) and
    must not be stored.  Sampled queries around the tile and group edges vs
    the oracle; every stored row of C_hat' and the cache is checked, and the
    output rows of the next sequence are not overwritten."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=s)
    case = synth.token_case(dims, B=B, T=T, seed=900 + 7 * s + T, dtype="bf16")
    run = PrefillRun(dims, "bf16", case.q_abs, case.q_rope, case.c, case.kR, case.lin).run()
    rng = np.random.default_rng(s * 31 + T)
    edges = [1, 2, s, s + 1, 15, 16, 17, 32, 33, T - 16, T - 15, T - 1, T]
    ms = sorted(set(m for m in edges + rng.integers(1, T + 1, size=12).tolist() if 1 <= m <= T))
    idx = np.array(ms) - 1
    P = oracle.pe_table(run.J, case.lin["W_p"], case.lin["b_p"])
    for b in range(B):
        Cp = oracle.partial_merge_sequence(case.c[b], case.kR[b], case.lin["W_c"], case.lin["b_c"], P, s)
        ref = np.stack([oracle.masked_forward_query(m, case.q_abs[b, m - 1], case.q_rope[b, m - 1], Cp, s,
                                                    dims.d_h)[0] for m in ms])
        got = host(run.out[b])
        assert np.isfinite(got).all(), "every query of the prompt is written"
        assert_close(got[idx], ref, "bf16", f"out B={B} s={s} T={T} b={b}")
        assert_close(host(run.cp[b]), Cp, "bf16", f"C_hat' b={b}")
        assert_close(host(run.cache[b]), oracle.compressed_cache(Cp, s), "bf16", f"cache b={b}")


@pytest.mark.parametrize("T", [5, 17, 100])
def test_prefill_ragged_prompt_writes_nothing_past_the_end(T):
    """The output lives inside a larger NaN-filled buffer: the ragged last
    query tile must not store the rows past the prompt."""
    dims = synth.Dims(H=8, d_h=64, r=256, d_R=32, s=2)
    B = 2
    case = synth.token_case(dims, B=B, T=T, seed=950 + T, dtype="bf16")
    run = PrefillRun(dims, "bf16", case.q_abs, case.q_rope, case.c, case.kR, case.lin)
    big = torch.full((B * T + 64, dims.H, dims.r), float("nan"), dtype=torch.bfloat16, device="cuda")
    run.out = big[:B * T].view(B, T, dims.H, dims.r)
    run.run()
    assert torch.isnan(big[B * T:].float()).all(), "rows past the prompt were written"
    assert torch.isfinite(big[:B * T].float()).all()
