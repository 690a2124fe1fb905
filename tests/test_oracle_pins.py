"""Pins for the fp64 oracle: each test ties it to something other than itself
(values worked by hand from the pages, closed forms, invariants the pages
state, special cases that reduce to a textbook routine, brute force).

Several tests plant a plausible mistake in the oracle (on the CPU) and check
that a pin catches it."""
import json
import math
import os

import numpy as np
import pytest
import torch

import mtla_synth as synth
import oracle
from oracle import mtla_oracle as om


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def _read_bitmap(path):
    rows = [ln.strip() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    return np.array([[ch == "1" for ch in row] for row in rows], dtype=bool)


def _small_case(dims, T, seed):
    case = synth.token_case(dims, B=1, T=T, seed=seed, dtype="f32")
    P = oracle.pe_table(synth.ceil_div(T, dims.s), case.lin["W_p"], case.lin["b_p"])
    return case, P


def _run_both(dims, T, seed):
    case, P = _small_case(dims, T, seed)
    c, kR, qa, qr = case.c[0], case.kR[0], case.q_abs[0], case.q_rope[0]
    Cp = oracle.partial_merge_sequence(c, kR, case.lin["W_c"], case.lin["b_c"], P, dims.s)
    par, par_lse = oracle.masked_forward(qa, qr, Cp, dims.s, dims.d_h)
    seq = oracle.decode_loop(c, kR, qa, qr, case.lin["W_c"], case.lin["b_c"], P, dims.s, dims.d_h)
    return case, P, Cp, par, par_lse, seq


# ---------------------------------------------------------------------------
# worked example (hand-derived fixture)
# ---------------------------------------------------------------------------

def test_worked_example_merge(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "merge_worked_example.json")))
    s = fx["dims"]["s"]
    rows = []
    for tok, expect in zip(fx["tokens"], fx["rows_after"]):
        t = tok["t"]
        j = oracle.group_index(t, s)
        w = oracle.merge_weight(tok["c"], fx["P"][j - 1], fx["W_c"], fx["b_c"])
        rows = oracle.merge_step(rows, t, s, tok["c"], tok["kR"], w)
        np.testing.assert_allclose(np.stack(rows), np.array(expect), rtol=0, atol=1e-15)


def test_worked_example_attention(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "merge_worked_example.json")))
    rows_after = {i + 1: np.array(r) for i, r in enumerate(fx["rows_after"])}
    d_h = fx["dims"]["d_h"]
    for case in fx["attention"]:
        o, _ = oracle.decode_attention(case["q_abs"], case["q_rope"], rows_after[case["after_t"]], d_h)
        np.testing.assert_allclose(o, np.array(case["o"]), rtol=1e-15, atol=1e-15)


# ---------------------------------------------------------------------------
# cache length (closed form ceil(t/s); hand-written table)
# ---------------------------------------------------------------------------

def test_cache_lengths_golden(golden_dir):
    for ln in open(os.path.join(golden_dir, "cache_lengths.txt")):
        if ln.startswith("#") or not ln.strip():
            continue
        s_str, seq = ln.split(":")
        s = int(s_str)
        expect = [int(v) for v in seq.split()]
        dims = synth.Dims(H=1, d_h=4, r=4, d_R=2, s=s)
        case, P = _small_case(dims, len(expect), seed=11)
        out = oracle.decode_loop(case.c[0], case.kR[0], case.q_abs[0], case.q_rope[0],
                                 case.lin["W_c"], case.lin["b_c"], P, s, dims.d_h)
        assert out["lengths"].tolist() == expect


@pytest.mark.parametrize("s", [1, 2, 3, 4, 8])
def test_cache_length_closed_form(s):
    for t in range(0, 4 * s * 5 + 1):
        assert oracle.cache_length(t, s) == math.ceil(t / s)
        if t:
            appended = sum(1 for u in range(1, t + 1) if oracle.opens_new_row(u, s))
            assert appended == math.ceil(t / s)


def test_cache_elements_per_token():
    # Notes, loss/training strategy: 9 d_h l / (2 s), 2.25 d_h l at s = 2.
    for d_h in (16, 64, 128):
        assert oracle.cache_elements_per_token(d_h, 2) == 2.25 * d_h
        for s in (1, 2, 3, 4, 8):
            assert math.isclose(oracle.cache_elements_per_token(d_h, s, layers=3),
                                9 * d_h * 3 / (2 * s))
    # and it is what the decode loop actually stores, at T a multiple of s
    dims = synth.Dims(H=1, d_h=8, r=32, d_R=4, s=4)
    T = 24
    case, P = _small_case(dims, T, seed=3)
    out = oracle.decode_loop(case.c[0], case.kR[0], case.q_abs[0], case.q_rope[0],
                             case.lin["W_c"], case.lin["b_c"], P, dims.s, dims.d_h)
    assert out["rows"].size / T == oracle.cache_elements_per_token(8, 4)


# ---------------------------------------------------------------------------
# mask
# ---------------------------------------------------------------------------

def test_mask_golden(golden_dir):
    np.testing.assert_array_equal(oracle.stride_mask(6, 2),
                                  _read_bitmap(os.path.join(golden_dir, "stride_mask_s2_T6.txt")))
    np.testing.assert_array_equal(oracle.stride_mask(7, 3),
                                  _read_bitmap(os.path.join(golden_dir, "stride_mask_s3_T7.txt")))


@pytest.mark.parametrize("s", [1, 2, 3, 4, 5, 8])
def test_mask_row_counts_and_special_cases(s):
    T = 40
    M = oracle.stride_mask(T, s)
    assert (M.sum(axis=1) == [math.ceil(m / s) for m in range(1, T + 1)]).all()
    assert not np.triu(M, 1).any()                      # never sees the future
    assert M.diagonal().all()                           # always sees itself
    if s == 1:
        np.testing.assert_array_equal(M, np.tril(np.ones((T, T), dtype=bool)))
    assert (oracle.stride_mask(6, 7) == np.eye(6, dtype=bool)).all()   # s > T


# ---------------------------------------------------------------------------
# training-inference consistency (the pages' central claim)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("s,T", [(1, 9), (2, 13), (3, 14), (4, 17), (8, 19)])
def test_parallel_equals_incremental(s, T):
    dims = synth.Dims(H=3, d_h=8, r=16, d_R=4, s=s)
    _, _, Cp, par, par_lse, seq = _run_both(dims, T, seed=100 + s)
    np.testing.assert_allclose(par, seq["o"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(par_lse, seq["lse"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.compressed_cache(Cp, s), seq["rows"], rtol=0, atol=1e-12)


def test_masked_forward_query_matches_full():
    dims = synth.Dims(H=2, d_h=8, r=16, d_R=4, s=3)
    case, _, Cp, par, par_lse, _ = _run_both(dims, 20, seed=7)
    for m in (1, 2, 3, 4, 11, 20):
        o, lse = oracle.masked_forward_query(m, case.q_abs[0, m - 1], case.q_rope[0, m - 1], Cp, 3, 8)
        np.testing.assert_allclose(o, par[m - 1], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse, par_lse[m - 1], rtol=1e-12, atol=1e-12)


def test_fig2a_odd_steps_attend_a_partial_row():
    # Figure 2(a), s = 2: at steps 1, 3, 5 the newest row holds one token only.
    dims = synth.Dims(H=1, d_h=4, r=8, d_R=2, s=2)
    case, P = _small_case(dims, 6, seed=5)
    W_c, b_c = case.lin["W_c"], case.lin["b_c"]
    rows = []
    for t in range(1, 7):
        j = oracle.group_index(t, 2)
        w = oracle.merge_weight(case.c[0, t - 1], P[j - 1], W_c, b_c)
        rows = oracle.merge_step(rows, t, 2, case.c[0, t - 1], case.kR[0, t - 1], w)
        only_t = w * np.concatenate([case.c[0, t - 1], case.kR[0, t - 1]])
        assert np.array_equal(rows[-1], only_t) == (t % 2 == 1)


def test_planted_causal_mask_breaks_consistency(monkeypatch):
    # Plant a plain causal mask: the parallel forward then sees every partial
    # merge, not only the completed groups, and no longer equals decoding.
    dims = synth.Dims(H=2, d_h=8, r=16, d_R=4, s=2)
    monkeypatch.setattr(om, "stride_visible", lambda m, n, s: n <= m)
    _, _, _, par, _, seq = _run_both(dims, 10, seed=9)
    assert np.abs(par - seq["o"]).max() > 1e-3


def test_planted_pre_downsampling_mismatches_inference():
    # Figure 2(b): a cache built by pre-downsampling (each query sees the fully
    # merged group, future tokens included) does not match incremental decoding.
    dims = synth.Dims(H=2, d_h=8, r=16, d_R=4, s=2)
    case, P, Cp, _, _, seq = _run_both(dims, 10, seed=13)
    cache = oracle.compressed_cache(Cp, 2)
    worst = 0.0
    for m in range(1, 11):
        rows = cache[:oracle.group_index(m, 2)]
        o, _ = oracle.decode_attention(case.q_abs[0, m - 1], case.q_rope[0, m - 1], rows, 8)
        worst = max(worst, np.abs(o - seq["o"][m - 1]).max())
    assert worst > 1e-3


# ---------------------------------------------------------------------------
# s = 1: MTLA reduces to MLA, i.e. ordinary causal attention on explicit K, V
# ---------------------------------------------------------------------------

def test_s1_equals_causal_sdpa():
    dims = synth.Dims(H=2, d_h=8, r=16, d_R=4, s=1)
    T, d = 12, 16
    mc = synth.model_case(dims, B=1, T=T, d=d, seed=21, dtype="f32")
    x, W = mc.x[0], mc.W
    q_abs, q_rope, c, kR = oracle.project_inputs(x, W)
    P = oracle.pe_table(T, mc.lin["W_p"], mc.lin["b_p"])
    Cp = oracle.partial_merge_sequence(c, kR, mc.lin["W_c"], mc.lin["b_c"], P, 1)
    o, _ = oracle.masked_forward(q_abs, q_rope, Cp, 1, dims.d_h)
    y = oracle.absorbed_output(o, W["W_V"], W["W_O"])

    # textbook: per-head causal SDPA on [q_h ; q^R_h] vs [K_h ; K^R], V_h
    xt = torch.tensor(x, dtype=torch.float64)
    Cpt = torch.tensor(Cp, dtype=torch.float64)
    qR = torch.tensor(q_rope, dtype=torch.float64)
    heads = []
    for h in range(dims.H):
        q = xt @ torch.tensor(W["W_Q"][:, h, :], dtype=torch.float64)
        K = Cpt[:, :dims.r] @ torch.tensor(W["W_K"][h], dtype=torch.float64)
        V = Cpt[:, :dims.r] @ torch.tensor(W["W_V"][h], dtype=torch.float64)
        Q2 = torch.cat([q, qR[:, h, :]], dim=1)[None, None]
        K2 = torch.cat([K, Cpt[:, dims.r:]], dim=1)[None, None]
        V2 = torch.cat([V, torch.zeros(T, dims.d_R, dtype=torch.float64)], dim=1)[None, None]
        out = torch.nn.functional.scaled_dot_product_attention(
            Q2, K2, V2, is_causal=True, scale=1.0 / math.sqrt(dims.d_h))
        heads.append(out[0, 0, :, :dims.d_h])
    y_ref = torch.cat(heads, dim=1) @ torch.tensor(W["W_O"], dtype=torch.float64)
    np.testing.assert_allclose(y, y_ref.numpy(), rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------
# absorption (Figure 1): absorbed == explicit per-head K and V
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("s", [2, 3])
def test_absorbed_equals_unabsorbed(s):
    dims = synth.Dims(H=3, d_h=8, r=32, d_R=4, s=s)
    T, d = 14, 24
    mc = synth.model_case(dims, B=1, T=T, d=d, seed=30 + s, dtype="f32")
    x, W = mc.x[0], mc.W
    q_abs, q_rope, c, kR = oracle.project_inputs(x, W)
    P = oracle.pe_table(synth.ceil_div(T, s), mc.lin["W_p"], mc.lin["b_p"])
    Cp = oracle.partial_merge_sequence(c, kR, mc.lin["W_c"], mc.lin["b_c"], P, s)
    o, _ = oracle.masked_forward(q_abs, q_rope, Cp, s, dims.d_h)
    y = oracle.absorbed_output(o, W["W_V"], W["W_O"])
    y_ref = oracle.unabsorbed_forward(x, W, Cp, s)
    np.testing.assert_allclose(y, y_ref, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------
# degenerate and invariant cases
# ---------------------------------------------------------------------------

def test_large_stride_keeps_one_entry():
    # News: with s large enough the cache holds about one entry; with s >= T
    # every query sees only its own running merge, so o_m = latent part of C_hat'_m.
    dims = synth.Dims(H=2, d_h=8, r=16, d_R=4, s=32)
    _, _, Cp, par, _, seq = _run_both(dims, 20, seed=17)
    assert (seq["lengths"] == 1).all()
    for m in range(20):
        for h in range(2):
            np.testing.assert_allclose(par[m, h], Cp[m, :16], rtol=1e-14, atol=1e-15)


def test_zero_gate_is_half_sum_pooling():
    # Linear(c) == 0 gives w = sigmoid(0) = 1/2 for every channel, so each cache
    # row is half the plain sum of its group (computed here by a reshape).
    dims = synth.Dims(H=1, d_h=4, r=8, d_R=2, s=3)
    T = 12
    case, P = _small_case(dims, T, seed=19)
    W0 = np.zeros_like(case.lin["W_c"])
    b0 = np.zeros_like(case.lin["b_c"])
    Cp = oracle.partial_merge_sequence(case.c[0], case.kR[0], W0, b0, P, 3)
    full = np.concatenate([case.c[0], case.kR[0]], axis=1).astype(np.float64)
    pooled = 0.5 * full.reshape(T // 3, 3, -1).sum(axis=1)
    np.testing.assert_allclose(oracle.compressed_cache(Cp, 3), pooled, rtol=1e-15, atol=1e-15)
    # the partial state inside a group is half the running sum
    np.testing.assert_allclose(Cp[4], 0.5 * (full[3] + full[4]), rtol=1e-15, atol=1e-15)


def test_gate_range():
    case, P = _small_case(synth.MAIN, 8, seed=23)
    for t in range(8):
        w = oracle.merge_weight(case.c[0, t], P[t // 2], case.lin["W_c"], case.lin["b_c"])
        assert w.shape == (288,) and (w > 0).all() and (w < 1).all()


def test_sigmoid_extremes():
    v = oracle.sigmoid(np.array([-800.0, -1.0, 0.0, 1.0, 800.0]))
    assert v[0] == 0.0 and v[-1] == 1.0 and v[2] == 0.5
    assert math.isclose(v[1] + v[3], 1.0, rel_tol=0, abs_tol=1e-16)


def test_decode_attention_invariants():
    rng = np.random.default_rng(0)
    H, r, d_R, L = 3, 16, 4, 9
    qa, qr = rng.standard_normal((H, r)), rng.standard_normal((H, d_R))
    rows = rng.standard_normal((L, r + d_R))
    o, lse = oracle.decode_attention(qa, qr, rows, 8)
    perm = rng.permutation(L)
    o2, lse2 = oracle.decode_attention(qa, qr, rows[perm], 8)
    np.testing.assert_allclose(o, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, lse2, rtol=1e-13, atol=1e-14)
    const = np.tile(rows[:1], (L, 1))
    o3, lse3 = oracle.decode_attention(qa, qr, const, 8)
    np.testing.assert_allclose(o3, np.tile(rows[0, :r], (H, 1)), rtol=1e-14, atol=1e-14)
    # identical rows: lse = score + ln L
    score = (qa @ rows[0, :r] + qr @ rows[0, r:]) / math.sqrt(8)
    np.testing.assert_allclose(lse3, score + math.log(L), rtol=1e-13, atol=1e-13)


def test_split_combine_identity():
    # Softmax over a union of row sets from the parts' (o, lse): the identity the
    # split-L decode relies on.
    rng = np.random.default_rng(1)
    H, r, d_R = 2, 8, 2
    qa, qr = rng.standard_normal((H, r)), rng.standard_normal((H, d_R))
    rows = rng.standard_normal((23, r + d_R)) * 2
    o, lse = oracle.decode_attention(qa, qr, rows, 4)
    parts = [rows[:5], rows[5:6], rows[6:20], rows[20:]]
    res = [oracle.decode_attention(qa, qr, p, 4) for p in parts]
    lse_all = np.logaddexp.reduce(np.stack([l for _, l in res]), axis=0)
    o_all = sum(np.exp(l - lse_all)[:, None] * oo for oo, l in res)
    np.testing.assert_allclose(lse_all, lse, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(o_all, o, rtol=1e-12, atol=1e-13)


def test_sinusoid_known_values():
    pe = oracle.sinusoidal_pe(50, 12)
    assert (pe[0, 0::2] == 0).all() and (pe[0, 1::2] == 1).all()
    np.testing.assert_allclose(pe[:, 0], np.sin(np.arange(50)), rtol=0, atol=1e-15)
    np.testing.assert_allclose(pe[:, 1], np.cos(np.arange(50)), rtol=0, atol=1e-15)
    np.testing.assert_allclose(pe[:, 0::2] ** 2 + pe[:, 1::2] ** 2, 1.0, rtol=0, atol=1e-15)
    # last pair has the slowest frequency 10000^(-10/12)
    np.testing.assert_allclose(pe[7, 10], math.sin(7 * 10000 ** (-10 / 12)), rtol=0, atol=1e-15)


def test_rope_properties():
    rng = np.random.default_rng(2)
    d_R = 8
    q = rng.standard_normal((1, d_R))
    k = rng.standard_normal((1, d_R))
    np.testing.assert_array_equal(oracle.rope(q, [0]), q)
    for p in (1, 7, 300):
        np.testing.assert_allclose(np.linalg.norm(oracle.rope(q, [p])), np.linalg.norm(q), rtol=1e-14)
    # scores depend only on the position difference
    a = oracle.rope(q, [9]) @ oracle.rope(k, [4]).T
    b = oracle.rope(q, [105]) @ oracle.rope(k, [100]).T
    np.testing.assert_allclose(a, b, rtol=1e-12)
    # pair 0 rotates by exactly the position (theta_0 = 1)
    e0 = np.zeros((1, d_R)); e0[0, 0] = 1.0
    np.testing.assert_allclose(oracle.rope(e0, [0.5])[0, :2], [math.cos(0.5), math.sin(0.5)], atol=1e-16)


def test_planted_wrong_scale_fails_sdpa_pin(monkeypatch):
    # A softmax scale of 1/sqrt(d_h + d_R) (instead of 1/sqrt(d_h)) must not
    # pass the causal-SDPA pin: plant it and compare directly.
    dims = synth.Dims(H=2, d_h=8, r=16, d_R=4, s=1)
    T = 10
    mc = synth.model_case(dims, B=1, T=T, d=16, seed=21, dtype="f32")
    q_abs, q_rope, c, kR = oracle.project_inputs(mc.x[0], mc.W)
    P = oracle.pe_table(T, mc.lin["W_p"], mc.lin["b_p"])
    Cp = oracle.partial_merge_sequence(c, kR, mc.lin["W_c"], mc.lin["b_c"], P, 1)
    good, _ = oracle.masked_forward(q_abs, q_rope, Cp, 1, dims.d_h)
    bad, _ = oracle.masked_forward(q_abs, q_rope, Cp, 1, dims.d_h + dims.d_R)
    assert np.abs(good - bad).max() > 1e-3


def test_synth_bf16_rounding():
    v = np.array([1.0, 1.00390625, 1.005859375, -2.0 ** -130, 3.0e38], dtype=np.float32)
    out = synth.round_to_bf16(v)
    t = torch.tensor(v).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(out, t)
    x = np.random.default_rng(3).standard_normal(10000).astype(np.float32)
    np.testing.assert_array_equal(synth.round_to_bf16(x),
                                  torch.tensor(x).to(torch.bfloat16).to(torch.float32).numpy())


def test_project_inputs_at_a_position():
    """A token projected on its own at position p gives row p of the whole
    sequence's projections (RoPE depends on the position only)."""
    mc = synth.tiny_e2e(0)
    x = mc.x[0]
    full = oracle.project_inputs(x, mc.W)
    for p in (0, 5, 63, 79):
        one = oracle.project_inputs(x[p:p + 1], mc.W, pos=[p])
        for a, b in zip(one, full):
            np.testing.assert_allclose(a[0], b[p], rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# more planted mistakes: each plausible slip in the oracle fails a pin
# ---------------------------------------------------------------------------

def test_planted_dropped_rope_term_fails_absorption_pin(monkeypatch):
    # the score loses its q^R . k^R term in the absorbed forward; the explicit
    # per-head brute force keeps it
    real = om.masked_forward

    def planted(q_abs, q_rope, Cp, s, d_h):
        return real(q_abs, np.zeros_like(np.asarray(q_rope, dtype=np.float64)), Cp, s, d_h)

    monkeypatch.setattr(om, "masked_forward", planted)
    dims = synth.Dims(H=3, d_h=8, r=32, d_R=4, s=2)
    T, d = 14, 24
    mc = synth.model_case(dims, B=1, T=T, d=d, seed=32, dtype="f32")
    q_abs, q_rope, c, kR = oracle.project_inputs(mc.x[0], mc.W)
    P = oracle.pe_table(synth.ceil_div(T, 2), mc.lin["W_p"], mc.lin["b_p"])
    Cp = oracle.partial_merge_sequence(c, kR, mc.lin["W_c"], mc.lin["b_c"], P, 2)
    y = oracle.absorbed_output(om.masked_forward(q_abs, q_rope, Cp, 2, dims.d_h)[0], mc.W["W_V"], mc.W["W_O"])
    assert np.abs(y - oracle.unabsorbed_forward(mc.x[0], mc.W, Cp, 2)).max() > 1e-3


def test_planted_wrong_sign_fails_worked_example(monkeypatch, golden_dir):
    # the in-place update subtracts the gated entry instead of adding it
    def planted(rows, t, s, c_t, kR_t, w):
        entry = np.asarray(w) * np.concatenate([np.asarray(c_t, np.float64), np.asarray(kR_t, np.float64)])
        rows = [np.array(r_, dtype=np.float64) for r_ in rows]
        if om.opens_new_row(t, s):
            rows.append(entry)
        else:
            rows[-1] = rows[-1] - entry
        return rows

    monkeypatch.setattr(om, "merge_step", planted)
    monkeypatch.setattr(oracle, "merge_step", planted)
    with pytest.raises(AssertionError):
        test_worked_example_merge(golden_dir)


def test_planted_off_by_one_group_fails_length_golden(monkeypatch, golden_dir):
    # j(t) = floor(t/s) + 1 agrees with ceil(t/s) except when s divides t
    monkeypatch.setattr(om, "group_index", lambda t, s: t // s + 1)
    monkeypatch.setattr(oracle, "group_index", lambda t, s: t // s + 1)
    # the golden lengths, or the merge's own check of the row count, fail
    with pytest.raises((AssertionError, ValueError)):
        test_cache_lengths_golden(golden_dir)


def test_planted_wrong_pe_row_fails_consistency(monkeypatch):
    # the parallel forward's running merge gates token n with the P row of the
    # next group (j instead of j - 1); decoding keeps the right row
    def planted(c, kR, W_c, b_c, P, s):
        c, kR, P = (np.asarray(a, dtype=np.float64) for a in (c, kR, P))
        pre = c @ np.asarray(W_c, np.float64) + np.asarray(b_c, np.float64)
        Cp = np.zeros((c.shape[0], pre.shape[1]))
        for n in range(1, c.shape[0] + 1):
            j = om.group_index(n, s)
            e = om.sigmoid(pre[n - 1] * P[j]) * np.concatenate([c[n - 1], kR[n - 1]])
            Cp[n - 1] = e if om.opens_new_row(n, s) else Cp[n - 2] + e
        return Cp

    dims = synth.Dims(H=2, d_h=8, r=16, d_R=4, s=2)
    case = synth.token_case(dims, B=1, T=10, seed=41, dtype="f32")
    P = oracle.pe_table(8, case.lin["W_p"], case.lin["b_p"])
    args = (case.c[0], case.kR[0], case.lin["W_c"], case.lin["b_c"], P, 2)
    seq = oracle.decode_loop(case.c[0], case.kR[0], case.q_abs[0], case.q_rope[0], case.lin["W_c"], case.lin["b_c"],
                             P, 2, dims.d_h)
    good = oracle.masked_forward(case.q_abs[0], case.q_rope[0], oracle.partial_merge_sequence(*args), 2, 8)[0]
    np.testing.assert_allclose(good, seq["o"], rtol=1e-11, atol=1e-12)
    monkeypatch.setattr(om, "partial_merge_sequence", planted)
    bad = oracle.masked_forward(case.q_abs[0], case.q_rope[0], om.partial_merge_sequence(*args), 2, 8)[0]
    assert np.abs(bad - seq["o"]).max() > 1e-3


def test_planted_transposed_value_map_fails_absorption_pin(monkeypatch):
    # the output side applies W_V^h transposed (square when r == d_h)
    def planted(o, W_V, W_O):
        o, W_V, W_O = (np.asarray(a, dtype=np.float64) for a in (o, W_V, W_O))
        H, d_h = W_V.shape[0], W_V.shape[2]
        return sum((o[:, h, :] @ W_V[h].T) @ W_O[h * d_h:(h + 1) * d_h, :] for h in range(H))

    dims = synth.Dims(H=2, d_h=8, r=8, d_R=4, s=2)
    T, d = 12, 16
    mc = synth.model_case(dims, B=1, T=T, d=d, seed=43, dtype="f32")
    q_abs, q_rope, c, kR = oracle.project_inputs(mc.x[0], mc.W)
    P = oracle.pe_table(synth.ceil_div(T, 2), mc.lin["W_p"], mc.lin["b_p"])
    Cp = oracle.partial_merge_sequence(c, kR, mc.lin["W_c"], mc.lin["b_c"], P, 2)
    o = oracle.masked_forward(q_abs, q_rope, Cp, 2, dims.d_h)[0]
    ref = oracle.unabsorbed_forward(mc.x[0], mc.W, Cp, 2)
    np.testing.assert_allclose(oracle.absorbed_output(o, mc.W["W_V"], mc.W["W_O"]), ref, rtol=1e-11, atol=1e-12)
    monkeypatch.setattr(om, "absorbed_output", planted)
    assert np.abs(om.absorbed_output(o, mc.W["W_V"], mc.W["W_O"]) - ref).max() > 1e-3



@pytest.mark.parametrize("s", [1, 2, 3])
def test_unabsorbed_heads_equal_absorbed_times_value_map(s):
    """Figure 1 per head: the explicit-key form's o_h equals the absorbed
    form's o_h (width r) times W_V^h, and concatenated through W_O it is the
    brute-force layer output."""
    dims = synth.Dims(H=3, d_h=8, r=32, d_R=4, s=s)
    T, d = 13, 24
    mc = synth.model_case(dims, B=1, T=T, d=d, seed=50 + s, dtype="f32")
    q_abs, q_rope, c, kR = oracle.project_inputs(mc.x[0], mc.W)
    P = oracle.pe_table(synth.ceil_div(T, s), mc.lin["W_p"], mc.lin["b_p"])
    Cp = oracle.partial_merge_sequence(c, kR, mc.lin["W_c"], mc.lin["b_c"], P, s)
    heads = oracle.unabsorbed_heads(mc.x[0], mc.W, Cp, s)
    o_abs, _ = oracle.masked_forward(q_abs, q_rope, Cp, s, dims.d_h)
    for h in range(dims.H):
        np.testing.assert_allclose(heads[:, h, :], o_abs[:, h, :] @ mc.W["W_V"][h], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(heads.reshape(T, -1) @ mc.W["W_O"], oracle.unabsorbed_forward(mc.x[0], mc.W, Cp, s),
                               rtol=1e-11, atol=1e-12)
