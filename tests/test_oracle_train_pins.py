"""Pins for the oracle's training path (the uncompressed-RoPE-key shortcut of
the notes page, *Key designs: decoupled RoPE with temporal compression*, and
its backward pass).

The backward functions are checked against central finite differences of
their own forward definitions, entry by entry, on tiny fp64 cases: a dropped
term, a wrong sign, a wrong index or a group boundary crossed in the wrong
place changes some entry's derivative and fails.  The forwards are tied to the
pinned inference-side functions."""
import dataclasses
import math

import numpy as np
import pytest

import mtla_synth as synth
import oracle
from oracle import mtla_oracle as om


def _num_grad(f, x, eps=1e-6):
    """Central differences of the scalar f() with respect to every entry of x (in place)."""
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + eps
        fp = f()
        x[i] = old - eps
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * eps)
    return g


def _close(got, want, what, tol=1e-6):
    scale = max(1.0, float(np.abs(want).max()))
    err = float(np.abs(got - want).max()) / scale
    assert err < tol, f"{what}: max|err|/max(1, max|ref|) = {err:.3e}"


def _attn_case(T, H, d_h, d_R, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H, d_h))
    qr = rng.standard_normal((T, H, d_R))
    k = rng.standard_normal((T, H, d_h))
    v = rng.standard_normal((T, H, d_h))
    kR = rng.standard_normal((T, d_R))
    G = rng.standard_normal((T, H, d_h))
    return q, qr, k, v, kR, G


@pytest.mark.parametrize("s,T", [(1, 7), (2, 9), (3, 10), (4, 4)])
def test_attention_backward_matches_finite_differences(s, T):
    q, qr, k, v, kR, G = _attn_case(T, 2, 4, 2, 300 + 10 * s + T)
    loss = lambda: float((oracle.shortcut_attention(q, qr, k, v, kR, s)[0] * G).sum())
    got = oracle.shortcut_attention_backward(q, qr, k, v, kR, s, G)
    for name, x, g in zip(("dq", "dq_rope", "dk", "dv", "dkR"), (q, qr, k, v, kR), got):
        _close(g, _num_grad(loss, x), f"{name} s={s} T={T}")


@pytest.mark.parametrize("s,T", [(2, 8), (3, 7)])
def test_kv_backward_matches_finite_differences(s, T):
    """dL/dC_hat'_latent through the key and value maps and the attention."""
    rng = np.random.default_rng(400 + s)
    H, d_h, d_R, r = 2, 4, 2, 6
    q, qr, _, _, kR, G = _attn_case(T, H, d_h, d_R, 410 + s)
    Cp = rng.standard_normal((T, r))
    W_K = rng.standard_normal((H, r, d_h)) / math.sqrt(r)
    W_V = rng.standard_normal((H, r, d_h)) / math.sqrt(r)

    def kv(C):
        return (np.stack([C @ W_K[h] for h in range(H)], axis=1), np.stack([C @ W_V[h] for h in range(H)], axis=1))

    def loss():
        k, v = kv(Cp)
        return float((oracle.shortcut_attention(q, qr, k, v, kR, s)[0] * G).sum())

    k, v = kv(Cp)
    _, _, dk, dv, _ = oracle.shortcut_attention_backward(q, qr, k, v, kR, s, G)
    _close(oracle.kv_backward(dk, dv, W_K, W_V), _num_grad(loss, Cp), f"dC' s={s}")


def _merge_case(T, r, d_R, s, seed):
    rng = np.random.default_rng(seed)
    D = r + d_R
    c = rng.standard_normal((T, r))
    W_c = rng.standard_normal((r, D)) / math.sqrt(r)
    b_c = 0.1 * rng.standard_normal(D)
    P = rng.standard_normal((synth.ceil_div(T, s) + 1, D))
    G = rng.standard_normal((T, r))
    return c, W_c, b_c, P, G


@pytest.mark.parametrize("s,T", [(1, 5), (2, 9), (3, 10), (5, 12)])
def test_merge_backward_matches_finite_differences(s, T):
    c, W_c, b_c, P, G = _merge_case(T, 4, 2, s, 500 + s + T)
    loss = lambda: float((oracle.latent_partial_merge(c, W_c, b_c, P, s) * G).sum())
    got = oracle.latent_merge_backward(c, W_c, b_c, P, s, G)
    for name, x, g in zip(("dc", "dW_c", "db_c", "dP"), (c, W_c, b_c, P), got):
        _close(g, _num_grad(loss, x), f"{name} s={s} T={T}")


def test_latent_merge_is_latent_part_of_running_merge():
    """The shortcut's merge is the pinned running merge's latent channels."""
    dims = dataclasses.replace(synth.MAIN, s=3)
    case = synth.token_case(dims, B=1, T=20, seed=77, dtype="f32")
    P = oracle.pe_table(synth.ceil_div(20, 3) + 1, case.lin["W_p"], case.lin["b_p"])
    full = oracle.partial_merge_sequence(case.c[0], case.kR[0], case.lin["W_c"], case.lin["b_c"], P, 3)
    lat = oracle.latent_partial_merge(case.c[0], case.lin["W_c"], case.lin["b_c"], P, 3)
    np.testing.assert_allclose(lat, full[:, :dims.r], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("s", [1, 2, 3])
def test_shortcut_with_merged_rope_keys_is_the_unabsorbed_forward(s):
    """Given the merged RoPE keys C_hat'_rope in place of K^R, the shortcut's
    attention is the pinned un-absorbed forward; its lse is the log of the
    softmax denominator."""
    dims = dataclasses.replace(synth.MAIN, s=s)
    mc = synth.model_case(dims, B=1, T=23, d=64, seed=610 + s, dtype="f32")
    x = mc.x[0].astype(np.float64)
    W = {k_: v_.astype(np.float64) for k_, v_ in mc.W.items()}
    P = oracle.pe_table(synth.ceil_div(23, s) + 1, mc.lin["W_p"], mc.lin["b_p"])
    _, _, c, kR = oracle.project_inputs(x, W)
    Cp = oracle.partial_merge_sequence(c, kR, mc.lin["W_c"], mc.lin["b_c"], P, s)
    r = dims.r
    H = W["W_K"].shape[0]
    q = np.stack([x @ W["W_Q"][:, h] for h in range(H)], axis=1)
    qr = np.stack([oracle.rope(x @ W["W_QR"][:, h], np.arange(23)) for h in range(H)], axis=1)
    k = np.stack([Cp[:, :r] @ W["W_K"][h] for h in range(H)], axis=1)
    v = np.stack([Cp[:, :r] @ W["W_V"][h] for h in range(H)], axis=1)
    o, lse = oracle.shortcut_attention(q, qr, k, v, Cp[:, r:], s)
    np.testing.assert_allclose(o, oracle.unabsorbed_heads(x, W, Cp, s), rtol=1e-10, atol=1e-12)
    # lse: exp(score - lse) sums to one over the visible columns of every row
    m, h = 17, 1
    cols = np.array(oracle.visible_columns(m, s)) - 1
    sc = (k[cols, h] @ q[m - 1, h] + Cp[cols, r:] @ qr[m - 1, h]) / math.sqrt(dims.d_h)
    assert abs(np.exp(sc - lse[m - 1, h]).sum() - 1.0) < 1e-12


def test_planted_sigmoid_slope_fails_merge_gradient_pin(monkeypatch):
    """A gate squashing function whose derivative is not w (1 - w) (here
    Sigmoid(2x)) makes the backward's gate term wrong: the finite-difference
    pin must catch it."""
    c, W_c, b_c, P, G = _merge_case(6, 4, 2, 2, 520)
    true_sig = om.sigmoid
    monkeypatch.setattr(om, "sigmoid", lambda x: true_sig(2.0 * np.asarray(x)))
    loss = lambda: float((oracle.latent_partial_merge(c, W_c, b_c, P, 2) * G).sum())
    _, dW_c, _, _ = oracle.latent_merge_backward(c, W_c, b_c, P, 2, G)
    with pytest.raises(AssertionError):
        _close(dW_c, _num_grad(loss, W_c), "planted dW_c")


def test_planted_group_boundary_fails_merge_gradient_pin(monkeypatch):
    """Summing dC' across a group boundary (an off-by-one in the reverse
    scan) must fail the pin: open_new_row shifted by one token."""
    c, W_c, b_c, P, G = _merge_case(9, 4, 2, 3, 530)
    loss = lambda: float((oracle.latent_partial_merge(c, W_c, b_c, P, 3) * G).sum())
    num = _num_grad(loss, c)
    true_open = om.opens_new_row
    monkeypatch.setattr(om, "opens_new_row", lambda t, s: true_open(t - 1, s) if t > 1 else True)
    # the forward keeps its own (true) result above; only the backward sees the shift
    dc, _, _, _ = oracle.latent_merge_backward(c, W_c, b_c, P, 3, G)
    with pytest.raises(AssertionError):
        _close(dc, num, "planted dc")
