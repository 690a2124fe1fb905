"""The training shortcut through the C ABI vs the oracle (MTLA paper notes,
"Key designs: decoupled RoPE with temporal compression": training may use the
uncompressed K^R; "stride-aware causal mask"; "hyper-network temporal
merging"):

- mtla_train_attn_fwd: the masked forward on explicit keys and values and
  the uncompressed RoPE keys, with its log-sum-exp;
- mtla_train_attn_bwd: dq, dq^R, dk, dv and dk^R (summed over heads);
- mtla_train_kv_bwd: dL/dC_hat'_latent through the key and value maps;
- mtla_train_merge_bwd: dc, dW_c, db_c and dP through the latent merge.

Every output buffer starts as NaN, so an element the library fails to write
fails the comparison.  Tolerance: max|err| <= 2e-2 max|ref| (bf16 operands,
fp32 accumulation), tighter where the arithmetic allows."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import mtla_synth as synth
import oracle
import temporally_compressed_latent_b200 as mtla
from gpu_harness import assert_close, host, mdims, rel_err
from temporally_compressed_latent_b200 import glue

pytestmark = pytest.mark.gpu
H, DH, DR, R = 8, 64, 32, 256
NAN = float("nan")


def _bf(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda().to(torch.bfloat16)


def _f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _dims(s):
    return mtla.dims(H, DH, R, DR, s, "bf16")


def _err():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _fwd(d, q, qr, k, v, kR):
    B, T = q.shape[0], q.shape[1]
    out = torch.full_like(q, NAN)
    lse = torch.full((B, T, H), NAN, device="cuda")
    err = _err()
    mtla.mtla_train_attn_fwd(d, B, T, q, qr, k, v, kR, out, lse, err)
    return out, lse, err


def _bwd(d, q, qr, k, v, kR, out, lse, dO):
    B, T = q.shape[0], q.shape[1]
    dq, dqr, dk, dv = (torch.full_like(t, NAN) for t in (q, qr, k, v))
    dkR = torch.full((B, T, DR), NAN, device="cuda")
    wsb = mtla.mtla_train_workspace_bytes(d, B, T, mtla.TRAIN_ATTN_BWD)
    ws = torch.full((wsb,), 0xFF, dtype=torch.uint8, device="cuda")  # NaN bit patterns
    err = _err()
    mtla.mtla_train_attn_bwd(d, B, T, q, qr, k, v, kR, out, lse, dO, dq, dqr, dk, dv, dkR, ws, wsb, err)
    return dq, dqr, dk, dv, dkR, err


def _kv_bwd(d, dk, dv, W_kv):
    B, T = dk.shape[0], dk.shape[1]
    dC = torch.full((B, T, R), NAN, device="cuda")
    wsb = mtla.mtla_train_workspace_bytes(d, B, T, mtla.TRAIN_KV_BWD)
    ws = torch.full((wsb,), 0xFF, dtype=torch.uint8, device="cuda")
    err = _err()
    mtla.mtla_train_kv_bwd(d, B, T, dk, dv, W_kv, dC, ws, wsb, err)
    return dC, err


def _merge_bwd(d, c, W_c, b_c, P, dC):
    B, T = c.shape[0], c.shape[1]
    J_max, D = P.shape
    dc = torch.full((B, T, R), NAN, device="cuda")
    dW = torch.full((R, D), NAN, device="cuda")
    db = torch.full((D,), NAN, device="cuda")
    dP = torch.full((J_max, D), NAN, device="cuda")
    wsb = mtla.mtla_train_workspace_bytes(d, B, T, mtla.TRAIN_MERGE_BWD)
    ws = torch.full((wsb,), 0xFF, dtype=torch.uint8, device="cuda")
    err = _err()
    mtla.mtla_train_merge_bwd(d, B, T, c, W_c, b_c, P, J_max, dC, dc, dW, db, dP, ws, wsb, err)
    return dc, dW, db, dP, err


def _close_floor(got, ref, what, floor=1.0, tol=2e-2):
    """max|err| <= tol * max(max|ref|, floor): for gradients that vanish
    exactly (a single visible column gives softmax a zero slope) the bar is
    relative to the inputs' unit scale instead of to zero."""
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    e = float(np.abs(got - ref).max()) / max(float(np.abs(ref).max()), floor)
    assert e <= tol, f"{what}: max|err|/max(max|ref|, {floor}) = {e:.3e} > {tol:.1e}"


def _rand_attn(B, T, seed):
    rng = np.random.default_rng(seed)
    shapes = [(B, T, H, DH), (B, T, H, DR), (B, T, H, DH), (B, T, H, DH), (B, T, DR), (B, T, H, DH)]
    return [_bf(rng.standard_normal(sh)) for sh in shapes]


@pytest.mark.parametrize("s,T", [(1, 33), (2, 1), (2, 64), (2, 129), (3, 130), (5, 77), (4, 256), (64, 200)])
def test_train_attention_forward_and_backward(s, T):
    """B = 2 sequences, H = 8, d_h = 64, d_R = 32: every output of the forward
    (out, lse) and of the backward (dq, dq^R, dk, dv, dk^R) against the
    oracle on the same bf16 inputs, across strides, ragged last tiles, a
    single token and a stride larger than a tile."""
    q, qr, k, v, kR, dO = _rand_attn(2, T, 700 + 10 * s + T)
    d = _dims(s)
    out, lse, e1 = _fwd(d, q, qr, k, v, kR)
    dq, dqr, dk, dv, dkR, e2 = _bwd(d, q, qr, k, v, kR, out, lse, dO)
    torch.cuda.synchronize()
    assert int(e1.item()) == 0 and int(e2.item()) == 0
    for b in range(2):
        args = [host(t[b]) for t in (q, qr, k, v, kR)]
        o_ref, lse_ref = oracle.shortcut_attention(*args, s)
        assert_close(host(out[b]), o_ref, "bf16", f"out s={s} T={T} b={b}")
        assert float(np.abs(host(lse[b]) - lse_ref).max()) < 1e-3, "lse"
        refs = oracle.shortcut_attention_backward(*args, s, host(dO[b]))
        for name, got, ref in zip(("dq", "dq_rope", "dk", "dv", "dkR"), (dq, dqr, dk, dv, dkR), refs):
            _close_floor(host(got[b]), ref, f"{name} s={s} T={T} b={b}")


@pytest.mark.parametrize("B,T", [(1, 1), (2, 100), (3, 257)])
def test_train_kv_backward(B, T):
    """dC_hat'_latent = sum_h dk_h (W_K^h)^T + dv_h (W_V^h)^T on the tensor cores,
    with M = B T ragged against the 128-row tiles: fp32 accumulation of bf16
    operands, so the error is rounding only."""
    rng = np.random.default_rng(800 + B * T)
    dk = _bf(rng.standard_normal((B, T, H, DH)))
    dv = _bf(rng.standard_normal((B, T, H, DH)))
    W = {"W_K": torch.from_numpy(rng.standard_normal((H, R, DH)) / 16), "W_V": torch.from_numpy(rng.standard_normal((H, R, DH)) / 16)}
    W_kv = glue.kv_weights(W).cuda()
    dC, err = _kv_bwd(_dims(2), dk, dv, W_kv)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    wkv = host(W_kv)  # the bf16 weights the GPU multiplies by
    W_K = np.stack([wkv[h * DH:(h + 1) * DH].T for h in range(H)])
    W_V = np.stack([wkv[H * DH + h * DH:H * DH + (h + 1) * DH].T for h in range(H)])
    for b in range(B):
        ref = oracle.kv_backward(host(dk[b]), host(dv[b]), W_K, W_V)
        assert rel_err(host(dC[b]), ref) < 1e-4, f"dC b={b}"


def _merge_inputs(B, T, s, seed, J_extra=3):
    rng = np.random.default_rng(seed)
    D = R + DR
    c = _bf(rng.standard_normal((B, T, R)))
    W_c = rng.standard_normal((R, D)) / math.sqrt(R)
    b_c = 0.1 * rng.standard_normal(D)
    P = rng.standard_normal((synth.ceil_div(T, s) + J_extra, D))
    dC = rng.standard_normal((B, T, R))
    return c, W_c, b_c, P, dC


def _merge_ref(c, W_c, b_c, P, s, dC):
    B = c.shape[0]
    dc, dW, db, dP = [], 0.0, 0.0, 0.0
    for b in range(B):
        g = oracle.latent_merge_backward(host(c[b]), W_c, b_c, P, s, dC[b])
        dc.append(g[0])
        dW, db, dP = dW + g[1], db + g[2], dP + g[3]
    return np.stack(dc), dW, db, dP


@pytest.mark.parametrize("s,B,T", [(1, 1, 37), (2, 2, 128), (3, 3, 100), (5, 1, 1), (2, 2, 300), (32, 1, 200)])
def test_train_merge_backward(s, B, T):
    """dc, dW_c, db_c and dP through the latent merge: the gate recomputed on
    the tensor cores from bf16 c and W_c, the chain rule in fp32.  The RoPE
    gate channels and the P rows past the sequence are exactly zero."""
    c, W_c, b_c, P, dC = _merge_inputs(B, T, s, 900 + 7 * s + T)
    dc, dW, db, dP, err = _merge_bwd(_dims(s), c, _f32(W_c), _f32(b_c), _f32(P), _f32(dC))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    r_dc, r_dW, r_db, r_dP = _merge_ref(c, W_c, b_c, P, s, dC)
    assert_close(host(dc), r_dc, "bf16", "dc")
    assert_close(host(dW), r_dW, "bf16", "dW_c")
    assert_close(host(db), r_db, "bf16", "db_c")
    assert_close(host(dP), r_dP, "bf16", "dP")
    J = synth.ceil_div(T, s)
    assert (host(dW)[:, R:] == 0).all() and (host(db)[R:] == 0).all()
    assert (host(dP)[:, R:] == 0).all() and (host(dP)[J:] == 0).all()


def _gpu_chain(mc, s, dO):
    """x -> (glue) q, q^R, c, k^R -> running merge -> k, v -> shortcut forward,
    then d_out -> attention backward -> key/value maps -> merge backward."""
    d = dataclasses.replace(mc.dims, s=s)
    md = mdims(d, "bf16")
    W = {k_: torch.from_numpy(v_).cuda() for k_, v_ in mc.W.items()}
    x = torch.from_numpy(mc.x).cuda()
    _, qr, c, kR = (t.to(torch.bfloat16).contiguous() for t in glue.project(x, W))
    q = glue.query_heads(x, W).to(torch.bfloat16)
    B, T = c.shape[0], c.shape[1]
    J = synth.ceil_div(T, s) + 2
    P = glue.pe_table(J, torch.from_numpy(mc.lin["W_p"]).cuda(), torch.from_numpy(mc.lin["b_p"]).cuda())
    W_c, b_c = torch.from_numpy(mc.lin["W_c"]).cuda(), torch.from_numpy(mc.lin["b_c"]).cuda()
    cp = torch.empty(B, T, d.D, dtype=torch.bfloat16, device="cuda")
    cache = torch.empty(B, synth.ceil_div(T, s), d.D, dtype=torch.bfloat16, device="cuda")
    err = _err()
    mtla.mtla_prefill_masked_attn(md, B, T, None, None, c, kR, W_c, b_c, P, J, cp, cache, None, err)
    k = torch.empty(B, T, H, DH, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    W_kv = glue.kv_weights(W)
    mtla.mtla_prefill_kv(md, B, T, cp, W_kv, k, v, err)
    out, lse, e1 = _fwd(md, q, qr, k, v, kR)
    dq, dqr, dk, dv, dkR, e2 = _bwd(md, q, qr, k, v, kR, out, lse, dO)
    dC, e3 = _kv_bwd(md, dk, dv, W_kv)
    dc, dW, db, dPt, e4 = _merge_bwd(md, c, W_c, b_c, P, dC)
    torch.cuda.synchronize()
    assert sum(int(e.item()) for e in (err, e1, e2, e3, e4)) == 0
    return dict(q=q, qr=qr, c=c, kR=kR, out=out, dq=dq, dqr=dqr, dkR=dkR, dC=dC, dc=dc, dW=dW, db=db, dP=dPt, J=J)


def _oracle_chain(mc, s, g, b, dO_b, heads=None):
    """The oracle's training chain for sequence b from the same bf16 q, q^R,
    c, k^R as the GPU got (fp64 from there on)."""
    W = {k_: v_.astype(np.float64) for k_, v_ in mc.W.items()}
    P = oracle.pe_table(g["J"], mc.lin["W_p"], mc.lin["b_p"])
    c = host(g["c"][b])
    Cl = oracle.latent_partial_merge(c, mc.lin["W_c"], mc.lin["b_c"], P, s)
    hs = list(range(H)) if heads is None else heads
    k = np.stack([Cl @ W["W_K"][h] for h in hs], axis=1)
    v = np.stack([Cl @ W["W_V"][h] for h in hs], axis=1)
    q, qr = host(g["q"][b])[:, hs], host(g["qr"][b])[:, hs]
    kR = host(g["kR"][b])
    o, _ = oracle.shortcut_attention(q, qr, k, v, kR, s)
    dq, dqr, dk, dv, dkR = oracle.shortcut_attention_backward(q, qr, k, v, kR, s, dO_b[:, hs])
    return dict(P=P, Cl=Cl, out=o, dq=dq, dqr=dqr, dkR=dkR, dk=dk, dv=dv, W=W, c=c)


@pytest.mark.parametrize("s,T", [(2, 128), (3, 100)])
def test_train_chain_from_layer_input(s, T):
    """The whole training step from the layer input x (B = 2, d = 512): the
    GPU chain against the oracle chain on the same bf16 projections, down to
    the gate parameters' gradients."""
    dims = dataclasses.replace(synth.MAIN, s=s)
    mc = synth.model_case(dims, B=2, T=T, d=512, seed=950 + s + T, dtype="bf16")
    dO = _bf(np.random.default_rng(960 + s).standard_normal((2, T, H, DH)))
    g = _gpu_chain(mc, s, dO)
    dc_ref, dW_ref, db_ref, dP_ref = [], 0.0, 0.0, 0.0
    for b in range(2):
        r = _oracle_chain(mc, s, g, b, host(dO[b]))
        assert_close(host(g["out"][b]), r["out"], "bf16", f"out b={b}")
        assert_close(host(g["dq"][b]), r["dq"], "bf16", f"dq b={b}")
        assert_close(host(g["dqr"][b]), r["dqr"], "bf16", f"dq_rope b={b}")
        assert_close(host(g["dkR"][b]), r["dkR"], "bf16", f"dkR b={b}")
        dCl = oracle.kv_backward(r["dk"], r["dv"], r["W"]["W_K"], r["W"]["W_V"])
        assert_close(host(g["dC"][b]), dCl, "bf16", f"dC b={b}")
        m = oracle.latent_merge_backward(r["c"], mc.lin["W_c"], mc.lin["b_c"], r["P"], s, dCl)
        dc_ref.append(m[0])
        dW_ref, db_ref, dP_ref = dW_ref + m[1], db_ref + m[2], dP_ref + m[3]
    assert_close(host(g["dc"]), np.stack(dc_ref), "bf16", "dc")
    assert_close(host(g["dW"]), dW_ref, "bf16", "dW_c")
    assert_close(host(g["db"]), db_ref, "bf16", "db_c")
    assert_close(host(g["dP"]), dP_ref, "bf16", "dP")


def test_train_b8_t4096_sampled():
    """The B=8, T=4096, s=2 prefill workload as a training step: forward and
    backward outputs of heads 0 and 5 of sequences 0 and 7 in full, the merge
    backward's parameter gradients over all eight sequences (from the GPU's
    own dC, so that this checks the merge backward at full size)."""
    mc = synth.prefill_model()
    dO = _bf(np.random.default_rng(970).standard_normal((8, 4096, H, DH)))
    g = _gpu_chain(mc, 2, dO)
    hs = [0, 5]
    for b in (0, 7):
        r = _oracle_chain(mc, 2, g, b, host(dO[b]), heads=hs)
        for name in ("out", "dq", "dqr"):
            assert_close(host(g[name][b])[:, hs], r[name], "bf16", f"{name} b={b}")
    dC = host(g["dC"])
    P = oracle.pe_table(g["J"], mc.lin["W_p"], mc.lin["b_p"])
    dW_ref, db_ref, dP_ref = 0.0, 0.0, 0.0
    for b in range(8):
        m = oracle.latent_merge_backward(host(g["c"][b]), mc.lin["W_c"], mc.lin["b_c"], P, 2, dC[b])
        if b in (0, 7):
            assert_close(host(g["dc"][b]), m[0], "bf16", f"dc b={b}")
        dW_ref, db_ref, dP_ref = dW_ref + m[1], db_ref + m[2], dP_ref + m[3]
    assert_close(host(g["dW"]), dW_ref, "bf16", "dW_c")
    assert_close(host(g["db"]), db_ref, "bf16", "db_c")
    assert_close(host(g["dP"]), dP_ref, "bf16", "dP")
