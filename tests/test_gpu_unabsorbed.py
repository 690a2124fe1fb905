"""The masked prefill in its un-absorbed form (explicit per-head keys and
values of width d_h) through the C ABI vs the oracle: mtla_prefill_kv
(k = C_hat' W_K^h, v = C_hat' W_V^h) and mtla_prefill_unabsorbed_attn (MTLA
paper notes, "Key designs: stride-aware causal mask" and "decoupled RoPE
with temporal compression"; abstract page, Figure 1)."""
import dataclasses

import numpy as np
import pytest
import torch

import mtla_synth as synth
import oracle
import temporally_compressed_latent_b200 as mtla
from gpu_harness import assert_close, host, mdims
from temporally_compressed_latent_b200 import glue

pytestmark = pytest.mark.gpu


def _gpu_unabsorbed(mc, s):
    """x -> (glue) q_h, q^R, c, k^R -> running merge (cache-only prefill) ->
    k, v -> un-absorbed masked attention.  Returns (out, k, v, C_hat')."""
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
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    mtla.mtla_prefill_masked_attn(md, B, T, None, None, c, kR, W_c, b_c, P, J, cp, cache, None, err)
    k = torch.full((B, T, d.H, d.d_h), float("nan"), dtype=torch.bfloat16, device="cuda")
    v = torch.full_like(k, float("nan"))
    mtla.mtla_prefill_kv(md, B, T, cp, glue.kv_weights(W), k, v, err)
    out = torch.full_like(k, float("nan"))
    mtla.mtla_prefill_unabsorbed_attn(md, B, T, q, qr, k, v, cp, out, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return out, k, v, cp


@pytest.mark.parametrize("s,T", [(1, 33), (2, 1), (2, 17), (2, 64), (3, 130), (5, 200), (2, 129)])
def test_unabsorbed_prefill_small(s, T):
    """B = 2, H = 8, d_h = 64, r = 256, d_R = 32, d = 512: every output against
    the oracle's explicit-key form on its own fp64 projections and merge."""
    dims = dataclasses.replace(synth.MAIN, s=s)
    mc = synth.model_case(dims, B=2, T=T, d=512, seed=2200 + s + T, dtype="bf16")
    out, k, v, cp = _gpu_unabsorbed(mc, s)
    P = oracle.pe_table(synth.ceil_div(T, s) + 2, mc.lin["W_p"], mc.lin["b_p"])
    for b in range(2):
        _, _, c_o, kR_o = oracle.project_inputs(mc.x[b], mc.W)
        Cp = oracle.partial_merge_sequence(c_o, kR_o, mc.lin["W_c"], mc.lin["b_c"], P, s)
        ref = oracle.unabsorbed_heads(mc.x[b], mc.W, Cp, s)
        assert_close(host(out[b]), ref, "bf16", f"out s={s} T={T} b={b}")
        k_ref = np.stack([Cp[:, :256] @ mc.W["W_K"][h] for h in range(8)], axis=1)
        v_ref = np.stack([Cp[:, :256] @ mc.W["W_V"][h] for h in range(8)], axis=1)
        assert_close(host(k[b]), k_ref, "bf16", "k")
        assert_close(host(v[b]), v_ref, "bf16", "v")


def test_unabsorbed_prefill_b8_t4096_sampled():
    """The B=8, T=4096, s=2 prefill workload: sampled queries of two
    sequences against the absorbed oracle times W_V^h (Figure 1), which the
    oracle's pins tie to the explicit-key form."""
    mc = synth.prefill_model()
    out, _, _, _ = _gpu_unabsorbed(mc, 2)
    rng = np.random.default_rng(2300)
    P = oracle.pe_table(synth.ceil_div(4096, 2) + 2, mc.lin["W_p"], mc.lin["b_p"])
    for b in (0, 7):
        qa, qr, c_o, kR_o = oracle.project_inputs(mc.x[b], mc.W)
        Cp = oracle.partial_merge_sequence(c_o, kR_o, mc.lin["W_c"], mc.lin["b_c"], P, 2)
        ms = sorted(set([1, 2, 3, 64, 65, 4095, 4096] + rng.integers(1, 4097, size=12).tolist()))
        got = host(out[b])[np.array(ms) - 1]
        ref = np.stack([np.stack([oracle.masked_forward_query(m, qa[m - 1], qr[m - 1], Cp, 2, 64)[0][h]
                                  @ mc.W["W_V"][h] for h in range(8)]) for m in ms])
        assert_close(got, ref, "bf16", f"out b={b}")


def test_unabsorbed_rejects_other_dims():
    d = mtla.dims(8, 32, 256, 32, 2, "bf16")  # d_h = 32: the kernel is for d_h = 64
    with pytest.raises(mtla.MtlaError) as ei:
        mtla.mtla_prefill_unabsorbed_attn(d, 1, 4, 16, 16, 16, 16, 16, 16, 16)
    assert ei.value.status == 2
