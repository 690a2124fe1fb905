"""Compression-ratio sweep: B=64 sequences of T=16384 merged tokens at
s in {1, 2, 3, 4, 8} (s = 1 is MLA), then one decode step at t = 16385.

The GPU builds its cache with the prefill's cache-only mode; the oracle merges
the same tokens itself (float64).  The caches of all 64 sequences are
compared at s = 2 and 3 (every fourth sequence at the other strides), and the
decode step on a sample of sequences."""
import math

import numpy as np
import pytest
import torch

import mtla_synth as synth
import oracle
import temporally_compressed_latent_b200 as mtla
from gpu_harness import TDT, assert_close, dev, host, mdims
from temporally_compressed_latent_b200 import glue

pytestmark = pytest.mark.gpu

B, T = 64, 16384


@pytest.mark.parametrize("s", [1, 2, 3, 4, 8])
def test_sweep_decode_step(s):
    tc = synth.sweep_tokens(s, B=B, T=T)
    dims = tc.dims
    D, L = dims.D, synth.ceil_div(T, s)
    J = synth.ceil_div(T + 1, s) + 1
    W_c = torch.from_numpy(tc.lin["W_c"]).cuda()
    b_c = torch.from_numpy(tc.lin["b_c"]).cuda()
    P = glue.pe_table(J, torch.from_numpy(tc.lin["W_p"]).cuda(), torch.from_numpy(tc.lin["b_p"]).cuda())
    c, kR = dev(tc.c, "bf16"), dev(tc.kR, "bf16")
    cp = torch.empty(B, T, D, dtype=torch.bfloat16, device="cuda")
    cache_out = torch.empty(B, L, D, dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    md = mdims(dims, "bf16")
    mtla.mtla_prefill_masked_attn(md, B, T, None, None, c, kR, W_c, b_c, P, J, cp, cache_out, None, err)
    del cp, c, kR
    # paged cache with one spare row per sequence for the decode step's append
    cap = L + 1
    buf = torch.full((B * cap, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    buf.view(B, cap, D)[:, :L] = cache_out
    offset = torch.arange(B, dtype=torch.int64, device="cuda") * cap
    capacity = torch.full((B,), cap, dtype=torch.int64, device="cuda")
    t = torch.full((B,), T, dtype=torch.int32, device="cuda")
    cache_len = torch.zeros(B, dtype=torch.int32, device="cuda")
    qa_np, qr_np, cn_np, kn_np = synth.sweep_step(s, B=B)
    qa, qr, cn, kn = dev(qa_np, "bf16"), dev(qr_np, "bf16"), dev(cn_np, "bf16"), dev(kn_np, "bf16")
    out = torch.empty(B, dims.H, dims.r, dtype=torch.float32, device="cuda")
    ws_bytes = mtla.mtla_workspace_bytes(md, B)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    merge = {"c_new": cn, "kR_new": kn, "W_c": W_c, "b_c": b_c, "P": P, "J_max": J}
    mtla.mtla_decode_attn(md, B, qa, qr, merge, buf, B * cap, D, offset, capacity, t, cache_len, out, None, ws,
                          ws_bytes, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    L_after = math.ceil((T + 1) / s)
    assert cache_len.cpu().tolist() == [L_after] * B
    assert t.cpu().tolist() == [T + 1] * B

    P_o = oracle.pe_table(J, tc.lin["W_p"], tc.lin["b_p"])
    # the cache the running merge builds: every sequence at the pages' strides
    # (2 and 3), every fourth at the others (the fp64 merge of a 16384-token
    # sequence takes a few tenths of a second)
    for b in (range(B) if s in (2, 3) else sorted(set(range(0, B, 4)) | {37, 63})):
        Cp = oracle.partial_merge_sequence(tc.c[b], tc.kR[b], tc.lin["W_c"], tc.lin["b_c"], P_o, s)
        rows = oracle.compressed_cache(Cp, s)
        assert_close(host(cache_out[b]), rows, "bf16", f"s={s} cache b={b}")
        if b not in (0, 37, 63):
            continue
        rows_after, o, _ = oracle.decode_step(list(rows), T, s, cn_np[b], kn_np[b], qa_np[b], qr_np[b],
                                              tc.lin["W_c"], tc.lin["b_c"], P_o, dims.d_h)
        assert_close(host(out[b]), o, "bf16", f"s={s} out b={b}")
        assert_close(host(buf[b * cap + L_after - 1]), rows_after[-1], "bf16", f"s={s} tail b={b}")
