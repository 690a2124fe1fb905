"""The layer maps around the decode attention with the key and value maps
absorbed (MTLA paper notes, "Key designs: decoupled RoPE with temporal
compression"; abstract page, Figure 1), through the C ABI vs the oracle:
mtla_project_in (x -> q_abs, q_rope, c_t, k^R_t with RoPE at the token's
position), mtla_project_out (o -> y = sum_h o_h W_V^h W_O^h), and a whole
decode layer step x -> y at the B=32 decode shapes and at the tiny fp32 shapes."""
import math

import numpy as np
import pytest
import torch

import mtla_synth as synth
import oracle
import temporally_compressed_latent_b200 as mtla
from gpu_harness import DeviceCache, TDT, assert_close, dev, host, mdims
from temporally_compressed_latent_b200 import glue

pytestmark = pytest.mark.gpu


class Proj:
    """Device weights and workspaces of the two maps for one model case."""

    def __init__(self, mc: synth.ModelCase, B: int, dtype: str):
        self.mc, self.B, self.dtype = mc, B, dtype
        self.dims = mc.dims
        self.md = mdims(mc.dims, dtype)
        W = {k: torch.from_numpy(v).cuda() for k, v in mc.W.items()}
        self.W_in, self.W_out = glue.absorbed_weights(W, TDT[dtype])
        self.ws_in_bytes = mtla.mtla_project_workspace_bytes(self.md, B, mc.d, mtla.PROJ_IN)
        self.ws_out_bytes = mtla.mtla_project_workspace_bytes(self.md, B, mc.d, mtla.PROJ_OUT)
        assert self.ws_in_bytes > 0 and self.ws_out_bytes > 0
        self.ws_in = torch.full((self.ws_in_bytes,), 0xFF, dtype=torch.uint8, device="cuda")  # needs no init
        self.ws_out = torch.full((self.ws_out_bytes,), 0xFF, dtype=torch.uint8, device="cuda")
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def project_in(self, x, pos):
        d = self.dims
        B = x.shape[0]
        t = TDT[self.dtype]
        qa = torch.full((B, d.H, d.r), float("nan"), dtype=t, device="cuda")
        qr = torch.full((B, d.H, d.d_R), float("nan"), dtype=t, device="cuda")
        cn = torch.full((B, d.r), float("nan"), dtype=t, device="cuda")
        kn = torch.full((B, d.d_R), float("nan"), dtype=t, device="cuda")
        self._pos = torch.tensor(pos, dtype=torch.int32, device="cuda")
        mtla.mtla_project_in(self.md, B, self.mc.d, x, self.W_in, self._pos, qa, qr, cn, kn, self.ws_in,
                             self.ws_in_bytes, self.err)
        return qa, qr, cn, kn

    def project_out(self, o):
        B = o.shape[0]
        y = torch.full((B, self.mc.d), float("nan"), dtype=torch.float32, device="cuda")
        mtla.mtla_project_out(self.md, B, self.mc.d, o, self.W_out, y, self.ws_out, self.ws_out_bytes, self.err)
        return y


def _oracle_in(mc, x, pos):
    """Per token: the oracle's projections at the token's own position."""
    outs = [oracle.project_inputs(x[b:b + 1], mc.W, pos=[pos[b]]) for b in range(x.shape[0])]
    return [np.concatenate([o[i] for o in outs]) for i in range(4)]


@pytest.mark.parametrize("B", [1, 17, 32, 33, 300])
def test_project_in_bf16(B):
    """d = 512, H = 8, r = 256, d_R = 32: absorbed query, RoPE query and key,
    latent; positions up to 16k.  B = 17 and 33 leave ragged token tiles;
    B = 300 runs two launches (256 + 44)."""
    mc = synth.model_case(synth.MAIN, B=B, T=1, d=512, seed=1100 + B, dtype="bf16")
    x = mc.x[:, 0, :]
    pos = np.random.default_rng(B).integers(0, 16384, size=B)
    pr = Proj(mc, B, "bf16")
    got = pr.project_in(dev(x, "bf16"), pos)
    torch.cuda.synchronize()
    assert int(pr.err.item()) == 0
    ref = _oracle_in(mc, x, pos)
    for name, g, r in zip(("q_abs", "q_rope", "c", "kR"), got, ref):
        assert_close(host(g), r, "bf16", f"{name} B={B}")


@pytest.mark.parametrize("B", [1, 17, 32, 33, 257])
def test_project_out_bf16(B):
    mc = synth.model_case(synth.MAIN, B=B, T=1, d=512, seed=1200 + B, dtype="bf16")
    rng = np.random.default_rng(1300 + B)
    o = rng.standard_normal((B, 8, 256)).astype(np.float32)
    pr = Proj(mc, B, "bf16")
    y = pr.project_out(torch.from_numpy(o).cuda())
    torch.cuda.synchronize()
    assert int(pr.err.item()) == 0
    ref = oracle.absorbed_output(o, mc.W["W_V"], mc.W["W_O"])
    assert_close(host(y), ref, "bf16", f"y B={B}")


def test_project_fp32_tiny():
    """The fp32 maps (SIMT path) at the tiny shapes: 1e-5 tolerance."""
    mc = synth.model_case(synth.TINY, B=5, T=1, d=64, seed=1400, dtype="f32")
    x = mc.x[:, 0, :]
    pos = [0, 1, 7, 63, 79]
    pr = Proj(mc, 5, "f32")
    got = pr.project_in(dev(x, "f32"), pos)
    o = np.random.default_rng(1401).standard_normal((5, 4, 64)).astype(np.float32)
    y = pr.project_out(torch.from_numpy(o).cuda())
    torch.cuda.synchronize()
    for name, g, r in zip(("q_abs", "q_rope", "c", "kR"), got, _oracle_in(mc, x, pos)):
        assert_close(host(g), r, "f32", f"{name}")
    assert_close(host(y), oracle.absorbed_output(o, mc.W["W_V"], mc.W["W_O"]), "f32", "y")


def _layer_step(mc, pr, x, pos, cache: DeviceCache, t, cache_len, J, P, W_c, b_c, dtype):
    """x -> (project_in) -> decode attention with the merge -> (project_out) -> y."""
    d = mc.dims
    B = x.shape[0]
    qa, qr, cn, kn = pr.project_in(x, pos)
    out = torch.empty(B, d.H, d.r, dtype=torch.float32, device="cuda")
    ws_bytes = mtla.mtla_workspace_bytes(pr.md, B)
    ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    merge = {"c_new": cn, "kR_new": kn, "W_c": W_c, "b_c": b_c, "P": P, "J_max": J}
    mtla.mtla_decode_attn(pr.md, B, qa, qr, merge, cache.buf, cache.cache_rows, cache.row_stride, cache.offset,
                          cache.capacity, t, cache_len, out, None, ws, ws_bytes, pr.err)
    return pr.project_out(out)


def test_layer_step_b32_bf16():
    """The B=32 decode shapes (4096 / 4095 processed tokens, s = 2, N(0,1)
    cache rows) with a layer around them: d = 512, x ~ N(0,1), weights
    N(0, 1/fan_in).  The new token's latent and RoPE key come from x."""
    case = synth.decode_uniform()
    d = case.dims
    mc = synth.model_case(d, B=case.B, T=1, d=512, seed=1500, dtype="bf16")
    x = mc.x[:, 0, :]
    pos = case.t_prev.copy()  # the new token is t = t_prev + 1, position t - 1
    pr = Proj(mc, case.B, "bf16")
    caps = [len(r) + 2 for r in case.rows]
    cache = DeviceCache(case.rows, d.D, "bf16", caps)
    t = torch.tensor(case.t_prev, dtype=torch.int32, device="cuda")
    cache_len = torch.zeros(case.B, dtype=torch.int32, device="cuda")
    J = synth.ceil_div(int(case.t_prev.max()) + 1, d.s) + 2
    P = glue.pe_table(J, torch.from_numpy(case.lin["W_p"]).cuda(), torch.from_numpy(case.lin["b_p"]).cuda())
    W_c, b_c = torch.from_numpy(case.lin["W_c"]).cuda(), torch.from_numpy(case.lin["b_c"]).cuda()
    y = _layer_step(mc, pr, dev(x, "bf16"), pos, cache, t, cache_len, J, P, W_c, b_c, "bf16")
    torch.cuda.synchronize()
    assert int(pr.err.item()) == 0
    # oracle: its own projections, merge + attention, absorbed output
    qa, qr, cn, kn = _oracle_in(mc, x, pos)
    P_o = oracle.pe_table(J, case.lin["W_p"], case.lin["b_p"])
    o = np.zeros((case.B, d.H, d.r))
    for b in range(case.B):
        _, o[b], _ = oracle.decode_step(case.rows[b], int(case.t_prev[b]), d.s, cn[b], kn[b], qa[b], qr[b],
                                        case.lin["W_c"], case.lin["b_c"], P_o, d.d_h)
    ref = oracle.absorbed_output(o, mc.W["W_V"], mc.W["W_O"])
    assert_close(host(y), ref, "bf16", "layer output y")
    assert cache_len.cpu().tolist() == [math.ceil((int(x_) + 1) / 2) for x_ in case.t_prev]


def test_layer_steps_tiny_fp32():
    """The tiny fp32 workload end to end through the layer maps: the prompt's
    64 tokens by the masked prefill (its inputs from mtla_project_in at
    positions 0..63), then 16 decode layer steps x -> y; y against the
    oracle's decode loop over all 80 tokens followed by the absorbed output."""
    mc = synth.tiny_e2e(0)
    d = mc.dims
    T0, T = 64, 80
    x = mc.x[0]
    pr = Proj(mc, T, "f32")
    qa, qr, cn, kn = pr.project_in(dev(x, "f32"), list(range(T)))
    J = synth.ceil_div(T, 2) + 2
    P = glue.pe_table(J, torch.from_numpy(mc.lin["W_p"]).cuda(), torch.from_numpy(mc.lin["b_p"]).cuda())
    W_c, b_c = torch.from_numpy(mc.lin["W_c"]).cuda(), torch.from_numpy(mc.lin["b_c"]).cuda()
    cp = torch.empty(1, T0, d.D, dtype=torch.float32, device="cuda")
    cache0 = torch.empty(1, T0 // 2, d.D, dtype=torch.float32, device="cuda")
    pout = torch.empty(1, T0, d.H, d.r, dtype=torch.float32, device="cuda")
    mtla.mtla_prefill_masked_attn(pr.md, 1, T0, qa[None, :T0].contiguous(), qr[None, :T0].contiguous(),
                                  cn[None, :T0].contiguous(), kn[None, :T0].contiguous(), W_c, b_c, P, J, cp,
                                  cache0, pout, pr.err)
    torch.cuda.synchronize()
    rows0 = host(cache0[0]).astype(np.float32)
    cache = DeviceCache([rows0], d.D, "f32", [T // 2 + 2])
    t = torch.tensor([T0], dtype=torch.int32, device="cuda")
    cache_len = torch.zeros(1, dtype=torch.int32, device="cuda")
    one = Proj(mc, 1, "f32")
    ys = [host(pr.project_out(pout[0].contiguous()))]
    for tok in range(T0, T):
        ys.append(host(_layer_step(mc, one, dev(x[tok:tok + 1], "f32"), [tok], cache, t, cache_len, J, P, W_c,
                                   b_c, "f32")))
    torch.cuda.synchronize()
    y = np.concatenate(ys)
    q_o, r_o, c_o, k_o = oracle.project_inputs(x, mc.W)
    P_o = oracle.pe_table(J, mc.lin["W_p"], mc.lin["b_p"])
    loop = oracle.decode_loop(c_o, k_o, q_o, r_o, mc.lin["W_c"], mc.lin["b_c"], P_o, 2, d.d_h)
    ref = oracle.absorbed_output(loop["o"], mc.W["W_V"], mc.W["W_O"])
    assert_close(y, ref, "f32", "layer outputs y, tokens 1..80")
    assert cache_len.cpu().tolist() == [40] and int(one.err.item()) == 0 and int(pr.err.item()) == 0
