"""Test-side plumbing for the CUDA library: device buffers for the seeded
inputs, calls through the C ABI binding, and the oracle on the same inputs.

The GPU side and the oracle share only the seeded inputs (mtla_synth); the
oracle computes its own P table, gates and merges in float64."""
from __future__ import annotations

import math

import numpy as np
import torch

import mtla_synth as synth
import oracle
import temporally_compressed_latent_b200 as mtla
from temporally_compressed_latent_b200 import glue

TOL = {"f32": 1e-5, "bf16": 2e-2}      # max|err| <= TOL * max|ref|
TDT = {"f32": torch.float32, "bf16": torch.bfloat16}


def dev(a, dtype="f32"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda().to(TDT[dtype])


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), "non-finite values in the GPU result"
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30))


def assert_close(got, ref, dtype, what=""):
    e = rel_err(got, ref)
    assert e <= TOL[dtype], f"{what}: max|err|/max|ref| = {e:.3e} > {TOL[dtype]:.1e}"
    return e


def mdims(d: synth.Dims, dtype):
    return mtla.dims(d.H, d.d_h, d.r, d.d_R, d.s, dtype)


class DeviceCache:
    """A paged-contiguous cache buffer on the device.

    Sequence b owns `capacity[b]` rows starting at `offset[b]`; `gap` unused
    rows separate sequences, and every row the caller did not fill is NaN so a
    read past a sequence's rows shows up in the results."""

    def __init__(self, rows_list, D, dtype, capacity, row_stride=None, gap=0, fill=float("nan")):
        self.dtype = dtype
        self.D = D
        self.row_stride = row_stride or D
        caps = [int(c) for c in capacity]
        offs, o = [], gap
        for c in caps:
            offs.append(o)
            o += c + gap
        self.cache_rows = o
        self.buf = torch.full((o, self.row_stride), fill, dtype=TDT[dtype], device="cuda")
        for b, rows in enumerate(rows_list):
            if len(rows):
                self.buf[offs[b]:offs[b] + len(rows), :D] = dev(rows, dtype)
        self.offset = torch.tensor(offs, dtype=torch.int64, device="cuda")
        self.capacity = torch.tensor(caps, dtype=torch.int64, device="cuda")
        self.offs = offs

    def rows(self, b, L):
        return host(self.buf[self.offs[b]:self.offs[b] + L, :self.D])


class DecodeRun:
    """Device state of a decode workload plus the calls into the library."""

    def __init__(self, case: synth.DecodeCase, extra_capacity=8, row_stride=None, gap=0, J_extra=4):
        d = case.dims
        self.case = case
        self.dims = d
        self.dtype = case.dtype
        B = case.B
        self.B = B
        caps = [len(r) + extra_capacity for r in case.rows]
        self.cache = DeviceCache(case.rows, d.D, case.dtype, caps, row_stride=row_stride, gap=gap)
        self.t = torch.tensor(case.t_prev, dtype=torch.int32, device="cuda")
        self.cache_len = torch.zeros(B, dtype=torch.int32, device="cuda")
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.J_max = synth.ceil_div(int(max(case.t_prev)) + extra_capacity * d.s, d.s) + J_extra
        lin = case.lin
        self.W_c = torch.from_numpy(lin["W_c"]).cuda()
        self.b_c = torch.from_numpy(lin["b_c"]).cuda()
        self.P = glue.pe_table(self.J_max, torch.from_numpy(lin["W_p"]).cuda(), torch.from_numpy(lin["b_p"]).cuda())
        self.md = mdims(d, case.dtype)
        self.ws_bytes = mtla.mtla_workspace_bytes(self.md, B)
        self.ws = torch.zeros(max(self.ws_bytes, 16), dtype=torch.uint8, device="cuda")
        self.out = torch.zeros(B, d.H, d.r, dtype=torch.float32, device="cuda")
        self.lse = torch.zeros(B, d.H, dtype=torch.float32, device="cuda")

    def step(self, q_abs, q_rope, c_new=None, kR_new=None):
        """One decode call; merges the new token when c_new is given."""
        merge = None
        if c_new is not None:
            self._c = dev(c_new, self.dtype)
            self._k = dev(kR_new, self.dtype)
            merge = {"c_new": self._c, "kR_new": self._k, "W_c": self.W_c, "b_c": self.b_c, "P": self.P,
                     "J_max": self.J_max}
        self._qa = dev(q_abs, self.dtype)
        self._qr = dev(q_rope, self.dtype)
        mtla.mtla_decode_attn(self.md, self.B, self._qa, self._qr, merge, self.cache.buf, self.cache.cache_rows,
                              self.cache.row_stride, self.cache.offset, self.cache.capacity, self.t,
                              self.cache_len, self.out, self.lse, self.ws, self.ws_bytes, self.err)
        torch.cuda.synchronize()
        return host(self.out), host(self.lse)


def oracle_P(lin, J):
    return oracle.pe_table(J, lin["W_p"], lin["b_p"])


def oracle_decode(case: synth.DecodeCase, J, merge=True, q_abs=None, q_rope=None, c_new=None, kR_new=None,
                  rows=None, t_prev=None, seqs=None):
    """Oracle decode step for every (or the listed) sequence; returns o, lse, rows_after."""
    d = case.dims
    P = oracle_P(case.lin, J)
    q_abs = case.q_abs if q_abs is None else q_abs
    q_rope = case.q_rope if q_rope is None else q_rope
    c_new = case.c_new if c_new is None else c_new
    kR_new = case.kR_new if kR_new is None else kR_new
    rows = case.rows if rows is None else rows
    t_prev = case.t_prev if t_prev is None else t_prev
    seqs = range(case.B) if seqs is None else seqs
    outs, lses, new_rows = {}, {}, {}
    for b in seqs:
        if merge:
            r_after, o, lse = oracle.decode_step(rows[b], int(t_prev[b]), d.s, c_new[b], kR_new[b], q_abs[b],
                                                 q_rope[b], case.lin["W_c"], case.lin["b_c"], P, d.d_h)
        else:
            r_after = list(rows[b])
            o, lse = oracle.decode_attention(q_abs[b], q_rope[b], np.asarray(rows[b]), d.d_h)
        outs[b], lses[b], new_rows[b] = o, lse, np.stack(r_after)
    return outs, lses, new_rows


def expected_lengths(t_prev, s, merge=True):
    return [math.ceil((int(t) + (1 if merge else 0)) / s) for t in t_prev]
