"""Benchmark of the MTLA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one call of mtla_decode_attn with the merge fused: every sequence
merges its new token into the compressed cache and attends all ceil(t/s)
rows.  Workload: B=32 sequences, H=8, d_h=64, r=256, d_R=32, s=2, 4096
processed tokens in even sequences (the new token opens row 2049) and 4095 in
odd ones (row 2048 is completed in place); cache rows, queries and the new
token ~ N(0,1), bf16 storage.  Sixteen independent replicas of that state
(~600 MB, more than the 126 MB L2) are visited in turn, so every step streams
its cache from HBM; each replica's state really advances (t grows by one per
visit, so the caches grow by ~2% over a default run) and the algorithmic
bytes are counted from the exact lengths of every step.

Metric: decode query-steps per second (sequences x steps / s) and the decode
kernel's achieved HBM GB/s against the measured copy bandwidth.  With
--gpus N (one process per GPU, torchrun), every rank runs its own B=32
workload (independent sequences: no collective on the data path); the time
is the max over ranks and value counts all ranks' query-steps.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mtla_synth as synth  # noqa: E402

METRIC = "MTLA decode query-steps/sec and achieved HBM GB/s (% of roofline) on 1 B200"
UNIT = "query-steps/s"
WORKLOAD = ("decode step bf16 with fused merge: B=32, H=8, d_h=64, r=256, d_R=32, s=2, "
            "4096/4095 processed tokens (2049/2048 cache rows)")
ROW_BYTES = 288 * 2
N_REPLICAS = 16
E2E_STEPS = 500
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "decode_tc_b32_s2.md")
KERNEL_SOURCES = ["temporally_compressed_latent_b200/csrc/decode_tc.cu",
                  "temporally_compressed_latent_b200/csrc/kernels.cuh",
                  "temporally_compressed_latent_b200/csrc/mtla_common.cuh"]


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def profiled_traffic():
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    if not os.path.exists(PROFILE_SUMMARY):
        return None
    vals = {}
    for ln in open(PROFILE_SUMMARY):
        if ln.startswith("- ") and ":" in ln:
            k, v = ln[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha") != kernel_source_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch_full_size"])
    except (KeyError, ValueError):
        return None


def max_over_ranks(value: float, dist, device) -> float:
    """The largest of all ranks' values (every rank calls this, in the same
    order); the value itself on a single process."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def decode_step_bytes(t_after, d) -> int:
    """Algorithmic bytes of one decode step with the merge, for B sequences that
    hold t_after[b] tokens after it: every cache row read once for all heads,
    the tail row written, the queries, the new token, out and lse, W_c and b_c
    once, one P row per sequence."""
    B = len(t_after)
    rows = int(sum(synth.ceil_div(int(x), d.s) for x in t_after))
    return (rows * ROW_BYTES + B * ROW_BYTES + B * d.H * d.D * 2 + B * d.D * 2 + B * d.H * d.r * 4 +
            B * d.H * 4 + d.r * d.D * 4 + d.D * 4 + B * d.D * 4)


def job_throughput(world: int, units_per_rank_step: int, steps: int, ms_max: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return world * units_per_rank_step * steps / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, read only)
# ---------------------------------------------------------------------------
class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self._nv = pynvml
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self._nv = None

    _NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
              0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
              0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = self._reasons_fn(self._h)
                for bit, name in self._NAMES.items():
                    if mask & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._nv is not None:
            self._t.join()

    def report(self):
        if self._nv is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
class Replica:
    def __init__(self, case, torch, mtla, glue, capacity_extra, J_max, dev):
        d = case.dims
        B = case.B
        self.B = B
        L0 = [len(r) for r in case.rows]
        cap = max(L0) + capacity_extra
        self.cap = cap
        self.cache_rows = B * cap
        host_buf = np.zeros((B, cap, d.D), dtype=np.float32)
        for b, r in enumerate(case.rows):
            host_buf[b, :len(r)] = r
        self.cache = torch.from_numpy(host_buf).to(dev).to(torch.bfloat16).reshape(B * cap, d.D)
        del host_buf
        self.offset = (torch.arange(B, dtype=torch.int64, device=dev) * cap).contiguous()
        self.capacity = torch.full((B,), cap, dtype=torch.int64, device=dev)
        self.t0 = case.t_prev.copy()
        self.t = torch.tensor(case.t_prev, dtype=torch.int32, device=dev)
        self.cache_len = torch.zeros(B, dtype=torch.int32, device=dev)
        bf = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev).to(torch.bfloat16)
        self.q_abs, self.q_rope = bf(case.q_abs), bf(case.q_rope)
        self.c_new, self.kR_new = bf(case.c_new), bf(case.kR_new)
        self.out = torch.empty(B, d.H, d.r, dtype=torch.float32, device=dev)
        self.lse = torch.empty(B, d.H, dtype=torch.float32, device=dev)


def run_ours(args, rank, world, local_rank):
    import torch
    import temporally_compressed_latent_b200 as mtla
    from temporally_compressed_latent_b200 import glue

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    case = synth.decode_uniform(B=32, seed=2)
    d = case.dims
    B = case.B
    W, K = args.warmup, args.steps
    # the timed graph is replayed twice (an untimed first replay, then the
    # timed one), so every replica needs room for W + 2K steps plus e2e
    visits = math.ceil((W + 2 * K + E2E_STEPS + 8) / N_REPLICAS) + 1
    extra = visits // d.s + 4
    J_max = synth.ceil_div(int(case.t_prev.max()) + visits + 8, d.s) + 1
    W_c = torch.from_numpy(case.lin["W_c"]).to(dev)
    b_c = torch.from_numpy(case.lin["b_c"]).to(dev)
    P = glue.pe_table(J_max, torch.from_numpy(case.lin["W_p"]).to(dev), torch.from_numpy(case.lin["b_p"]).to(dev))
    md = mtla.dims(d.H, d.d_h, d.r, d.d_R, d.s, "bf16")
    reps = [Replica(case, torch, mtla, glue, extra, J_max, dev) for _ in range(N_REPLICAS)]
    ws_bytes = mtla.mtla_workspace_bytes(md, B)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(rep, st):
        merge = {"c_new": rep.c_new, "kR_new": rep.kR_new, "W_c": W_c, "b_c": b_c, "P": P, "J_max": J_max}
        mtla.mtla_decode_attn(md, B, rep.q_abs, rep.q_rope, merge, rep.cache, rep.cache_rows, d.D, rep.offset,
                              rep.capacity, rep.t, rep.cache_len, rep.out, rep.lse, ws, ws_bytes, err, stream=st)

    # algorithmic bytes of every step, from the exact lengths the state goes through
    visit = [0] * N_REPLICAS

    def step_bytes(i):
        rep_i = i % N_REPLICAS
        v = visit[rep_i]
        visit[rep_i] += 1
        return decode_step_bytes(case.t_prev + v + 1, d)

    # warm-up graph, the untimed first replay of the timed graph, the timed replay
    bytes_per_step = [step_bytes(i) for i in list(range(W)) + list(range(W, W + K)) * 2]
    timed_bytes = bytes_per_step[W + K:]

    # capture W warm-up steps and K timed steps as two CUDA graphs (launch cost
    # of a ~6 us kernel must not be Python's); replica i % 8 at step i
    torch.cuda.synchronize()
    # one call per replica outside capture without a merge (no state change):
    # sets the kernel's attributes and checks the arguments before capture
    for rp in reps:
        mtla.mtla_decode_attn(md, B, rp.q_abs, rp.q_rope, None, rp.cache, rp.cache_rows, d.D, rp.offset,
                              rp.capacity, rp.t, rp.cache_len, rp.out, rp.lse, ws, ws_bytes, err, stream=stream)
    torch.cuda.synchronize()
    g_warm, g_timed = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_warm, stream=stream, capture_error_mode="thread_local"):
        for i in range(W):
            step(reps[i % N_REPLICAS], torch.cuda.current_stream())
    with torch.cuda.graph(g_timed, stream=stream, capture_error_mode="thread_local"):
        for i in range(W, W + K):
            step(reps[i % N_REPLICAS], torch.cuda.current_stream())
    torch.cuda.synchronize()

    # the first replay of a graph pays its upload, and the replicas the warm-up
    # did not reach are cold: replay the timed graph once untimed, so the timed
    # replay measures steady-state steps whatever K and W are
    with torch.cuda.stream(stream):
        g_warm.replay()
        g_timed.replay()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        # a short device-side sleep keeps the GPU busy while the host launches
        # the graph, so the timed region holds steps only, not launch latency
        with torch.cuda.stream(stream):
            torch.cuda._sleep(200_000)
        e0.record(stream)
        with torch.cuda.stream(stream):
            g_timed.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    dev_err = int(err.item())
    if dev_err:
        raise RuntimeError(f"device error bits {dev_err} during the timed steps")
    ms_max = max_over_ranks(ms, dist, dev)
    ms_step = ms_max / K
    value = job_throughput(world, B, K, ms_max)

    hbm_peak, _, _, peak_kind = measured_peaks()
    achieved_gbs = (sum(timed_bytes) / K) / (ms / K / 1e3) / 1e9
    traffic = profiled_traffic()

    # end to end through the public API with host buffers: per step, H2D of the
    # step's inputs from pinned memory, the call, D2H of the result, and a sync
    e2e = run_e2e(torch, mtla, md, case, reps, W_c, b_c, P, J_max, ws, ws_bytes, err, stream, dev, K, W)

    prefill = None
    if not args.no_prefill and rank == 0:
        prefill = run_prefill(torch, mtla, glue, dev)
    configs = None
    if not args.no_configs and rank == 0:
        configs = run_configs(torch, mtla, glue, dev, set(args.configs.split(",")))

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1) cache rows, queries and new tokens)",
        "config": {"workload": WORKLOAD, "B_per_gpu": B, "H": d.H, "d_h": d.d_h, "r": d.r, "d_R": d.d_R,
                   "s": d.s, "parallelism": f"independent sequences per GPU x{world}",
                   "l2": f"inputs larger than L2: {N_REPLICAS} rotating cache replicas "
                         f"(~{N_REPLICAS * 37.8:.0f} MB > 126 MB L2)",
                   "timing": "CUDA graph of K steps (3 kernels each: gate and tail row, attention, split combine, "
                             "chained by programmatic dependent launch), replayed once untimed, then timed with "
                             "CUDA events on the launching stream"},
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved_gbs / hbm_peak, "traffic": traffic,
                     "kernel": "mtla::dtc::decode_tc_kernel with its merge and split-combine kernels (the whole step)",
                     "peak_kind": f"{peak_kind} copy bandwidth",
                     "algorithmic_bytes_per_launch": sum(timed_bytes) / K},
        "gpu_launches": 3 * K,  # merge, decode and split-combine kernels per step
        "e2e": e2e,
        "clocks": clk.report(),
    }
    if prefill:
        res["prefill"] = prefill
    if configs:
        res["configs"] = configs
    if args.cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    return res


def run_e2e(torch, mtla, md, case, reps, W_c, b_c, P, J_max, ws, ws_bytes, err, stream, dev, K, W):
    """The decode step through the public API with host buffers: every step
    copies its inputs (queries, RoPE queries, new latents, new RoPE keys,
    packed in one pinned buffer) to the device in one copy, runs
    mtla_decode_attn, reads `out` back and synchronises."""
    B = case.B
    d = case.dims
    parts = [(B, d.H, d.r), (B, d.H, d.d_R), (B, d.r), (B, d.d_R)]  # bf16 each
    sizes = [int(np.prod(sh)) * 2 for sh in parts]
    offs = [0]
    for n_b in sizes[:-1]:
        offs.append(offs[-1] + (n_b + 15) // 16 * 16)
    total = offs[-1] + sizes[-1]
    h_in = torch.empty(total, dtype=torch.uint8, pin_memory=True)
    d_in = torch.empty(total, dtype=torch.uint8, device=dev)
    h_out = torch.empty((B, d.H, d.r), dtype=torch.float32, pin_memory=True)

    def view(buf, k):
        return buf[offs[k]:offs[k] + sizes[k]].view(torch.bfloat16).view(parts[k])

    for k, arr in enumerate([case.q_abs, case.q_rope, case.c_new, case.kR_new]):
        view(h_in, k).copy_(torch.from_numpy(arr).to(torch.bfloat16))
    qa, qr, cn, kn = (view(d_in, k) for k in range(4))
    n = min(K, E2E_STEPS)
    h2d = sum(sizes)
    d2h = h_out.numel() * 4

    merge = {"c_new": cn, "kR_new": kn, "W_c": W_c, "b_c": b_c, "P": P, "J_max": J_max}
    handle = stream.cuda_stream  # the calls' stream (current inside the block below)

    def one(i):
        rep = reps[i % N_REPLICAS]
        d_in.copy_(h_in, non_blocking=True)
        mtla.mtla_decode_attn(md, B, qa, qr, merge, rep.cache, rep.cache_rows, d.D, rep.offset,
                              rep.capacity, rep.t, rep.cache_len, rep.out, rep.lse, ws, ws_bytes, err,
                              stream=handle)
        h_out.copy_(rep.out, non_blocking=True)
        stream.synchronize()

    # the replicas may run out of spare rows: e2e reuses at most n steps
    with torch.cuda.stream(stream):
        for i in range(3):
            one(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(n):
            one(3 + i)
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    return {"value": B * n / (ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n, "ms_per_step": ms / n}


def run_prefill(torch, mtla, glue, dev):
    """Companion measurement: the masked parallel forward, B=8, T=4096, s=2."""
    mc = synth.prefill_model()
    d = mc.dims
    W = {k: torch.from_numpy(v).to(dev) for k, v in mc.W.items()}
    qa, qr, c, kR = (t.to(torch.bfloat16).contiguous() for t in glue.project(torch.from_numpy(mc.x).to(dev), W))
    B, T = c.shape[0], c.shape[1]
    J = synth.ceil_div(T, d.s) + 1
    P = glue.pe_table(J, torch.from_numpy(mc.lin["W_p"]).to(dev), torch.from_numpy(mc.lin["b_p"]).to(dev))
    W_c = torch.from_numpy(mc.lin["W_c"]).to(dev)
    b_c = torch.from_numpy(mc.lin["b_c"]).to(dev)
    cp = torch.empty(B, T, d.D, dtype=torch.bfloat16, device=dev)
    cache = torch.empty(B, J - 1, d.D, dtype=torch.bfloat16, device=dev)
    out = torch.empty(B, T, d.H, d.r, dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    md = mtla.dims(d.H, d.d_h, d.r, d.d_R, d.s, "bf16")
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def call(with_out=True):
        mtla.mtla_prefill_masked_attn(md, B, T, qa, qr, c, kR, W_c, b_c, P, J, cp, cache,
                                      out if with_out else None, err)

    def timed(with_out):
        for _ in range(3):
            call(with_out)
        torch.cuda.synchronize()
        times = []
        for _ in range(7):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            call(with_out)
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        return statistics.median(times)

    ms = timed(True)
    ms_merge = timed(False)  # cache-only call: the running-merge kernel alone
    if int(err.item()):
        raise RuntimeError(f"device error bits {int(err.item())} in the prefill")
    unabs = run_unabsorbed(torch, mtla, glue, dev, mc, W, qr, cp, md, err, flush, timed_call=time_calls)
    train = run_train(torch, mtla, glue, dev, mc, W, qr, c, kR, cp, md, err, flush, P, W_c, b_c, J)
    ms_attn = ms - ms_merge
    # algorithmic work: every visible (query, head, column) pair, one score of
    # length D and one value row of length r, 2 flops per multiply-add
    pairs = B * d.H * sum(math.ceil(m / d.s) for m in range(1, T + 1))
    flops = pairs * (2 * d.D + 2 * d.r)
    _, tflops_peak, _, kind = measured_peaks()
    attn_tflops = flops / (ms_attn / 1e3) / 1e12
    return {"workload": "masked prefill bf16: B=8, T=4096, d=512, H=8, d_h=64, r=256, d_R=32, s=2",
            "ms": ms, "ms_running_merge": ms_merge, "ms_attention": ms_attn,
            "algorithmic_tflop": flops / 1e12, "call_tflops": flops / (ms / 1e3) / 1e12,
            "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": tflops_peak, "unit": "TFLOP/s",
                         "frac": attn_tflops / tflops_peak, "kernel": "mtla::ptc::prefill_tc_kernel",
                         "peak_kind": f"{kind} cuBLAS bf16 (burst)"},
            "note": "attention time = full call - cache-only call (the running merge alone); "
                    "L2 flushed before each call",
            "unabsorbed": unabs, "training": train}


def run_train(torch, mtla, glue, dev, mc, W, qr, c, kR, cp, md, err, flush, P, W_c, b_c, J):
    """One training step of the shortcut on the prefill workload (B=8, T=4096,
    s=2): the forward on the uncompressed RoPE keys and the backward chain
    attention -> key/value maps -> merge, each call timed alone."""
    d = mc.dims
    B, T = c.shape[0], c.shape[1]
    q = glue.query_heads(torch.from_numpy(mc.x).to(dev), W).to(torch.bfloat16).contiguous()
    W_kv = glue.kv_weights(W)
    k = torch.empty(B, T, d.H, d.d_h, dtype=torch.bfloat16, device=dev)
    v, out, dO, dq, dk, dv = (torch.empty_like(k) for _ in range(6))
    dO.normal_(generator=torch.Generator(device=dev).manual_seed(5))
    dqr = torch.empty_like(qr)
    lse = torch.empty(B, T, d.H, device=dev)
    dkR = torch.empty(B, T, d.d_R, device=dev)
    dC = torch.empty(B, T, d.r, device=dev)
    dc = torch.empty(B, T, d.r, device=dev)
    dW = torch.empty(d.r, d.D, device=dev)
    db = torch.empty(d.D, device=dev)
    dP = torch.empty(J, d.D, device=dev)
    mtla.mtla_prefill_kv(md, B, T, cp, W_kv, k, v, err)
    wa, wk, wm = (mtla.mtla_train_workspace_bytes(md, B, T, w)
                  for w in (mtla.TRAIN_ATTN_BWD, mtla.TRAIN_KV_BWD, mtla.TRAIN_MERGE_BWD))
    ws = torch.empty(max(wa, wk, wm), dtype=torch.uint8, device=dev)
    ms_fwd = time_calls(torch, lambda: mtla.mtla_train_attn_fwd(md, B, T, q, qr, k, v, kR, out, lse, err), 7, 3, flush)
    ms_bwd = time_calls(torch, lambda: mtla.mtla_train_attn_bwd(md, B, T, q, qr, k, v, kR, out, lse, dO, dq, dqr, dk, dv,
                                                               dkR, ws, wa, err), 7, 3, flush)
    ms_kv = time_calls(torch, lambda: mtla.mtla_train_kv_bwd(md, B, T, dk, dv, W_kv, dC, ws, wk, err), 7, 3, flush)
    ms_merge = time_calls(torch, lambda: mtla.mtla_train_merge_bwd(md, B, T, c, W_c, b_c, P, J, dC, dc, dW, db, dP, ws,
                                                                   wm, err), 7, 3, flush)
    if int(err.item()):
        raise RuntimeError(f"device error bits {int(err.item())} in the training step")
    hbm_peak, tflops_peak, _, kind = measured_peaks()
    pairs = B * d.H * sum(math.ceil(m / d.s) for m in range(1, T + 1))
    f_fwd = pairs * (2 * (d.d_h + d.d_R) + 2 * d.d_h)
    # backward per visible pair: score recompute 2 (d_h + d_R), dP 2 d_h, dv 2 d_h, [dk | dk^R] and
    # [dq | dq^R] 2 (d_h + d_R) each
    f_bwd = pairs * (3 * 2 * (d.d_h + d.d_R) + 2 * 2 * d.d_h)
    BT = B * T
    kv_bytes = 2 * BT * d.H * d.d_h * 2 + BT * d.r * 4 + W_kv.numel() * 2
    merge_bytes = BT * d.r * 2 + 2 * BT * d.r * 4  # c and dC read, dc written
    tf = lambda f, ms: f / (ms / 1e3) / 1e12
    gb = lambda by, ms: by / (ms / 1e3) / 1e9
    return {"workload": "training step of the shortcut (uncompressed K^R), B=8, T=4096, H=8, d_h=64, r=256, "
                        "d_R=32, s=2; d_out drawn N(0, 1)",
            "ms_forward": ms_fwd, "ms_attn_backward": ms_bwd, "ms_kv_backward": ms_kv, "ms_merge_backward": ms_merge,
            "ms_total": ms_fwd + ms_bwd + ms_kv + ms_merge,
            "attn_forward": {"algorithmic_tflop": f_fwd / 1e12, "tflops": tf(f_fwd, ms_fwd),
                             "frac": tf(f_fwd, ms_fwd) / tflops_peak},
            "roofline": {"bound": "tensor", "achieved": tf(f_bwd, ms_bwd), "peak": tflops_peak, "unit": "TFLOP/s",
                         "frac": tf(f_bwd, ms_bwd) / tflops_peak, "kernel": "mtla::bwt::dkv::bwd_dkv_tc_kernel + mtla::bwt::dq::bwd_dq_tc_kernel",
                         "algorithmic_tflop": f_bwd / 1e12, "peak_kind": f"{kind} cuBLAS bf16 (burst)"},
            "kv_backward": {"algorithmic_bytes": kv_bytes, "achieved_gbs": gb(kv_bytes, ms_kv),
                            "frac_hbm": gb(kv_bytes, ms_kv) / hbm_peak},
            "merge_backward": {"algorithmic_bytes": merge_bytes, "achieved_gbs": gb(merge_bytes, ms_merge),
                               "frac_hbm": gb(merge_bytes, ms_merge) / hbm_peak},
            "note": "each call alone, median of 7 after 3, L2 flushed before each; the backward's flops count "
                    "each product once (the kernels recompute the scores in both the dq and dk/dv passes)"}


def run_unabsorbed(torch, mtla, glue, dev, mc, W, qr, cp, md, err, flush, timed_call):
    """The same prefill in the un-absorbed form on the running merge's C_hat':
    mtla_prefill_kv (k, v = C_hat' W_K^h, C_hat' W_V^h) and
    mtla_prefill_unabsorbed_attn (d_h = 64 keys plus the d_R = 32 RoPE keys)."""
    d = mc.dims
    B, T = cp.shape[0], cp.shape[1]
    q = glue.query_heads(torch.from_numpy(mc.x).to(dev), W).to(torch.bfloat16).contiguous()
    W_kv = glue.kv_weights(W)
    k = torch.empty(B, T, d.H, d.d_h, dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    out = torch.empty_like(k)
    ms_kv = timed_call(torch, lambda: mtla.mtla_prefill_kv(md, B, T, cp, W_kv, k, v, err), 7, 3, flush)
    ms_at = timed_call(torch, lambda: mtla.mtla_prefill_unabsorbed_attn(md, B, T, q, qr, k, v, cp, out, err),
                       7, 3, flush)
    if int(err.item()):
        raise RuntimeError(f"device error bits {int(err.item())} in the un-absorbed prefill")
    hbm_peak, tflops_peak, _, kind = measured_peaks()
    pairs = B * d.H * sum(math.ceil(m / d.s) for m in range(1, T + 1))
    flops = pairs * (2 * (d.d_h + d.d_R) + 2 * d.d_h)
    kv_flops = 2 * B * T * d.r * 2 * d.H * d.d_h
    kv_bytes = B * T * (d.D * 2 + 2 * d.H * d.d_h * 2) + W_kv.numel() * 2
    at = flops / (ms_at / 1e3) / 1e12
    return {"ms_kv": ms_kv, "ms_attention": ms_at, "algorithmic_tflop": flops / 1e12,
            "kv": {"algorithmic_bytes": kv_bytes, "algorithmic_tflop": kv_flops / 1e12,
                   "achieved_gbs": kv_bytes / (ms_kv / 1e3) / 1e9,
                   "frac_hbm": kv_bytes / (ms_kv / 1e3) / 1e9 / hbm_peak},
            "roofline": {"bound": "tensor", "achieved": at, "peak": tflops_peak, "unit": "TFLOP/s",
                         "frac": at / tflops_peak, "kernel": "mtla::utc::prefill_unabs_tc_kernel",
                         "peak_kind": f"{kind} cuBLAS bf16 (burst)"},
            "note": "320 flop per visible (query, head, column): 2 (d_h + d_R) for the score, 2 d_h for the "
                    "value; median of 7 calls, L2 flushed before each"}


class DecodeState:
    """One decode workload resident on the device: a paged-contiguous cache
    with spare rows, lengths, queries and the merge inputs."""

    def __init__(self, torch, mtla, glue, dev, d, t_prev, cache_rows_dev, lin, q_abs, q_rope, c_new, kR_new,
                 spare_tokens):
        B = len(t_prev)
        self.B, self.d, self.mtla = B, d, mtla
        L = [synth.ceil_div(int(t), d.s) for t in t_prev]
        caps = [l + spare_tokens // d.s + 2 for l in L]
        offs = np.concatenate([[0], np.cumsum(caps)])[:-1]
        self.cache_rows = int(sum(caps))
        self.cache = torch.zeros(self.cache_rows, d.D, dtype=torch.bfloat16, device=dev)
        for b in range(B):
            self.cache[int(offs[b]):int(offs[b]) + L[b]] = cache_rows_dev(b)
        self.offset = torch.tensor(offs, dtype=torch.int64, device=dev)
        self.capacity = torch.tensor(caps, dtype=torch.int64, device=dev)
        self.t_host = np.asarray(t_prev, dtype=np.int64).copy()
        self.t = torch.tensor(t_prev, dtype=torch.int32, device=dev)
        self.cache_len = torch.zeros(B, dtype=torch.int32, device=dev)
        J = synth.ceil_div(int(max(t_prev)) + spare_tokens + 1, d.s) + 1
        bf = lambda a: (a if torch.is_tensor(a) else torch.from_numpy(np.ascontiguousarray(a, np.float32))).to(
            dev).to(torch.bfloat16).contiguous()
        self.q_abs, self.q_rope, c, k = bf(q_abs), bf(q_rope), bf(c_new), bf(kR_new)
        W_c, b_c = torch.from_numpy(lin["W_c"]).to(dev), torch.from_numpy(lin["b_c"]).to(dev)
        P = glue.pe_table(J, torch.from_numpy(lin["W_p"]).to(dev), torch.from_numpy(lin["b_p"]).to(dev))
        self.merge = {"c_new": c, "kR_new": k, "W_c": W_c, "b_c": b_c, "P": P, "J_max": J}
        self.md = mtla.dims(d.H, d.d_h, d.r, d.d_R, d.s, "bf16")
        self.ws_bytes = mtla.mtla_workspace_bytes(self.md, B)
        self.ws = torch.zeros(max(self.ws_bytes, 16), dtype=torch.uint8, device=dev)
        self.out = torch.empty(B, d.H, d.r, dtype=torch.float32, device=dev)
        self.lse = torch.empty(B, d.H, dtype=torch.float32, device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)

    def call(self):
        self.mtla.mtla_decode_attn(self.md, self.B, self.q_abs, self.q_rope, self.merge, self.cache,
                                   self.cache_rows, self.d.D, self.offset, self.capacity, self.t, self.cache_len,
                                   self.out, self.lse, self.ws, self.ws_bytes, self.err)
        self.t_host += 1


def time_decode_calls(torch, state: DecodeState, n: int, warm: int, flush):
    """Median time of single decode calls (merge + attention + combine) with
    L2 flushed before each: the flush also keeps the GPU busy while the call is
    launched, so the events bracket the call's own kernels.  Each call really
    advances the state; its algorithmic bytes come from its lengths."""
    for _ in range(warm):
        state.call()
    torch.cuda.synchronize()
    times, nbytes = [], []
    for _ in range(n):
        flush.zero_()
        torch.cuda._sleep(100_000)  # the GPU stays busy while the host launches the call
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        state.call()
        e1.record()
        nbytes.append(decode_step_bytes(state.t_host, state.d))
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    if int(state.err.item()):
        raise RuntimeError(f"device error bits {int(state.err.item())}")
    ms = statistics.median(times)
    by = statistics.median(nbytes)
    hbm_peak, _, _, kind = measured_peaks()
    gbs = by / (ms / 1e3) / 1e9
    return {"ms_per_step": ms, "value": state.B / (ms / 1e3), "unit": UNIT, "algorithmic_bytes_per_step": by,
            "achieved_gbs": gbs, "frac": gbs / hbm_peak, "peak_gbs": hbm_peak, "peak_kind": kind,
            "roofline_ms": by / (hbm_peak * 1e9) * 1e3, "calls": n}


def run_configs(torch, mtla, glue, dev, which=("ragged", "sweep", "layer", "multi")):
    """The other decode workloads, one call at a time (L2 flushed before each):
    ragged B=128 (processed lengths uniform in [512, 8192], seed 1) and the
    compression-ratio sweep B=64, T=16384, s in {1, 2, 3, 4, 8}, whose caches
    are built on the device by the library's cache-only prefill from latents
    and RoPE keys drawn on the device (torch generator seeded 4 + s; the merge
    Linears are the shared generator's draws for that seed)."""
    import dataclasses
    n, warm = 20, 3
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    res = {"timing": f"median of {n} single calls after {warm}, CUDA events, L2 flushed before each call and a "
                     "device sleep covering the host's launch"}
    if "layer" in which:
        res["layer_maps_b32"] = run_layer_maps(torch, mtla, glue, dev, flush, n, warm)
    if "multi" in which:
        res["multi_token_b32_n4"] = run_multi(torch, mtla, glue, dev, flush, n, warm)
    if "ragged" in which:
        res["ragged_b128"] = run_ragged(torch, mtla, glue, dev, flush, n, warm)
    if "sweep" in which:
        res["sweep_b64_t16384"] = run_sweep(torch, mtla, glue, dev, flush, n, warm)
    return res


def run_ragged(torch, mtla, glue, dev, flush, n, warm):
    case = synth.decode_ragged()
    d = case.dims
    rows_dev = lambda b: torch.from_numpy(case.rows[b]).to(dev).to(torch.bfloat16)
    st = DecodeState(torch, mtla, glue, dev, d, case.t_prev, rows_dev, case.lin, case.q_abs, case.q_rope,
                     case.c_new, case.kR_new, n + warm + 2)
    r = time_decode_calls(torch, st, n, warm, flush)
    r["workload"] = ("ragged decode bf16: B=128, H=8, d_h=64, r=256, d_R=32, s=2, processed lengths uniform in "
                     f"[512, 8192] (seed 1), {int(sum(len(x) for x in case.rows))} cache rows before the calls")
    return r


def run_sweep(torch, mtla, glue, dev, flush, n, warm):
    import dataclasses
    sweep = {}
    B, T = 64, 16384
    for s in (1, 2, 3, 4, 8):
        d = dataclasses.replace(synth.MAIN, s=s)
        lin = synth.merge_linears(synth.rng_for(4 + s), d)
        g = torch.Generator(device=dev)
        g.manual_seed(4 + s)
        c = torch.randn(B, T, d.r, generator=g, device=dev).to(torch.bfloat16)
        kR = torch.randn(B, T, d.d_R, generator=g, device=dev).to(torch.bfloat16)
        L = synth.ceil_div(T, s)
        J = synth.ceil_div(T + n + warm + 4, s) + 1
        P = glue.pe_table(J, torch.from_numpy(lin["W_p"]).to(dev), torch.from_numpy(lin["b_p"]).to(dev))
        cp = torch.empty(B, T, d.D, dtype=torch.bfloat16, device=dev)
        built = torch.empty(B, L, d.D, dtype=torch.bfloat16, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        mtla.mtla_prefill_masked_attn(mtla.dims(d.H, d.d_h, d.r, d.d_R, s, "bf16"), B, T, None, None, c, kR,
                                      torch.from_numpy(lin["W_c"]).to(dev), torch.from_numpy(lin["b_c"]).to(dev),
                                      P, J, cp, built, None, err)
        torch.cuda.synchronize()
        if int(err.item()):
            raise RuntimeError(f"device error bits {int(err.item())} building the s={s} cache")
        del cp, c, kR
        qa, qr, cn, kn = synth.sweep_step(s, B=B)
        st = DecodeState(torch, mtla, glue, dev, d, [T] * B, lambda b: built[b], lin, qa, qr, cn, kn,
                         n + warm + 2)
        del built
        r = time_decode_calls(torch, st, n, warm, flush)
        r["rows_per_sequence_before"] = L
        sweep[f"s={s}"] = r
        del st
        torch.cuda.empty_cache()
    return {"workload": "compression-ratio sweep bf16: B=64, t=16384 processed tokens, H=8, d_h=64, r=256, "
                        "d_R=32; cache merged from N(0,1) latents with the sigmoid gates", **sweep}


def time_calls(torch, call, n, warm, flush):
    """Median of n single calls (after warm ones), L2 flushed before each."""
    for _ in range(warm):
        call()
    torch.cuda.synchronize()
    times = []
    for _ in range(n):
        flush.zero_()
        torch.cuda._sleep(100_000)  # the GPU stays busy while the host launches the call
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def run_layer_maps(torch, mtla, glue, dev, flush, n, warm):
    """The absorbed input and output maps of the decode layer at B=32, d=512
    (mtla_project_in: x -> q_abs, q_rope, c_t, k^R_t with RoPE; mtla_project_out:
    o -> y): bound by streaming their bf16 weights."""
    mc = synth.model_case(synth.MAIN, B=32, T=1, d=512, seed=7, dtype="bf16")
    d = mc.dims
    B, dm = 32, mc.d
    W = {k: torch.from_numpy(v).to(dev) for k, v in mc.W.items()}
    W_in, W_out = glue.absorbed_weights(W, torch.bfloat16)
    md = mtla.dims(d.H, d.d_h, d.r, d.d_R, d.s, "bf16")
    x = torch.from_numpy(mc.x[:, 0, :]).to(dev).to(torch.bfloat16)
    pos = torch.arange(B, dtype=torch.int32, device=dev) * 97
    qa = torch.empty(B, d.H, d.r, dtype=torch.bfloat16, device=dev)
    qr = torch.empty(B, d.H, d.d_R, dtype=torch.bfloat16, device=dev)
    cn = torch.empty(B, d.r, dtype=torch.bfloat16, device=dev)
    kn = torch.empty(B, d.d_R, dtype=torch.bfloat16, device=dev)
    o = torch.randn(B, d.H, d.r, device=dev)
    y = torch.empty(B, dm, dtype=torch.float32, device=dev)
    wi = mtla.mtla_project_workspace_bytes(md, B, dm, mtla.PROJ_IN)
    wo = mtla.mtla_project_workspace_bytes(md, B, dm, mtla.PROJ_OUT)
    ws_i = torch.empty(wi, dtype=torch.uint8, device=dev)
    ws_o = torch.empty(wo, dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ms_in = time_calls(torch, lambda: mtla.mtla_project_in(md, B, dm, x, W_in, pos, qa, qr, cn, kn, ws_i, wi, err),
                       n, warm, flush)
    ms_out = time_calls(torch, lambda: mtla.mtla_project_out(md, B, dm, o, W_out, y, ws_o, wo, err), n, warm, flush)
    if int(err.item()):
        raise RuntimeError(f"device error bits {int(err.item())} in the layer maps")
    hbm_peak, _, _, kind = measured_peaks()
    b_in = W_in.numel() * 2 + x.numel() * 2 + B * (d.H * d.D + d.D) * 2
    b_out = W_out.numel() * 2 + o.numel() * 4 + y.numel() * 4
    row = lambda ms, by: {"ms": ms, "algorithmic_bytes": by, "achieved_gbs": by / (ms / 1e3) / 1e9,
                          "frac": by / (ms / 1e3) / 1e9 / hbm_peak}
    return {"workload": "absorbed layer maps bf16, B=32 tokens, d=512, H=8, r=256, d_R=32 "
                        f"(W_in {tuple(W_in.shape)}, W_out {tuple(W_out.shape)})",
            "project_in": row(ms_in, b_in), "project_out": row(ms_out, b_out), "peak_gbs": hbm_peak,
            "peak_kind": kind, "bound": "hbm (weights streamed once per call)"}


def run_multi(torch, mtla, glue, dev, flush, n_calls, warm):
    """Four new tokens per sequence in one call on the B=32 workload
    (mtla_decode_attn_multi): 128 queries over the shared rows."""
    case = synth.decode_uniform(B=32, seed=2)
    d = case.dims
    B, n = case.B, 4
    rng = np.random.default_rng(11)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(synth.cast(a, "bf16"))).to(dev).to(torch.bfloat16)
    qa = bf(rng.standard_normal((B, n, d.H, d.r)))
    qr = bf(rng.standard_normal((B, n, d.H, d.d_R)))
    cn = bf(rng.standard_normal((B, n, d.r)))
    kn = bf(rng.standard_normal((B, n, d.d_R)))
    calls = warm + n_calls
    st = DecodeState(torch, mtla, glue, dev, d, case.t_prev,
                     lambda b: torch.from_numpy(case.rows[b]).to(dev).to(torch.bfloat16), case.lin, qa[:, 0],
                     qr[:, 0], cn[:, 0], kn[:, 0], calls * n + 4)
    ws_bytes = mtla.mtla_decode_multi_workspace_bytes(st.md, B, n)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    out = torch.empty(B, n, d.H, d.r, dtype=torch.float32, device=dev)
    merge = dict(st.merge, c_new=cn, kR_new=kn)
    nbytes = []

    def call():
        mtla.mtla_decode_attn_multi(st.md, B, n, qa, qr, merge, st.cache, st.cache_rows, d.D, st.offset,
                                    st.capacity, st.t, st.cache_len, out, None, ws, ws_bytes, st.err)
        st.t_host += n
        # unique bytes: every row once, the queries, the new tokens, out
        rows = int(sum(synth.ceil_div(int(t), d.s) for t in st.t_host))
        nbytes.append(rows * ROW_BYTES + B * n * (d.H * d.D * 2 + d.D * 2 + d.H * d.r * 4) + B * ROW_BYTES)

    ms = time_calls(torch, call, n_calls, warm, flush)
    if int(st.err.item()):
        raise RuntimeError(f"device error bits {int(st.err.item())} in the multi-token decode")
    hbm_peak, _, _, kind = measured_peaks()
    by = statistics.median(nbytes)
    return {"workload": "B=32 decode workload (4096 / 4095 processed tokens, s=2) with n=4 new tokens per "
                        "sequence in one call", "ms_per_call": ms, "value": B * n / (ms / 1e3), "unit": UNIT,
            "unique_bytes_per_call": by, "achieved_gbs": by / (ms / 1e3) / 1e9,
            "frac": by / (ms / 1e3) / 1e9 / hbm_peak, "peak_kind": kind,
            "note": "query-steps/s counts the B n queries; bytes count every cache row once"}


# ---------------------------------------------------------------------------
# the oracle on the host cores (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------
# Worker processes are started with "spawn" (never forked from a process that
# may hold a CUDA context) and read the B=32 workload from one shared-memory
# block; each runs numpy with one BLAS thread, so the core count is the number
# of worker processes.
_WK = {}


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover - non-Linux
        return os.cpu_count() or 1


def _oracle_inputs():
    """The B=32 decode workload and its P table, as the oracle sees them."""
    import oracle
    case = synth.decode_uniform(B=32, seed=2)
    d = case.dims
    P = oracle.pe_table(synth.ceil_div(int(case.t_prev.max()) + 1, d.s) + 1, case.lin["W_p"], case.lin["b_p"])
    arrays = {"rows": np.concatenate(case.rows).astype(np.float32), "q_abs": case.q_abs, "q_rope": case.q_rope,
              "c_new": case.c_new, "kR_new": case.kR_new, "W_c": case.lin["W_c"], "b_c": case.lin["b_c"],
              "P": P.astype(np.float64)}
    lens = [len(r) for r in case.rows]
    return case, arrays, lens


def _worker_init(shm_name, layout, lens, t_prev, dims):
    from multiprocessing import shared_memory

    from threadpoolctl import threadpool_limits
    threadpool_limits(limits=1)
    # spawned children share the parent's resource tracker: attaching registers
    # the same name again, and the parent's unlink is the one that counts
    shm = shared_memory.SharedMemory(name=shm_name)
    a = {k: np.ndarray(shape, dtype=np.dtype(dt), buffer=shm.buf, offset=off) for k, (off, shape, dt) in
         layout.items()}
    starts = np.concatenate([[0], np.cumsum(lens)])
    _WK.update(shm=shm, a=a, rows=[a["rows"][starts[b]:starts[b + 1]] for b in range(len(lens))],
               t_prev=t_prev, dims=dims)


def _worker_seq(b):
    """The oracle's decode step (merge + attention) of sequence b."""
    import oracle
    a, (H, d_h, r, d_R, s) = _WK["a"], _WK["dims"]
    oracle.decode_step(_WK["rows"][b], int(_WK["t_prev"][b]), s, a["c_new"][b], a["kR_new"][b], a["q_abs"][b],
                       a["q_rope"][b], a["W_c"], a["b_c"], a["P"], d_h)
    return b


def _worker_loop(k, n, seconds):
    """Sequences k, k + n, ... (cyclically) for `seconds`: (steps done, seconds taken)."""
    B = len(_WK["rows"])
    done, b = 0, k % B
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        _worker_seq(b)
        done += 1
        b = (b + n) % B
    return done, time.perf_counter() - t0


class OraclePool:
    """A pool of spawned oracle workers over the shared B=32 workload."""

    def __init__(self, workers: int):
        import multiprocessing as mp
        from multiprocessing import shared_memory
        case, arrays, lens = _oracle_inputs()
        self.case = case
        layout, off = {}, 0
        for k, v in arrays.items():
            v = np.ascontiguousarray(v)
            layout[k] = (off, v.shape, v.dtype.str)
            off += (v.nbytes + 63) // 64 * 64
        self.shm = shared_memory.SharedMemory(create=True, size=max(off, 64))
        for k, v in arrays.items():
            o, shape, dt = layout[k]
            np.ndarray(shape, dtype=np.dtype(dt), buffer=self.shm.buf, offset=o)[...] = v
        d = case.dims
        env_keys = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
        saved = {k: os.environ.get(k) for k in env_keys}
        os.environ.update({k: "1" for k in env_keys})
        try:
            self.pool = mp.get_context("spawn").Pool(
                workers, initializer=_worker_init,
                initargs=(self.shm.name, layout, lens, case.t_prev, (d.H, d.d_h, d.r, d.d_R, d.s)))
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        self.workers = workers
        # every worker imported numpy and attached the block before timing starts
        self.pool.map(_worker_seq, [b % case.B for b in range(workers)], chunksize=1)

    def close(self):
        self.pool.close()
        self.pool.join()
        self.shm.close()
        self.shm.unlink()


def cpu_baseline(seconds: float):
    """The oracle as it stands on the host: one worker (one thread) for
    `seconds`, then every host core for `seconds`, each cycling over the
    32 sequences of the B=32 decode step (merge + attention per sequence)."""
    cores = host_cores()
    one = OraclePool(1)
    try:
        n1, el1 = one.pool.apply(_worker_loop, (0, 1, seconds))
    finally:
        one.close()
    allp = OraclePool(cores)
    try:
        res = allp.pool.starmap(_worker_loop, [(k, cores, seconds) for k in range(cores)], chunksize=1)
    finally:
        allp.close()
    n_all = sum(r[0] for r in res)
    el_all = max(r[1] for r in res)
    return {"value": n_all / el_all, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n_all} sequence-steps of the B=32 decode workload (merge + attention over 2048/2049 rows "
                      f"per sequence, cycling over the 32 sequences) by {cores} worker processes with one "
                      f"numpy float64 thread each, {el_all:.1f} s; host cores (sched_getaffinity): {cores}",
            "single_thread": {"value": n1 / el1, "unit": UNIT, "cores": 1,
                              "sample": f"{n1} sequence-steps in {el1:.1f} s, one worker, one thread"}}


def run_reference(args, rank, world):
    """The oracle, as it stands, on the host cores: a step is the whole B=32
    decode step (every sequence's merge and attention), its 32 sequences spread
    over min(host cores, 32) worker processes; W untimed steps, then K timed."""
    if rank != 0:
        return None
    W, K = args.warmup, args.steps
    cores = host_cores()
    workers = min(cores, 32)
    pool = OraclePool(workers)
    B = pool.case.B
    try:
        for _ in range(W):
            pool.pool.map(_worker_seq, range(B), chunksize=1)
        t0 = time.perf_counter()
        for _ in range(K):
            pool.pool.map(_worker_seq, range(B), chunksize=1)
        el = time.perf_counter() - t0
    finally:
        pool.close()
    value = B * K / el
    cb = {"value": value, "unit": UNIT, "cores": workers, "kind": "oracle",
          "sample": f"{K} timed steps of the whole B=32 decode workload (merge + attention of all 32 sequences, "
                    f"2048/2049 rows each) over {workers} worker processes, numpy float64, one thread each, "
                    f"{el:.1f} s; host cores: {cores}"}
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": el / K * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1))",
            "config": {"workload": WORKLOAD, "B_per_gpu": B, "step": "the whole B=32 step on the host cores"},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=500)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the ragged and s-sweep decode workloads")
    ap.add_argument("--configs", default="ragged,sweep,layer,multi",
                    help="which extra workloads to time (comma-separated: ragged, sweep, layer, multi)")
    ap.add_argument("--cpu-baseline", dest="cpu_baseline", action="store_true", default=True)
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-seconds", type=float, default=8.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        res = run_ours(args, rank, world, local_rank)
    if res is not None:
        print(json.dumps(res))


if __name__ == "__main__":
    main()
