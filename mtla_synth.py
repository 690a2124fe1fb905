"""Seeded synthetic inputs for the MTLA hot path.

This module only draws random numbers, rounds them to the storage dtype and
lays them out; it holds none of the method's arithmetic (no merge, no gate, no
attention, no projection).  Both the fp64 oracle (through the tests) and the
CUDA path (through the tests and the benchmark) take their inputs from here,
so the two sides see bit-identical values.

Generator: numpy's PCG64 (``numpy.random.Generator(PCG64(seed))``), normal
draws with ``standard_normal`` in float64, then cast to the storage dtype:
float32, or bfloat16 by round-to-nearest-even of the float32 value.  bfloat16
values are returned as float32 arrays that hold exactly representable bf16
numbers, so ``torch.from_numpy(a).to(torch.bfloat16)`` is exact and the oracle
widens the same numbers to float64.

Workload shapes follow the MTLA notation: B sequences, H heads, head width
d_h, latent width r, decoupled-RoPE width d_R, temporal stride s, cache row
width D = r + d_R (row = [c_hat | k_hat^R]).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


# --------------------------------------------------------------------------
# dtype helpers (rounding only)
# --------------------------------------------------------------------------

def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even); return float32 holding it."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) >> 16
    out = (u.astype(np.uint32) << 16).view(np.float32)
    return out.reshape(f.shape)


def cast(a: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32)
    if dtype == "bf16":
        return round_to_bf16(a)
    raise ValueError(f"unknown dtype {dtype!r}")


def normal(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float64) * scale


def rng_for(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


# --------------------------------------------------------------------------
# problem dimensions
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Dims:
    H: int
    d_h: int
    r: int
    d_R: int
    s: int

    @property
    def D(self) -> int:
        return self.r + self.d_R


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


# --------------------------------------------------------------------------
# merge hyper-network parameters (the two Linears), all ~ N(0,1)/sqrt(fan_in)
# --------------------------------------------------------------------------

def merge_linears(rng: np.random.Generator, dims: Dims):
    """W_c [r, D], b_c [D] (input c, fan_in r); W_p [D, D], b_p [D] (input pe, fan_in D).

    Returned as float32 (the library takes the merge Linears in float32)."""
    r, D = dims.r, dims.D
    W_c = normal(rng, (r, D), 1.0 / math.sqrt(r)).astype(np.float32)
    b_c = normal(rng, (D,), 1.0 / math.sqrt(r)).astype(np.float32)
    W_p = normal(rng, (D, D), 1.0 / math.sqrt(D)).astype(np.float32)
    b_p = normal(rng, (D,), 1.0 / math.sqrt(D)).astype(np.float32)
    return {"W_c": W_c, "b_c": b_c, "W_p": W_p, "b_p": b_p}


# --------------------------------------------------------------------------
# decode-step workloads
# --------------------------------------------------------------------------

@dataclasses.dataclass
class DecodeCase:
    """One decode step for B sequences.

    rows[b]   : [L_prev_b, D] cache rows of sequence b before the step
    t_prev[b] : tokens processed before the step (cache holds ceil(t_prev/s) rows)
    q_abs     : [B, H, r] absorbed queries; q_rope: [B, H, d_R]
    c_new     : [B, r] new latents; kR_new: [B, d_R] new rotated RoPE keys
    lin       : merge Linears (W_c, b_c, W_p, b_p), float32
    """
    dims: Dims
    dtype: str
    t_prev: np.ndarray
    rows: list
    q_abs: np.ndarray
    q_rope: np.ndarray
    c_new: np.ndarray
    kR_new: np.ndarray
    lin: dict

    @property
    def B(self) -> int:
        return len(self.t_prev)


def decode_case(dims: Dims, t_prev, seed: int, dtype: str = "bf16") -> DecodeCase:
    """Cache rows, queries and the new token all ~ N(0,1) (decode-step workloads).

    Draw order: merge Linears, then per sequence its cache rows, then q_abs,
    q_rope, c_new, kR_new."""
    rng = rng_for(seed)
    t_prev = np.asarray(t_prev, dtype=np.int64)
    B = len(t_prev)
    lin = merge_linears(rng, dims)
    rows = []
    for b in range(B):
        L = ceil_div(int(t_prev[b]), dims.s)
        rows.append(cast(normal(rng, (L, dims.D)), dtype))
    q_abs = cast(normal(rng, (B, dims.H, dims.r)), dtype)
    q_rope = cast(normal(rng, (B, dims.H, dims.d_R)), dtype)
    c_new = cast(normal(rng, (B, dims.r)), dtype)
    kR_new = cast(normal(rng, (B, dims.d_R)), dtype)
    return DecodeCase(dims, dtype, t_prev, rows, q_abs, q_rope, c_new, kR_new, lin)


def uniform_lengths(B: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """Per-sequence processed lengths, uniform integers in [lo, hi]."""
    rng = rng_for(seed)
    return rng.integers(lo, hi + 1, size=B, dtype=np.int64)


# --------------------------------------------------------------------------
# token-sequence workloads (prefill / cache building)
# --------------------------------------------------------------------------

@dataclasses.dataclass
class TokenCase:
    """B sequences of T tokens given directly as hot-path inputs.

    c [B,T,r], kR [B,T,d_R] (rotated), q_abs [B,T,H,r], q_rope [B,T,H,d_R]."""
    dims: Dims
    dtype: str
    c: np.ndarray
    kR: np.ndarray
    q_abs: np.ndarray
    q_rope: np.ndarray
    lin: dict


def token_case(dims: Dims, B: int, T: int, seed: int, dtype: str = "bf16",
               with_queries: bool = True) -> TokenCase:
    """Latents, RoPE keys (and queries) ~ N(0,1).  Draw order: Linears, c, kR, q_abs, q_rope."""
    rng = rng_for(seed)
    lin = merge_linears(rng, dims)
    c = cast(normal(rng, (B, T, dims.r)), dtype)
    kR = cast(normal(rng, (B, T, dims.d_R)), dtype)
    if with_queries:
        q_abs = cast(normal(rng, (B, T, dims.H, dims.r)), dtype)
        q_rope = cast(normal(rng, (B, T, dims.H, dims.d_R)), dtype)
    else:
        q_abs = q_rope = None
    return TokenCase(dims, dtype, c, kR, q_abs, q_rope, lin)


@dataclasses.dataclass
class ModelCase:
    """Attention-layer input x [B,T,d] and every weight of one MTLA layer.

    W_Q [d, H, d_h], W_K [H, r, d_h], W_V [H, r, d_h], W_O [H*d_h, d],
    W_down [d, r], W_QR [d, H, d_R], W_KR [d, d_R], plus the merge Linears.
    All weights ~ N(0,1)/sqrt(fan_in)."""
    dims: Dims
    d: int
    x: np.ndarray
    W: dict
    lin: dict


def model_case(dims: Dims, B: int, T: int, d: int, seed: int, dtype: str) -> ModelCase:
    """Draw order: x, W_Q, W_K, W_V, W_O, W_down, W_QR, W_KR, then the merge Linears."""
    rng = rng_for(seed)
    H, d_h, r, d_R = dims.H, dims.d_h, dims.r, dims.d_R
    x = cast(normal(rng, (B, T, d)), dtype)
    W = {
        "W_Q": normal(rng, (d, H, d_h), 1.0 / math.sqrt(d)),
        "W_K": normal(rng, (H, r, d_h), 1.0 / math.sqrt(r)),
        "W_V": normal(rng, (H, r, d_h), 1.0 / math.sqrt(r)),
        "W_O": normal(rng, (H * d_h, d), 1.0 / math.sqrt(H * d_h)),
        "W_down": normal(rng, (d, r), 1.0 / math.sqrt(d)),
        "W_QR": normal(rng, (d, H, d_R), 1.0 / math.sqrt(d)),
        "W_KR": normal(rng, (d, d_R), 1.0 / math.sqrt(d)),
    }
    W = {k: v.astype(np.float32) for k, v in W.items()}
    lin = merge_linears(rng, dims)
    return ModelCase(dims, d, x, W, lin)


# --------------------------------------------------------------------------
# the named workloads
# --------------------------------------------------------------------------

TINY = Dims(H=4, d_h=16, r=64, d_R=8, s=2)          # tiny fp32 end-to-end check
MAIN = Dims(H=8, d_h=64, r=256, d_R=32, s=2)        # decode / prefill bf16 workloads


def tiny_e2e(seed: int = 0) -> ModelCase:
    """Tiny fp32 end-to-end: B=1, prompt T=64 then 16 decode steps (80 tokens), d = H*d_h."""
    return model_case(TINY, B=1, T=80, d=TINY.H * TINY.d_h, seed=seed, dtype="f32")


def decode_uniform(B: int = 32, seed: int = 2) -> DecodeCase:
    """Decode step bf16, B=32: even sequences have 4096 processed tokens (2048 full
    rows, the new token opens row 2049), odd ones 4095 (row 2048 is partial and the
    new token completes it in place)."""
    t_prev = np.array([4096 if b % 2 == 0 else 4095 for b in range(B)], dtype=np.int64)
    return decode_case(MAIN, t_prev, seed, "bf16")


def decode_ragged(B: int = 128, seed: int = 1) -> DecodeCase:
    """Ragged decode bf16: processed lengths uniform in [512, 8192]."""
    t_prev = uniform_lengths(B, 512, 8192, seed)
    return decode_case(MAIN, t_prev, seed + 1000, "bf16")


def sweep_tokens(s: int, B: int = 64, T: int = 16384, seed_base: int = 4) -> TokenCase:
    """Compression-ratio sweep: B sequences of T merged tokens at stride s."""
    dims = dataclasses.replace(MAIN, s=s)
    return token_case(dims, B, T, seed_base + s, "bf16", with_queries=False)


def sweep_step(s: int, B: int = 64, seed_base: int = 4):
    """The decode step after the sweep's T tokens: queries and the new token ~ N(0,1)."""
    rng = rng_for(10_000 + seed_base + s)
    dims = dataclasses.replace(MAIN, s=s)
    q_abs = cast(normal(rng, (B, dims.H, dims.r)), "bf16")
    q_rope = cast(normal(rng, (B, dims.H, dims.d_R)), "bf16")
    c_new = cast(normal(rng, (B, dims.r)), "bf16")
    kR_new = cast(normal(rng, (B, dims.d_R)), "bf16")
    return q_abs, q_rope, c_new, kR_new


def prefill_model(B: int = 8, T: int = 4096, seed: int = 5) -> ModelCase:
    """Stride-aware masked prefill bf16: B=8, T=4096, d=512, x ~ N(0,1)."""
    return model_case(MAIN, B=B, T=T, d=512, seed=seed, dtype="bf16")
