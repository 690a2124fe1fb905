"""The layer around the MTLA hot path, in plain torch (fp32), on the device.

This is the model side that produces the hot path's inputs from a layer
input x: the latent projection, the absorbed query, the decoupled RoPE
query/key and the table P of Linear(pe_j).  It is not part of the hot path
and the C ABI never calls it; tests and the benchmark use it to build inputs
for the workloads that start from x.

Forms (the pages name these maps but do not spell them out):
  c = x W_down;  q_abs_h = (x W_Q^h) (W_K^h)^T  (MTLA paper notes, "Overall
  framework" and the decoupled-RoPE formula: W_K is absorbed into the query);
  q^R_h = RoPE(x W_QR^h), k^R = RoPE(x W_KR) with the RoFormer rotation of
  channel pairs (2k, 2k+1) by pos * 10000^(-2k/d_R), pos = t - 1;
  P[j-1] = pe_j W_p + b_p with the Transformer sinusoid pe of width D at
  position j - 1 (pe_j indexed by the merged group j).
"""
from __future__ import annotations

import torch


def sinusoid(J: int, D: int, device) -> torch.Tensor:
    pos = torch.arange(J, dtype=torch.float64, device=device)[:, None]
    k = torch.arange(D // 2, dtype=torch.float64, device=device)[None, :]
    ang = pos / torch.pow(torch.tensor(10000.0, dtype=torch.float64, device=device), 2.0 * k / D)
    pe = torch.empty(J, D, dtype=torch.float64, device=device)
    pe[:, 0::2] = torch.sin(ang)
    pe[:, 1::2] = torch.cos(ang)
    return pe


def pe_table(J: int, W_p: torch.Tensor, b_p: torch.Tensor) -> torch.Tensor:
    """P [J, D] fp32: row j-1 = Linear(pe_j)."""
    D = W_p.shape[0]
    pe = sinusoid(J, D, W_p.device).to(torch.float32)
    return (pe @ W_p.to(torch.float32) + b_p.to(torch.float32)).contiguous()


def rope(v: torch.Tensor, pos: torch.Tensor) -> torch.Tensor:
    """Rotate channel pairs of v [..., T, d_R] by pos[T] * 10000^(-2k/d_R)."""
    d_R = v.shape[-1]
    k = torch.arange(d_R // 2, dtype=torch.float64, device=v.device)
    theta = torch.pow(torch.tensor(10000.0, dtype=torch.float64, device=v.device), -2.0 * k / d_R)
    ang = (pos.to(torch.float64)[:, None] * theta[None, :]).to(torch.float32)
    cos, sin = torch.cos(ang), torch.sin(ang)
    x0, x1 = v[..., 0::2], v[..., 1::2]
    out = torch.empty_like(v)
    out[..., 0::2] = x0 * cos - x1 * sin
    out[..., 1::2] = x0 * sin + x1 * cos
    return out


def project(x: torch.Tensor, W: dict):
    """x [B, T, d] -> q_abs [B,T,H,r], q_rope [B,T,H,d_R], c [B,T,r], kR [B,T,d_R], all fp32."""
    x = x.to(torch.float32)
    B, T, d = x.shape
    W_Q, W_K, W_QR = W["W_Q"], W["W_K"], W["W_QR"]
    H, r, d_h = W_K.shape
    d_R = W_QR.shape[2]
    pos = torch.arange(T, device=x.device)
    c = x @ W["W_down"]
    kR = rope(x @ W["W_KR"], pos)
    q = (x @ W_Q.reshape(d, H * d_h)).reshape(B, T, H, d_h)
    q_abs = torch.einsum("bthe,hre->bthr", q, W_K)
    qR = (x @ W_QR.reshape(d, H * d_R)).reshape(B, T, H, d_R)
    q_rope = rope(qR.permute(0, 2, 1, 3), pos).permute(0, 2, 1, 3)
    return q_abs.contiguous(), q_rope.contiguous(), c.contiguous(), kR.contiguous()


def absorbed_weights(W: dict, dtype=torch.bfloat16):
    """The weight matrices of mtla_project_in / mtla_project_out (row-major,
    one row per output feature), from the layer's maps W_Q [d,H,d_h],
    W_K [H,r,d_h], W_V [H,r,d_h], W_O [H*d_h,d], W_down [d,r], W_QR [d,H,d_R],
    W_KR [d,d_R]:
      W_in  [H r + H d_R + r + d_R, d]: rows of (W_Q^h W_K^h^T)^T per head,
            W_QR^h^T per head, W_down^T, W_KR^T;
      W_out [d, H r]: column block h is (W_V^h W_O^h)^T.
    The products are formed in float64 and rounded once to `dtype`."""
    f = lambda t: t.to(torch.float64)
    W_Q, W_K, W_V, W_O = f(W["W_Q"]), f(W["W_K"]), f(W["W_V"]), f(W["W_O"])
    H, r, d_h = W_K.shape
    rows = [(W_Q[:, h, :] @ W_K[h].T).T for h in range(H)]
    rows += [f(W["W_QR"])[:, h, :].T for h in range(H)]
    rows += [f(W["W_down"]).T, f(W["W_KR"]).T]
    W_in = torch.cat(rows, dim=0)
    W_out = torch.cat([(W_V[h] @ W_O[h * d_h:(h + 1) * d_h, :]).T for h in range(H)], dim=1)
    return W_in.to(dtype).contiguous(), W_out.to(dtype).contiguous()


def query_heads(x: torch.Tensor, W: dict) -> torch.Tensor:
    """q_h = x W_Q^h for the un-absorbed forward: x [B, T, d] -> [B, T, H, d_h] (fp32)."""
    W_Q = W["W_Q"].to(torch.float32)
    d, H, d_h = W_Q.shape
    return (x.to(torch.float32) @ W_Q.reshape(d, H * d_h)).reshape(*x.shape[:-1], H, d_h).contiguous()


def kv_weights(W: dict, dtype=torch.bfloat16) -> torch.Tensor:
    """W_kv [2 H d_h, r] of mtla_prefill_kv: row h d_h + e is column e of
    W_K^h, row H d_h + h d_h + e is column e of W_V^h."""
    W_K, W_V = W["W_K"], W["W_V"]
    H, r, d_h = W_K.shape
    rows = [W_K[h].T for h in range(H)] + [W_V[h].T for h in range(H)]
    return torch.cat(rows, dim=0).to(dtype).contiguous()
