"""Plain float64 restatement of MTLA's hot path — test infrastructure only.

Notation (1-indexed in time, as on the pages): a sequence has tokens
t = 1..T; token t carries a latent c_t (width r) and a rotated RoPE key
k^R_t (width d_R); the temporal stride is s; group j(t) = ceil(t/s); a cache
row is [c_hat_j | k_hat^R_j] of width D = r + d_R.

Every function cites the passage it follows (page title + section, see the
package docstring).  No blocking, no fusion, no reordering beyond the
definition: a reader should be able to check each line against the pages.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "group_index", "cache_length", "opens_new_row", "stride_visible",
    "visible_columns", "stride_mask", "sigmoid", "sinusoidal_pe", "pe_table",
    "merge_weight", "merge_step", "decode_attention", "decode_step",
    "decode_loop", "partial_merge_sequence", "compressed_cache",
    "masked_forward", "masked_forward_query", "rope", "project_inputs",
    "absorbed_output", "unabsorbed_forward", "unabsorbed_heads", "cache_elements_per_token",
    "latent_partial_merge", "shortcut_attention", "shortcut_attention_backward", "kv_backward",
    "latent_merge_backward",
]


# ---------------------------------------------------------------------------
# integer bookkeeping
# ---------------------------------------------------------------------------

def group_index(t: int, s: int) -> int:
    """j(t) = ceil(t/s): the cache row that token t is merged into.

    Notes, *Key designs: hyper-network temporal merging* — every s adjacent
    latents merge into one c_hat_j, so the cache holds ceil(T/s) vectors."""
    if t < 1 or s < 1:
        raise ValueError("t and s are 1-based positive integers")
    return (t + s - 1) // s


def cache_length(t: int, s: int) -> int:
    """Rows in the compressed cache after t processed tokens: ceil(t/s) (0 for t=0).

    Notes, *Key designs: hyper-network temporal merging* (cache goes from T
    vectors to ceil(T/s)); News, s = 2 walk-through (length 1 after token 1 and
    still 1 after token 2)."""
    return 0 if t == 0 else group_index(t, s)


def opens_new_row(t: int, s: int) -> bool:
    """True when token t starts a new group (appends a row), i.e. (t-1) mod s == 0.

    For s >= 2 this is "t mod s == 1"; written this way it also covers s = 1,
    where every token opens its own row (MLA).  Figure 2(a): at steps 1, 3, 5
    (s = 2) the model works on a temporary c_hat'_j that the next step updates."""
    return (t - 1) % s == 0


def stride_visible(m: int, n: int, s: int) -> bool:
    """Stride-aware causal mask: query m may attend column n of C_hat' iff
    n == m, or n < m and n mod s == 0.

    Notes, *Key designs: stride-aware causal mask*; Figure 2(c)."""
    return n == m or (n < m and n % s == 0)


def visible_columns(m: int, s: int) -> list:
    """The 1-based columns of C_hat' that query m sees, in increasing order."""
    return [n for n in range(1, m + 1) if stride_visible(m, n, s)]


def stride_mask(T: int, s: int) -> np.ndarray:
    """The [T, T] boolean mask, entry [m-1, n-1] = stride_visible(m, n, s)."""
    M = np.zeros((T, T), dtype=bool)
    for m in range(1, T + 1):
        for n in range(1, T + 1):
            M[m - 1, n - 1] = stride_visible(m, n, s)
    return M


def cache_elements_per_token(d_h: int, s: int, layers: int = 1, r=None, d_R=None) -> float:
    """Average cache elements per processed token: (r + d_R) * layers / s.

    Notes, *Loss / training strategy*: with r = 4 d_h and d_R = d_h / 2 this is
    9 d_h l / (2 s), i.e. 2.25 d_h l at s = 2."""
    r = 4 * d_h if r is None else r
    d_R = d_h // 2 if d_R is None else d_R
    return (r + d_R) * layers / s


# ---------------------------------------------------------------------------
# hyper-network merge
# ---------------------------------------------------------------------------

def sigmoid(x):
    """Logistic function, evaluated without overflow for large |x|."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    e = np.exp(x[~pos])
    out[~pos] = e / (1.0 + e)
    return out


def sinusoidal_pe(J: int, D: int) -> np.ndarray:
    """Sinusoidal position encoding of width D for groups j = 1..J (row j-1).

    Row for group j uses position p = j - 1: pe[p, 2k] = sin(p / 10000^(2k/D)),
    pe[p, 2k+1] = cos(p / 10000^(2k/D)).  The pages name pe_j without giving
    its form; this is the Transformer sinusoid (the plainest reading)."""
    if D % 2:
        raise ValueError("D must be even")
    pe = np.zeros((J, D), dtype=np.float64)
    for p in range(J):
        for k in range(D // 2):
            angle = p / (10000.0 ** (2.0 * k / D))
            pe[p, 2 * k] = math.sin(angle)
            pe[p, 2 * k + 1] = math.cos(angle)
    return pe


def pe_table(J: int, W_p, b_p) -> np.ndarray:
    """P[j-1] = Linear(pe_j) = pe_j W_p + b_p, for j = 1..J (shape [J, D])."""
    W_p = np.asarray(W_p, dtype=np.float64)
    b_p = np.asarray(b_p, dtype=np.float64)
    return sinusoidal_pe(J, W_p.shape[0]) @ W_p + b_p


def merge_weight(c_t, P_j, W_c, b_c) -> np.ndarray:
    """w_t = Sigmoid(Linear(c_t) ⊙ Linear(pe_j)), channel-wise, width D.

    Notes, *Key designs: hyper-network temporal merging*: the weight is the
    sigmoid of the element-wise product of a Linear of the content c_t and a
    Linear of the position encoding of its group.  Linear(c_t) = c_t W_c + b_c
    (input width r, output width D, so the same gate covers [c_t ; k^R_t]);
    Linear(pe_j) arrives precomputed as P_j."""
    c_t = np.asarray(c_t, dtype=np.float64)
    g = c_t @ np.asarray(W_c, dtype=np.float64) + np.asarray(b_c, dtype=np.float64)
    return sigmoid(g * np.asarray(P_j, dtype=np.float64))


def merge_step(rows: list, t: int, s: int, c_t, kR_t, w) -> list:
    """Fold token t into the cache: returns the new list of rows.

    Notes, *Key designs*: c_hat_j = sum over the group of w_i ⊙ c_i (e.g.
    c_hat_1 = w_1 c_1 + w_2 c_2 at s = 2), and the RoPE keys are compressed the
    same way into k_hat^R.  Token t opens row j(t) when (t-1) mod s == 0 and is
    added in place to that (tail) row otherwise.  No normalisation."""
    entry = np.asarray(w, dtype=np.float64) * np.concatenate(
        [np.asarray(c_t, dtype=np.float64), np.asarray(kR_t, dtype=np.float64)])
    rows = [np.array(r_, dtype=np.float64) for r_ in rows]
    if opens_new_row(t, s):
        if len(rows) != group_index(t, s) - 1:
            raise ValueError("cache length does not match t-1 processed tokens")
        rows.append(entry)
    else:
        if len(rows) != group_index(t, s):
            raise ValueError("cache length does not match t-1 processed tokens")
        rows[-1] = rows[-1] + entry
    return rows


# ---------------------------------------------------------------------------
# absorbed attention
# ---------------------------------------------------------------------------

def decode_attention(q_abs, q_rope, rows, d_h: int):
    """Absorbed attention of one query position over cache rows.

    Notes, *Key designs: decoupled RoPE with temporal compression*:
    Y = softmax((X W_Q W_K^T C_hat^T + Q^R K_hat^R^T) / sqrt(d_h)) C_hat (W_V W_O).
    Per head h: score_j = (q_abs_h · c_hat_j + q^R_h · k_hat^R_j) / sqrt(d_h),
    p = softmax over j, o_h = sum_j p_j c_hat_j (width r; W_V W_O applied later).

    q_abs [H, r], q_rope [H, d_R], rows [L, r + d_R].  Returns (o [H, r],
    lse [H]) with lse the natural log of sum_j exp(score_j)."""
    q_abs = np.asarray(q_abs, dtype=np.float64)
    q_rope = np.asarray(q_rope, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64)
    H, r = q_abs.shape
    if rows.ndim != 2 or rows.shape[0] == 0:
        raise ValueError("attention needs at least one cache row")
    c_hat, k_hat = rows[:, :r], rows[:, r:]
    o = np.zeros((H, r))
    lse = np.zeros(H)
    for h in range(H):
        score = (c_hat @ q_abs[h] + k_hat @ q_rope[h]) / math.sqrt(d_h)
        mx = score.max()
        p = np.exp(score - mx)
        denom = p.sum()
        o[h] = (p @ c_hat) / denom
        lse[h] = mx + math.log(denom)
    return o, lse


def decode_step(rows, t_prev: int, s: int, c_new, kR_new, q_abs, q_rope,
                W_c, b_c, P, d_h: int):
    """One incremental decode step for one sequence (Figure 2(a)).

    Token t = t_prev + 1 is merged into the cache (append or in-place update
    of the tail row j(t), weight from its own group's P[j-1]), then the query
    attends every cached row, the partial tail included.
    Returns (rows_after, o [H, r], lse [H])."""
    t = t_prev + 1
    j = group_index(t, s)
    w = merge_weight(c_new, np.asarray(P)[j - 1], W_c, b_c)
    rows = merge_step(list(rows), t, s, c_new, kR_new, w)
    o, lse = decode_attention(q_abs, q_rope, np.stack(rows), d_h)
    return rows, o, lse


def decode_loop(c, kR, q_abs, q_rope, W_c, b_c, P, s: int, d_h: int):
    """Run tokens 1..T one at a time from an empty cache.

    c [T, r], kR [T, d_R], q_abs [T, H, r], q_rope [T, H, d_R].
    Returns dict with outputs o [T, H, r], lse [T, H], the cache length after
    each step, whether the tail row was partial (group not yet closed) after
    each step, and the final rows."""
    T = np.asarray(c).shape[0]
    rows: list = []
    outs, lses, lengths, partial = [], [], [], []
    for t in range(1, T + 1):
        rows, o, lse = decode_step(rows, t - 1, s, c[t - 1], kR[t - 1],
                                   q_abs[t - 1], q_rope[t - 1], W_c, b_c, P, d_h)
        outs.append(o)
        lses.append(lse)
        lengths.append(len(rows))
        partial.append(t % s != 0)
    return {"o": np.stack(outs), "lse": np.stack(lses),
            "lengths": np.array(lengths), "tail_partial": np.array(partial),
            "rows": np.stack(rows)}


# ---------------------------------------------------------------------------
# parallel (training / prefill) view
# ---------------------------------------------------------------------------

def partial_merge_sequence(c, kR, W_c, b_c, P, s: int) -> np.ndarray:
    """C_hat' [T, D]: position n holds the running merge of its group up to n.

    Notes, *Key designs: stride-aware causal mask*: training builds C_hat'
    where the positions of each group of s hold the intermediate and the final
    merged states; Figure 2(c).  C_hat'_n = sum_{i=(j(n)-1)s+1}^{n} w_i ⊙ [c_i ; k^R_i]."""
    c = np.asarray(c, dtype=np.float64)
    kR = np.asarray(kR, dtype=np.float64)
    W_c = np.asarray(W_c, dtype=np.float64)
    b_c = np.asarray(b_c, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    T = c.shape[0]
    gate_pre = c @ W_c + b_c                                   # Linear(c_n), all n
    Cp = np.zeros((T, W_c.shape[1]))
    for n in range(1, T + 1):
        j = group_index(n, s)
        w = sigmoid(gate_pre[n - 1] * P[j - 1])
        entry = w * np.concatenate([c[n - 1], kR[n - 1]])
        Cp[n - 1] = entry if opens_new_row(n, s) else Cp[n - 2] + entry
    return Cp


def compressed_cache(Cp: np.ndarray, s: int) -> np.ndarray:
    """The inference cache after T tokens: row g = C_hat'_{min(g s, T)}, g = 1..ceil(T/s)."""
    T = Cp.shape[0]
    L = cache_length(T, s)
    return np.stack([Cp[min(g * s, T) - 1] for g in range(1, L + 1)]) if L else Cp[:0]


def masked_forward(q_abs, q_rope, Cp, s: int, d_h: int):
    """Parallel forward under the stride-aware causal mask (explicit [T, T] mask).

    Notes, *Key designs: stride-aware causal mask* and *decoupled RoPE*:
    scores of every query against every column of C_hat', masked, softmax,
    o_{m,h} = sum_n p_{m,n} c_hat'_n.  q_abs [T, H, r], q_rope [T, H, d_R],
    Cp [T, D].  Returns (o [T, H, r], lse [T, H])."""
    q_abs = np.asarray(q_abs, dtype=np.float64)
    q_rope = np.asarray(q_rope, dtype=np.float64)
    Cp = np.asarray(Cp, dtype=np.float64)
    T, H, r = q_abs.shape
    mask = stride_mask(T, s)
    o = np.zeros((T, H, r))
    lse = np.zeros((T, H))
    for h in range(H):
        S = (q_abs[:, h, :] @ Cp[:, :r].T + q_rope[:, h, :] @ Cp[:, r:].T) / math.sqrt(d_h)
        S = np.where(mask, S, -np.inf)
        mx = S.max(axis=1, keepdims=True)
        E = np.exp(S - mx)
        denom = E.sum(axis=1, keepdims=True)
        o[:, h, :] = (E / denom) @ Cp[:, :r]
        lse[:, h] = mx[:, 0] + np.log(denom[:, 0])
    return o, lse


def masked_forward_query(m: int, q_abs_m, q_rope_m, Cp, s: int, d_h: int):
    """Row m (1-based) of ``masked_forward`` for one query, over its visible columns only.

    Used for sampled outputs at sizes where the [T, T] form is too large."""
    cols = np.array(visible_columns(m, s), dtype=np.int64) - 1
    return decode_attention(q_abs_m, q_rope_m, np.asarray(Cp)[cols], d_h)


# ---------------------------------------------------------------------------
# layer glue around the hot path (used for end-to-end checks)
# ---------------------------------------------------------------------------

def rope(v, pos):
    """Rotary position embedding of rows v [T, d_R] at 0-based positions pos [T].

    The pages use decoupled RoPE (as in MLA) without giving its form; this is
    the RoFormer rotation of channel pairs (2k, 2k+1) by angle
    pos * 10000^(-2k/d_R)."""
    v = np.asarray(v, dtype=np.float64)
    pos = np.asarray(pos, dtype=np.float64)
    T, d_R = v.shape
    out = np.zeros_like(v)
    for k in range(d_R // 2):
        theta = 10000.0 ** (-2.0 * k / d_R)
        a = pos * theta
        x0, x1 = v[:, 2 * k], v[:, 2 * k + 1]
        out[:, 2 * k] = x0 * np.cos(a) - x1 * np.sin(a)
        out[:, 2 * k + 1] = x0 * np.sin(a) + x1 * np.cos(a)
    return out


def project_inputs(x, W, pos=None):
    """Hot-path inputs of one sequence from the layer input x [T, d].

    Notes, *Overall framework*: Q = X W_Q, latent C = X W_down; Figure 1 and
    the decoupled-RoPE formula: the key map is absorbed into the query,
    q_abs_h = (x W_Q^h)(W_K^h)^T (width r); RoPE query/key from their own maps.
    W: W_Q [d,H,d_h], W_K [H,r,d_h], W_down [d,r], W_QR [d,H,d_R], W_KR [d,d_R].
    pos: 0-based positions of the T rows for RoPE (default 0..T-1, a whole
    sequence from its start; a decode step passes its token's t - 1).
    Returns q_abs [T,H,r], q_rope [T,H,d_R], c [T,r], kR [T,d_R]."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    W_Q = np.asarray(W["W_Q"], dtype=np.float64)
    W_K = np.asarray(W["W_K"], dtype=np.float64)
    W_QR = np.asarray(W["W_QR"], dtype=np.float64)
    H = W_Q.shape[1]
    r = W_K.shape[1]
    d_R = W_QR.shape[2]
    pos = np.arange(T) if pos is None else np.asarray(pos)
    c = x @ np.asarray(W["W_down"], dtype=np.float64)
    kR = rope(x @ np.asarray(W["W_KR"], dtype=np.float64), pos)
    q_abs = np.zeros((T, H, r))
    q_rope = np.zeros((T, H, d_R))
    for h in range(H):
        q_abs[:, h, :] = (x @ W_Q[:, h, :]) @ W_K[h].T
        q_rope[:, h, :] = rope(x @ W_QR[:, h, :], pos)
    return q_abs, q_rope, c, kR


def absorbed_output(o, W_V, W_O):
    """y = sum_h o_h (W_V^h W_O^h): the value and output maps applied after
    attention (Figure 1: absorbed into the output linear layer).

    o [T, H, r], W_V [H, r, d_h], W_O [H*d_h, d]."""
    o = np.asarray(o, dtype=np.float64)
    W_V = np.asarray(W_V, dtype=np.float64)
    W_O = np.asarray(W_O, dtype=np.float64)
    T, H, r = o.shape
    d_h = W_V.shape[2]
    y = np.zeros((T, W_O.shape[1]))
    for h in range(H):
        y += (o[:, h, :] @ W_V[h]) @ W_O[h * d_h:(h + 1) * d_h, :]
    return y


def unabsorbed_forward(x, W, Cp, s: int):
    """Brute force with explicit per-head keys and values (tiny sizes only).

    q_h = x W_Q^h, q^R_h = RoPE(x W_QR^h), K_h = C_hat'_latent W_K^h,
    V_h = C_hat'_latent W_V^h, K^R = C_hat'_rope; score = (q_h·K_h,n +
    q^R_h·K^R_n)/sqrt(d_h) under the stride-aware mask; y = concat_h(p V_h) W_O.
    Figure 1: this must equal the absorbed computation by associativity."""
    x = np.asarray(x, dtype=np.float64)
    Cp = np.asarray(Cp, dtype=np.float64)
    W_Q = np.asarray(W["W_Q"], dtype=np.float64)
    W_K = np.asarray(W["W_K"], dtype=np.float64)
    W_V = np.asarray(W["W_V"], dtype=np.float64)
    W_QR = np.asarray(W["W_QR"], dtype=np.float64)
    W_O = np.asarray(W["W_O"], dtype=np.float64)
    T = x.shape[0]
    H, r, d_h = W_K.shape
    pos = np.arange(T)
    mask = stride_mask(T, s)
    heads = []
    for h in range(H):
        q = x @ W_Q[:, h, :]
        qR = rope(x @ W_QR[:, h, :], pos)
        K = Cp[:, :r] @ W_K[h]
        V = Cp[:, :r] @ W_V[h]
        KR = Cp[:, r:]
        S = (q @ K.T + qR @ KR.T) / math.sqrt(d_h)
        S = np.where(mask, S, -np.inf)
        E = np.exp(S - S.max(axis=1, keepdims=True))
        heads.append((E / E.sum(axis=1, keepdims=True)) @ V)
    return np.concatenate(heads, axis=1) @ W_O


def unabsorbed_heads(x, W, Cp, s: int, pos=None):
    """Per-head outputs of the masked forward with explicit keys and values
    (the un-absorbed form the notes page describes before absorbing W_K and
    W_V, *Key designs: decoupled RoPE with temporal compression*):
    q_h = x W_Q^h, q^R_h = RoPE(x W_QR^h), K_h = C_hat'_latent W_K^h,
    V_h = C_hat'_latent W_V^h, K^R = C_hat'_rope;
    score = (q_h . K_h,n + q^R_h . K^R_n) / sqrt(d_h) under the stride-aware
    mask; o_h = sum_n softmax(score)_n V_h,n.  Returns [T, H, d_h]."""
    x = np.asarray(x, dtype=np.float64)
    Cp = np.asarray(Cp, dtype=np.float64)
    W_Q = np.asarray(W["W_Q"], dtype=np.float64)
    W_K = np.asarray(W["W_K"], dtype=np.float64)
    W_V = np.asarray(W["W_V"], dtype=np.float64)
    W_QR = np.asarray(W["W_QR"], dtype=np.float64)
    T = x.shape[0]
    H, r, d_h = W_K.shape
    pos = np.arange(T) if pos is None else np.asarray(pos)
    mask = stride_mask(T, s)
    out = np.zeros((T, H, d_h))
    for h in range(H):
        q = x @ W_Q[:, h, :]
        qR = rope(x @ W_QR[:, h, :], pos)
        K = Cp[:, :r] @ W_K[h]
        V = Cp[:, :r] @ W_V[h]
        S = (q @ K.T + qR @ Cp[:, r:].T) / math.sqrt(d_h)
        S = np.where(mask, S, -np.inf)
        E = np.exp(S - S.max(axis=1, keepdims=True))
        out[:, h, :] = (E / E.sum(axis=1, keepdims=True)) @ V
    return out


# ---------------------------------------------------------------------------
# training path: the uncompressed-RoPE-key shortcut and its backward pass
# ---------------------------------------------------------------------------

def latent_partial_merge(c, W_c, b_c, P, s: int) -> np.ndarray:
    """C_hat'_latent [T, r]: the latent channels of the running merge.

    Notes, *Key designs: stride-aware causal mask* (C_hat') and *hyper-network
    temporal merging* (the gate): C_hat'_n = sum_{i=(j(n)-1)s+1}^{n} w_i[:r] ⊙ c_i
    with w_i = Sigmoid(Linear(c_i) ⊙ P[j(i)-1]).  Under the training shortcut
    (*decoupled RoPE with temporal compression*: training may take the
    uncompressed K^R in place of K_hat^R) only these channels feed the
    attention, so gate channels r.. play no part."""
    c = np.asarray(c, dtype=np.float64)
    W_c = np.asarray(W_c, dtype=np.float64)
    b_c = np.asarray(b_c, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    T, r = c.shape
    gate_pre = c @ W_c[:, :r] + b_c[:r]
    Cp = np.zeros((T, r))
    for n in range(1, T + 1):
        j = group_index(n, s)
        entry = sigmoid(gate_pre[n - 1] * P[j - 1, :r]) * c[n - 1]
        Cp[n - 1] = entry if opens_new_row(n, s) else Cp[n - 2] + entry
    return Cp


def shortcut_attention(q, q_rope, k, v, kR, s: int):
    """Masked attention with explicit per-head keys and values and the
    uncompressed RoPE keys (the training shortcut).

    Notes, *Key designs: decoupled RoPE with temporal compression* (training
    may use K^R itself instead of the merged K_hat^R) and *stride-aware causal
    mask*: per head h, score_{m,n} = (q_{m,h} . k_{n,h} + q^R_{m,h} . k^R_n) /
    sqrt(d_h) for n == m or (n < m and n mod s == 0), p = softmax over n,
    o_{m,h} = sum_n p_{m,n} v_{n,h}.  q, k, v [T, H, d_h], q_rope [T, H, d_R],
    kR [T, d_R].  Returns (o [T, H, d_h], lse [T, H]), lse the natural log of
    sum_n exp(score_{m,n})."""
    q, q_rope, k, v, kR = (np.asarray(a, dtype=np.float64) for a in (q, q_rope, k, v, kR))
    T, H, d_h = q.shape
    mask = stride_mask(T, s)
    o = np.zeros((T, H, d_h))
    lse = np.zeros((T, H))
    for h in range(H):
        S = (q[:, h] @ k[:, h].T + q_rope[:, h] @ kR.T) / math.sqrt(d_h)
        S = np.where(mask, S, -np.inf)
        mx = S.max(axis=1, keepdims=True)
        E = np.exp(S - mx)
        denom = E.sum(axis=1, keepdims=True)
        o[:, h] = (E / denom) @ v[:, h]
        lse[:, h] = mx[:, 0] + np.log(denom[:, 0])
    return o, lse


def shortcut_attention_backward(q, q_rope, k, v, kR, s: int, d_out):
    """Gradients of a loss through ``shortcut_attention``, given d_out = dL/do.

    The chain rule through score -> softmax -> weighted sum, per head:
    dP = d_out V^T; dS = P ⊙ (dP - rowsum(P ⊙ dP)) (the softmax Jacobian);
    dq = dS K / sqrt(d_h), dq^R = dS K^R / sqrt(d_h), dk = dS^T q / sqrt(d_h),
    dv = P^T d_out, dk^R = sum_h dS^T q^R_h / sqrt(d_h) (K^R is shared by
    every head).  Returns (dq, dq_rope, dk, dv, dkR) shaped like the inputs."""
    q, q_rope, k, v, kR, d_out = (np.asarray(a, dtype=np.float64) for a in (q, q_rope, k, v, kR, d_out))
    T, H, d_h = q.shape
    mask = stride_mask(T, s)
    sc = 1.0 / math.sqrt(d_h)
    dq, dq_rope, dk, dv = (np.zeros_like(a) for a in (q, q_rope, k, v))
    dkR = np.zeros_like(kR)
    for h in range(H):
        S = (q[:, h] @ k[:, h].T + q_rope[:, h] @ kR.T) * sc
        S = np.where(mask, S, -np.inf)
        E = np.exp(S - S.max(axis=1, keepdims=True))
        Pm = E / E.sum(axis=1, keepdims=True)
        dP = d_out[:, h] @ v[:, h].T
        dS = Pm * (dP - (Pm * dP).sum(axis=1, keepdims=True))
        dq[:, h] = dS @ k[:, h] * sc
        dq_rope[:, h] = dS @ kR * sc
        dk[:, h] = dS.T @ q[:, h] * sc
        dv[:, h] = Pm.T @ d_out[:, h]
        dkR += dS.T @ q_rope[:, h] * sc
    return dq, dq_rope, dk, dv, dkR


def kv_backward(dk, dv, W_K, W_V) -> np.ndarray:
    """dL/dC_hat'_latent through k_h = C_hat'_latent W_K^h and v_h = C_hat'_latent W_V^h
    (the un-absorbed key and value maps, Figure 1): sum_h dk_h (W_K^h)^T + dv_h (W_V^h)^T.
    dk, dv [T, H, d_h]; W_K, W_V [H, r, d_h].  Returns [T, r]."""
    dk, dv, W_K, W_V = (np.asarray(a, dtype=np.float64) for a in (dk, dv, W_K, W_V))
    H = W_K.shape[0]
    return sum(dk[:, h] @ W_K[h].T + dv[:, h] @ W_V[h].T for h in range(H))


def latent_merge_backward(c, W_c, b_c, P, s: int, dCp):
    """Gradients of a loss through ``latent_partial_merge``, given dCp = dL/dC_hat'_latent.

    Chain rule in the order of the forward (Notes, *hyper-network temporal
    merging*):
    - de_i = sum of dCp_n over the positions n >= i of token i's group
      (C_hat'_n sums the gated entries e_i of its group up to n);
    - e_i = w_i ⊙ c_i gives dw_i = de_i ⊙ c_i and a direct dc_i = de_i ⊙ w_i;
    - w_i = Sigmoid(z_i) gives dz_i = dw_i ⊙ w_i ⊙ (1 - w_i);
    - z_i = g_i ⊙ P[j(i)-1] gives dg_i = dz_i ⊙ P[j(i)-1] and dP[j(i)-1] += dz_i ⊙ g_i;
    - g_i = c_i W_c + b_c gives dc_i += dg_i W_c^T, dW_c += c_i^T dg_i, db_c += dg_i.
    Only the first r gate channels reach C_hat'_latent; the other channels of
    dW_c, db_c and dP are zero.  Returns (dc [T, r], dW_c, db_c, dP) shaped
    like c, W_c, b_c and P."""
    c, W_c, b_c, P, dCp = (np.asarray(a, dtype=np.float64) for a in (c, W_c, b_c, P, dCp))
    T, r = c.shape
    g = c @ W_c[:, :r] + b_c[:r]
    de = np.zeros((T, r))
    for i in range(T, 0, -1):
        de[i - 1] = dCp[i - 1]
        if i < T and not opens_new_row(i + 1, s):
            de[i - 1] += de[i]
    dc = np.zeros((T, r))
    dW_c = np.zeros_like(W_c)
    db_c = np.zeros_like(b_c)
    dP = np.zeros_like(P)
    for i in range(1, T + 1):
        j = group_index(i, s)
        u = P[j - 1, :r]
        w = sigmoid(g[i - 1] * u)
        dw = de[i - 1] * c[i - 1]
        dz = dw * w * (1.0 - w)
        dg = dz * u
        dP[j - 1, :r] += dz * g[i - 1]
        dc[i - 1] = de[i - 1] * w + W_c[:, :r] @ dg
        dW_c[:, :r] += np.outer(c[i - 1], dg)
        db_c[:r] += dg
    return dc, dW_c, db_c, dP
