// Backward pass of the masked attention with explicit per-head keys and
// values and the uncompressed RoPE keys: the training shortcut of the MTLA
// paper notes ("Key designs: decoupled RoPE with temporal compression":
// training may use K^R itself instead of the merged K_hat^R) under the
// stride-aware causal mask ("Key designs: stride-aware causal mask").
//
// For query m, head h and visible column n (n == m, or n = g s < m):
//   score = (q . k_n + q^R . k^R_n) / sqrt(d_h),  P = softmax over n,
//   dP = dO . v_n,  dS = P (dP - Delta_m),  Delta_m = dO_m . O_m,
//   dq += dS [k_n | k^R_n] / sqrt(d_h),  d[k_n | k^R_n] += dS [q | q^R] / sqrt(d_h),
//   dv_n += P dO_m.
// bf16 operands, d_h = 64, d_R = 32 (score width 96), fp32 accumulation on
// warp-level tensor-core MMAs (m16n8k16), P and dS rounded to bf16 as MMA
// operands.
//
// Four kernels, no atomics (every output row is written by exactly one block):
// - prep: Delta and the log2-unit lse per (sequence, head, query);
// - dq: a block is 64 queries of one head; it streams the 64-wide tiles of
//   the group columns they see (like the forward) and accumulates dq in
//   registers.  It also takes every row's own column (n == m), and writes the
//   key and value gradients of the rows no later query sees (n mod s != 0);
// - dkv: a block is 64 group columns (n = g s) of one head; it streams the
//   64-query tiles that see them (m > g s) and accumulates dk, dk^R and dv in
//   registers, its own columns' terms included;
// - the RoPE key gradient summed over heads.
#include "kernels.cuh"

namespace mtla {
namespace tbw {

constexpr int DH = 64, DR = 32, DK = DH + DR;
constexpr int TB = 64;                          // queries (dq) or key columns (dkv) per block, and tile width
constexpr int NW = 4, NT = 32 * NW;
constexpr int KS = DK + 8;                      // padded row stride of 96-wide rows (elements)
constexpr int VS = DH + 8;                      // padded row stride of 64-wide rows
constexpr int KTILE = TB * KS, VTILE = TB * VS; // elements
constexpr size_t SMEM_DQ = (size_t)2 * (KTILE + VTILE) * 2;
constexpr size_t SMEM_DKV = SMEM_DQ + (size_t)2 * 2 * TB * 4;

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g, bool valid) {
  // a chunk that is not valid is filled with zeros (src-size 0)
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr), "l"(g), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ uint32_t ld_u32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }
__device__ __forceinline__ float2 bf2(uint32_t u) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
}
__device__ __forceinline__ float dot2(uint32_t a, uint32_t b) {
  const float2 x = bf2(a), y = bf2(b);
  return x.x * y.x + x.y * y.y;
}
__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v + __shfl_xor_sync(0xffffffffu, v, 2);
}

// Fragment positions of m16n8k16 operands held by this thread: for k-chunk kk,
// columns c0 = 16 kk + 2 (lane & 3) (two elements) and c1 = c0 + 8, rows
// (lane >> 2) and (lane >> 2) + 8; registers ordered (rowA, c0), (rowB, c0),
// (rowA, c1), (rowB, c1).  A row of the 96-wide operand is [x (64) | x^R (32)].
__device__ __forceinline__ uint32_t at96(const __nv_bfloat16* x, const __nv_bfloat16* xr, int c) {
  return c < DH ? ld_u32(x + c) : ld_u32(xr + (c - DH));
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdArgs p) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // (b, t, h)
  if (idx >= (int64_t)p.B * p.T * p.H) return;
  const int h = (int)(idx % p.H);
  const int64_t bt = idx / p.H;
  const int64_t b = bt / p.T, t = bt % p.T;
  const uint4* o4 = reinterpret_cast<const uint4*>(p.o + idx * DH);
  const uint4* d4 = reinterpret_cast<const uint4*>(p.dout + idx * DH);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < DH / 8; ++i) {
    const uint4 a = o4[i], c = d4[i];
    acc += dot2(a.x, c.x) + dot2(a.y, c.y) + dot2(a.z, c.z) + dot2(a.w, c.w);
  }
  const int64_t o = (b * p.H + h) * p.T + t;
  p.ws_delta[o] = acc;
  p.ws_lse2[o] = p.lse[idx] * 1.4426950408889634f;
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(NT) bwd_dq_kernel(const BwdArgs p) {
  extern __shared__ __align__(16) __nv_bfloat16 smq[];
  __nv_bfloat16* Kt = smq;             // [2][TB][KS] [k | k^R] rows of the group columns
  __nv_bfloat16* Vt = Kt + 2 * KTILE;  // [2][TB][VS] v rows
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int T = p.T, H = p.H, s = p.s;
  const int nqb = (T + TB - 1) / TB;
  const int qb = nqb - 1 - (int)(blockIdx.x / (p.B * H));  // heaviest first
  const int bh = (int)(blockIdx.x % (p.B * H));
  const int b = bh / H, h = bh % H;
  const int m0 = qb * TB + 1;
  const int m_last = m0 + TB - 1 < T ? m0 + TB - 1 : T;
  const int vis_max = (int)group_of(m_last, s) - 1;
  const int nkt = (vis_max + TB - 1) / TB;
  const int64_t row0 = (int64_t)b * T;
  const int n_groups = T / s;

  // key tile kt: groups kt TB .. + TB - 1 (column n = (grp + 1) s)
  auto load_tile = [&](int kt, int buf) {
    const uint32_t kb = smem_u32(Kt + buf * KTILE), vb = smem_u32(Vt + buf * VTILE);
    for (int i = tid; i < TB * 20; i += NT) {
      const int r = i / 20, c = i % 20;
      const int grp = kt * TB + r;
      const bool valid = grp < n_groups;
      const int64_t pos = row0 + (valid ? (int64_t)(grp + 1) * s - 1 : 0);  // a row of the sequence even when not read
      if (c < 8) cp_async16(kb + (uint32_t)(r * KS + c * 8) * 2, p.k + (pos * H + h) * DH + c * 8, valid);
      else if (c < 12)
        cp_async16(kb + (uint32_t)(r * KS + DH + (c - 8) * 8) * 2, p.kr + pos * DR + (c - 8) * 8, valid);
      else cp_async16(vb + (uint32_t)(r * VS + (c - 12) * 8) * 2, p.v + (pos * H + h) * DH + (c - 12) * 8, valid);
    }
  };
  if (nkt > 0) load_tile(0, 0);
  cp_commit();

  const int r0 = 16 * warp + g;
  const int ma = m0 + r0, mb = ma + 8;  // this thread's two queries (1-based)
  const bool va = ma <= T, vb = mb <= T;
  const int64_t rA = row0 + (va ? ma - 1 : 0), rB = row0 + (vb ? mb - 1 : 0);
  const int64_t lbase = ((int64_t)b * H + h) * T;
  const float lA = va ? p.ws_lse2[lbase + ma - 1] : 0.f, lB = vb ? p.ws_lse2[lbase + mb - 1] : 0.f;
  const float dA = va ? p.ws_delta[lbase + ma - 1] : 0.f, dB = vb ? p.ws_delta[lbase + mb - 1] : 0.f;
  const float sl2 = p.scale_log2, sc = p.scale;

  uint32_t qf[6][4], of[4][4];
  float dq[12][4];
  {
    const __nv_bfloat16 *qa = p.q + (rA * H + h) * DH, *qb_ = p.q + (rB * H + h) * DH;
    const __nv_bfloat16 *ra = p.qr + (rA * H + h) * DR, *rb = p.qr + (rB * H + h) * DR;
    const __nv_bfloat16 *ka = p.k + (rA * H + h) * DH, *kb = p.k + (rB * H + h) * DH;
    const __nv_bfloat16 *kra = p.kr + rA * DR, *krb = p.kr + rB * DR;
    const __nv_bfloat16 *oa = p.dout + (rA * H + h) * DH, *ob = p.dout + (rB * H + h) * DH;
    const __nv_bfloat16 *wa = p.v + (rA * H + h) * DH, *wb = p.v + (rB * H + h) * DH;
    uint32_t kf[6][4], vf[4][4];
    float sA = 0.f, sB = 0.f, pdA = 0.f, pdB = 0.f;
#pragma unroll
    for (int kk = 0; kk < 6; ++kk) {
      const int c0 = 16 * kk + 2 * q, c1 = c0 + 8;
      qf[kk][0] = va ? at96(qa, ra, c0) : 0u;
      qf[kk][1] = vb ? at96(qb_, rb, c0) : 0u;
      qf[kk][2] = va ? at96(qa, ra, c1) : 0u;
      qf[kk][3] = vb ? at96(qb_, rb, c1) : 0u;
      kf[kk][0] = va ? at96(ka, kra, c0) : 0u;
      kf[kk][1] = vb ? at96(kb, krb, c0) : 0u;
      kf[kk][2] = va ? at96(ka, kra, c1) : 0u;
      kf[kk][3] = vb ? at96(kb, krb, c1) : 0u;
      sA += dot2(qf[kk][0], kf[kk][0]) + dot2(qf[kk][2], kf[kk][2]);
      sB += dot2(qf[kk][1], kf[kk][1]) + dot2(qf[kk][3], kf[kk][3]);
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int c0 = 16 * kk + 2 * q, c1 = c0 + 8;
      of[kk][0] = va ? ld_u32(oa + c0) : 0u;
      of[kk][1] = vb ? ld_u32(ob + c0) : 0u;
      of[kk][2] = va ? ld_u32(oa + c1) : 0u;
      of[kk][3] = vb ? ld_u32(ob + c1) : 0u;
      vf[kk][0] = va ? ld_u32(wa + c0) : 0u;
      vf[kk][1] = vb ? ld_u32(wb + c0) : 0u;
      vf[kk][2] = va ? ld_u32(wa + c1) : 0u;
      vf[kk][3] = vb ? ld_u32(wb + c1) : 0u;
      pdA += dot2(of[kk][0], vf[kk][0]) + dot2(of[kk][2], vf[kk][2]);
      pdB += dot2(of[kk][1], vf[kk][1]) + dot2(of[kk][3], vf[kk][3]);
    }
    sA = quad_sum(sA);
    sB = quad_sum(sB);
    pdA = quad_sum(pdA);
    pdB = quad_sum(pdB);
    // the own column n == m
    const float pA = va ? exp2f(sA * sl2 - lA) : 0.f, pB = vb ? exp2f(sB * sl2 - lB) : 0.f;
    const float gA = pA * (pdA - dA), gB = pB * (pdB - dB);
#pragma unroll
    for (int kk = 0; kk < 6; ++kk) {
      const float2 k0 = bf2(kf[kk][0]), k1 = bf2(kf[kk][1]), k2 = bf2(kf[kk][2]), k3 = bf2(kf[kk][3]);
      dq[2 * kk][0] = gA * k0.x;
      dq[2 * kk][1] = gA * k0.y;
      dq[2 * kk][2] = gB * k1.x;
      dq[2 * kk][3] = gB * k1.y;
      dq[2 * kk + 1][0] = gA * k2.x;
      dq[2 * kk + 1][1] = gA * k2.y;
      dq[2 * kk + 1][2] = gB * k3.x;
      dq[2 * kk + 1][3] = gB * k3.y;
    }
    // rows that no later query sees (n mod s != 0): their key and value
    // gradients are the own column's terms alone
    const bool ownA = va && (ma % s) != 0, ownB = vb && (mb % s) != 0;
#pragma unroll
    for (int kk = 0; kk < 6; ++kk) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int c = 16 * kk + 2 * q + 8 * half;
        const float2 xa = bf2(qf[kk][2 * half]), xb = bf2(qf[kk][2 * half + 1]);
        if (c < DH) {
          if (ownA) *reinterpret_cast<uint32_t*>(p.dk + (rA * H + h) * DH + c) = pack_bf16x2(gA * sc * xa.x, gA * sc * xa.y);
          if (ownB) *reinterpret_cast<uint32_t*>(p.dk + (rB * H + h) * DH + c) = pack_bf16x2(gB * sc * xb.x, gB * sc * xb.y);
        } else {
          if (ownA) *reinterpret_cast<float2*>(p.ws_dkrh + (rA * H + h) * DR + (c - DH)) = make_float2(gA * sc * xa.x, gA * sc * xa.y);
          if (ownB) *reinterpret_cast<float2*>(p.ws_dkrh + (rB * H + h) * DR + (c - DH)) = make_float2(gB * sc * xb.x, gB * sc * xb.y);
        }
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int c = 16 * kk + 2 * q + 8 * half;
        const float2 xa = bf2(of[kk][2 * half]), xb = bf2(of[kk][2 * half + 1]);
        if (ownA) *reinterpret_cast<uint32_t*>(p.dv + (rA * H + h) * DH + c) = pack_bf16x2(pA * xa.x, pA * xa.y);
        if (ownB) *reinterpret_cast<uint32_t*>(p.dv + (rB * H + h) * DH + c) = pack_bf16x2(pB * xb.x, pB * xb.y);
      }
    }
  }
  const int visA = va ? (int)group_of(ma, s) - 1 : 0;  // completed groups each query sees
  const int visB = vb ? (int)group_of(mb, s) - 1 : 0;

  const int lrow = lane & 7, lsel = lane >> 3;
  for (int kt = 0; kt < nkt; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nkt) load_tile(kt + 1, buf ^ 1);
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    const uint32_t kbase = smem_u32(Kt + buf * KTILE), vbase = smem_u32(Vt + buf * VTILE);
#pragma unroll
    for (int half = 0; half < 2; ++half) {  // keys 32 half .. 32 half + 31 of the tile
      float S[4][4], dP[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) S[i][0] = S[i][1] = S[i][2] = S[i][3] = dP[i][0] = dP[i][1] = dP[i][2] = dP[i][3] = 0.f;
#pragma unroll
      for (int nl = 0; nl < 4; ++nl) {
        const int nb = 4 * half + nl;
#pragma unroll
        for (int kk2 = 0; kk2 < 3; ++kk2) {  // S = [q | q^R] [k | k^R]^T
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kbase + (uint32_t)((8 * nb + lrow) * KS + 32 * kk2 + 8 * lsel) * 2, b0, b1, b2, b3);
          mma_bf16(S[nl], qf[2 * kk2][0], qf[2 * kk2][1], qf[2 * kk2][2], qf[2 * kk2][3], b0, b1);
          mma_bf16(S[nl], qf[2 * kk2 + 1][0], qf[2 * kk2 + 1][1], qf[2 * kk2 + 1][2], qf[2 * kk2 + 1][3], b2, b3);
        }
#pragma unroll
        for (int kk2 = 0; kk2 < 2; ++kk2) {  // dP = dO v^T
          uint32_t b0, b1, b2, b3;
          ldsm_x4(vbase + (uint32_t)((8 * nb + lrow) * VS + 32 * kk2 + 8 * lsel) * 2, b0, b1, b2, b3);
          mma_bf16(dP[nl], of[2 * kk2][0], of[2 * kk2][1], of[2 * kk2][2], of[2 * kk2][3], b0, b1);
          mma_bf16(dP[nl], of[2 * kk2 + 1][0], of[2 * kk2 + 1][1], of[2 * kk2 + 1][2], of[2 * kk2 + 1][3], b2, b3);
        }
      }
      uint32_t ds[4][2];
#pragma unroll
      for (int nl = 0; nl < 4; ++nl) {
        const int gi = kt * TB + 8 * (4 * half + nl) + 2 * q;  // 0-based group of the column
        const float p0 = gi < visA ? exp2f(S[nl][0] * sl2 - lA) : 0.f;
        const float p1 = gi + 1 < visA ? exp2f(S[nl][1] * sl2 - lA) : 0.f;
        const float p2 = gi < visB ? exp2f(S[nl][2] * sl2 - lB) : 0.f;
        const float p3 = gi + 1 < visB ? exp2f(S[nl][3] * sl2 - lB) : 0.f;
        ds[nl][0] = pack_bf16x2(p0 * (dP[nl][0] - dA), p1 * (dP[nl][1] - dA));
        ds[nl][1] = pack_bf16x2(p2 * (dP[nl][2] - dB), p3 * (dP[nl][3] - dB));
      }
      // dq [16 x 96] += dS [16 x 32 keys] [k | k^R] [32 keys x 96]
#pragma unroll
      for (int kl = 0; kl < 2; ++kl) {
        const uint32_t a0 = ds[2 * kl][0], a1 = ds[2 * kl][1], a2 = ds[2 * kl + 1][0], a3 = ds[2 * kl + 1][1];
#pragma unroll
        for (int nb2 = 0; nb2 < 6; ++nb2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(kbase + (uint32_t)((32 * half + 16 * kl + lrow + 8 * (lsel & 1)) * KS + 16 * nb2 + 8 * (lsel >> 1)) * 2,
                    b0, b1, b2, b3);
          mma_bf16(dq[2 * nb2], a0, a1, a2, a3, b0, b1);
          mma_bf16(dq[2 * nb2 + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    __syncthreads();  // the buffer is refilled by the next iteration's prefetch
  }
  cp_wait<0>();

#pragma unroll
  for (int nb = 0; nb < 12; ++nb) {
    const int c = 8 * nb + 2 * q;
    if (c < DH) {
      if (va) *reinterpret_cast<uint32_t*>(p.dq + (rA * H + h) * DH + c) = pack_bf16x2(dq[nb][0] * sc, dq[nb][1] * sc);
      if (vb) *reinterpret_cast<uint32_t*>(p.dq + (rB * H + h) * DH + c) = pack_bf16x2(dq[nb][2] * sc, dq[nb][3] * sc);
    } else {
      if (va) *reinterpret_cast<uint32_t*>(p.dqr + (rA * H + h) * DR + (c - DH)) = pack_bf16x2(dq[nb][0] * sc, dq[nb][1] * sc);
      if (vb) *reinterpret_cast<uint32_t*>(p.dqr + (rB * H + h) * DR + (c - DH)) = pack_bf16x2(dq[nb][2] * sc, dq[nb][3] * sc);
    }
  }
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(NT) bwd_dkv_kernel(const BwdArgs p) {
  extern __shared__ __align__(16) __nv_bfloat16 smk[];
  __nv_bfloat16* Qt = smk;                                // [2][TB][KS] [q | q^R] rows of the query tile
  __nv_bfloat16* Ot = Qt + 2 * KTILE;                     // [2][TB][VS] dO rows
  float* Ls = reinterpret_cast<float*>(Ot + 2 * VTILE);   // [2][TB] lse2
  float* Ds = Ls + 2 * TB;                                // [2][TB] Delta
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int T = p.T, H = p.H, s = p.s;
  const int n_groups = T / s;
  const int kb = (int)(blockIdx.x / (p.B * H));  // earliest groups (the most queries) first
  const int bh = (int)(blockIdx.x % (p.B * H));
  const int b = bh / H, h = bh % H;
  const int g0 = kb * TB;                         // groups g0 + 1 .. g0 + TB (1-based)
  const int64_t row0 = (int64_t)b * T;
  const int64_t lbase = ((int64_t)b * H + h) * T;
  const int m_start = (g0 + 1) * s + 1;           // first query that sees the block's first column
  const int nqt = m_start <= T ? (T - m_start + TB) / TB : 0;

  auto load_tile = [&](int qt, int buf) {
    const uint32_t qs = smem_u32(Qt + buf * KTILE), os = smem_u32(Ot + buf * VTILE);
    const int mt0 = m_start + qt * TB;
    for (int i = tid; i < TB * 20; i += NT) {
      const int r = i / 20, c = i % 20;
      const bool valid = mt0 + r <= T;
      const int64_t pos = row0 + (valid ? mt0 - 1 + r : 0);
      if (c < 8) cp_async16(qs + (uint32_t)(r * KS + c * 8) * 2, p.q + (pos * H + h) * DH + c * 8, valid);
      else if (c < 12)
        cp_async16(qs + (uint32_t)(r * KS + DH + (c - 8) * 8) * 2, p.qr + (pos * H + h) * DR + (c - 8) * 8, valid);
      else cp_async16(os + (uint32_t)(r * VS + (c - 12) * 8) * 2, p.dout + (pos * H + h) * DH + (c - 12) * 8, valid);
    }
  };
  if (nqt > 0) {
    load_tile(0, 0);
    if (tid < TB) {
      const int m = m_start + tid;
      Ls[tid] = m <= T ? p.ws_lse2[lbase + m - 1] : 0.f;
      Ds[tid] = m <= T ? p.ws_delta[lbase + m - 1] : 0.f;
    }
  }
  cp_commit();

  const int r0 = 16 * warp + g;
  const int gA = g0 + r0 + 1, gB = gA + 8;  // this thread's two key columns: groups gA, gB
  const bool va = gA <= n_groups, vb = gB <= n_groups;
  const int nA = gA * s, nB = gB * s;       // their 1-based positions
  const int64_t rA = row0 + (va ? nA - 1 : 0), rB = row0 + (vb ? nB - 1 : 0);
  const float sl2 = p.scale_log2, sc = p.scale;

  uint32_t kf[6][4], vf[4][4];
  float dk[12][4], dv[8][4];
  {
    const __nv_bfloat16 *ka = p.k + (rA * H + h) * DH, *kb_ = p.k + (rB * H + h) * DH;
    const __nv_bfloat16 *kra = p.kr + rA * DR, *krb = p.kr + rB * DR;
    const __nv_bfloat16 *qa = p.q + (rA * H + h) * DH, *qb = p.q + (rB * H + h) * DH;
    const __nv_bfloat16 *ra = p.qr + (rA * H + h) * DR, *rb = p.qr + (rB * H + h) * DR;
    const __nv_bfloat16 *wa = p.v + (rA * H + h) * DH, *wb = p.v + (rB * H + h) * DH;
    const __nv_bfloat16 *oa = p.dout + (rA * H + h) * DH, *ob = p.dout + (rB * H + h) * DH;
    uint32_t qo[6][4], oo[4][4];
    float sA = 0.f, sB = 0.f, pdA = 0.f, pdB = 0.f;
#pragma unroll
    for (int kk = 0; kk < 6; ++kk) {
      const int c0 = 16 * kk + 2 * q, c1 = c0 + 8;
      kf[kk][0] = va ? at96(ka, kra, c0) : 0u;
      kf[kk][1] = vb ? at96(kb_, krb, c0) : 0u;
      kf[kk][2] = va ? at96(ka, kra, c1) : 0u;
      kf[kk][3] = vb ? at96(kb_, krb, c1) : 0u;
      qo[kk][0] = va ? at96(qa, ra, c0) : 0u;
      qo[kk][1] = vb ? at96(qb, rb, c0) : 0u;
      qo[kk][2] = va ? at96(qa, ra, c1) : 0u;
      qo[kk][3] = vb ? at96(qb, rb, c1) : 0u;
      sA += dot2(qo[kk][0], kf[kk][0]) + dot2(qo[kk][2], kf[kk][2]);
      sB += dot2(qo[kk][1], kf[kk][1]) + dot2(qo[kk][3], kf[kk][3]);
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int c0 = 16 * kk + 2 * q, c1 = c0 + 8;
      vf[kk][0] = va ? ld_u32(wa + c0) : 0u;
      vf[kk][1] = vb ? ld_u32(wb + c0) : 0u;
      vf[kk][2] = va ? ld_u32(wa + c1) : 0u;
      vf[kk][3] = vb ? ld_u32(wb + c1) : 0u;
      oo[kk][0] = va ? ld_u32(oa + c0) : 0u;
      oo[kk][1] = vb ? ld_u32(ob + c0) : 0u;
      oo[kk][2] = va ? ld_u32(oa + c1) : 0u;
      oo[kk][3] = vb ? ld_u32(ob + c1) : 0u;
      pdA += dot2(oo[kk][0], vf[kk][0]) + dot2(oo[kk][2], vf[kk][2]);
      pdB += dot2(oo[kk][1], vf[kk][1]) + dot2(oo[kk][3], vf[kk][3]);
    }
    sA = quad_sum(sA);
    sB = quad_sum(sB);
    pdA = quad_sum(pdA);
    pdB = quad_sum(pdB);
    // own column: the query at the column's own position, m == n
    const float lA = va ? p.ws_lse2[lbase + nA - 1] : 0.f, lB = vb ? p.ws_lse2[lbase + nB - 1] : 0.f;
    const float dA = va ? p.ws_delta[lbase + nA - 1] : 0.f, dB = vb ? p.ws_delta[lbase + nB - 1] : 0.f;
    const float pA = va ? exp2f(sA * sl2 - lA) : 0.f, pB = vb ? exp2f(sB * sl2 - lB) : 0.f;
    const float gA_ = pA * (pdA - dA), gB_ = pB * (pdB - dB);
#pragma unroll
    for (int kk = 0; kk < 6; ++kk) {
      const float2 x0 = bf2(qo[kk][0]), x1 = bf2(qo[kk][1]), x2 = bf2(qo[kk][2]), x3 = bf2(qo[kk][3]);
      dk[2 * kk][0] = gA_ * x0.x;
      dk[2 * kk][1] = gA_ * x0.y;
      dk[2 * kk][2] = gB_ * x1.x;
      dk[2 * kk][3] = gB_ * x1.y;
      dk[2 * kk + 1][0] = gA_ * x2.x;
      dk[2 * kk + 1][1] = gA_ * x2.y;
      dk[2 * kk + 1][2] = gB_ * x3.x;
      dk[2 * kk + 1][3] = gB_ * x3.y;
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const float2 x0 = bf2(oo[kk][0]), x1 = bf2(oo[kk][1]), x2 = bf2(oo[kk][2]), x3 = bf2(oo[kk][3]);
      dv[2 * kk][0] = pA * x0.x;
      dv[2 * kk][1] = pA * x0.y;
      dv[2 * kk][2] = pB * x1.x;
      dv[2 * kk][3] = pB * x1.y;
      dv[2 * kk + 1][0] = pA * x2.x;
      dv[2 * kk + 1][1] = pA * x2.y;
      dv[2 * kk + 1][2] = pB * x3.x;
      dv[2 * kk + 1][3] = pB * x3.y;
    }
  }

  const int lrow = lane & 7, lsel = lane >> 3;
  for (int qt = 0; qt < nqt; ++qt) {
    const int buf = qt & 1;
    float nl = 0.f, nd = 0.f;  // the next tile's lse2 and Delta, stored after this tile's work
    if (qt + 1 < nqt) {
      load_tile(qt + 1, buf ^ 1);
      const int m = m_start + (qt + 1) * TB + tid;
      if (tid < TB && m <= T) {
        nl = p.ws_lse2[lbase + m - 1];
        nd = p.ws_delta[lbase + m - 1];
      }
    }
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    const uint32_t qbase = smem_u32(Qt + buf * KTILE), obase = smem_u32(Ot + buf * VTILE);
    const float* L = Ls + buf * TB;
    const float* Dd = Ds + buf * TB;
    const int mt0 = m_start + qt * TB;
#pragma unroll
    for (int half = 0; half < 2; ++half) {  // queries 32 half .. 32 half + 31 of the tile
      float S[4][4], dP[4][4];              // transposed: rows are this warp's keys, columns queries
#pragma unroll
      for (int i = 0; i < 4; ++i) S[i][0] = S[i][1] = S[i][2] = S[i][3] = dP[i][0] = dP[i][1] = dP[i][2] = dP[i][3] = 0.f;
#pragma unroll
      for (int nl2 = 0; nl2 < 4; ++nl2) {
        const int nb = 4 * half + nl2;
#pragma unroll
        for (int kk2 = 0; kk2 < 3; ++kk2) {  // S^T = [k | k^R] [q | q^R]^T
          uint32_t b0, b1, b2, b3;
          ldsm_x4(qbase + (uint32_t)((8 * nb + lrow) * KS + 32 * kk2 + 8 * lsel) * 2, b0, b1, b2, b3);
          mma_bf16(S[nl2], kf[2 * kk2][0], kf[2 * kk2][1], kf[2 * kk2][2], kf[2 * kk2][3], b0, b1);
          mma_bf16(S[nl2], kf[2 * kk2 + 1][0], kf[2 * kk2 + 1][1], kf[2 * kk2 + 1][2], kf[2 * kk2 + 1][3], b2, b3);
        }
#pragma unroll
        for (int kk2 = 0; kk2 < 2; ++kk2) {  // dP^T = v dO^T
          uint32_t b0, b1, b2, b3;
          ldsm_x4(obase + (uint32_t)((8 * nb + lrow) * VS + 32 * kk2 + 8 * lsel) * 2, b0, b1, b2, b3);
          mma_bf16(dP[nl2], vf[2 * kk2][0], vf[2 * kk2][1], vf[2 * kk2][2], vf[2 * kk2][3], b0, b1);
          mma_bf16(dP[nl2], vf[2 * kk2 + 1][0], vf[2 * kk2 + 1][1], vf[2 * kk2 + 1][2], vf[2 * kk2 + 1][3], b2, b3);
        }
      }
      uint32_t pa[4][2], ds[4][2];
#pragma unroll
      for (int nl2 = 0; nl2 < 4; ++nl2) {
        const int j = 8 * (4 * half + nl2) + 2 * q;  // query index within the tile
        const int m = mt0 + j;
        const float L0 = L[j], L1 = L[j + 1], D0 = Dd[j], D1 = Dd[j + 1];
        // column n is seen by query m iff n < m (and m <= T)
        const float p0 = va && nA < m && m <= T ? exp2f(S[nl2][0] * sl2 - L0) : 0.f;
        const float p1 = va && nA < m + 1 && m + 1 <= T ? exp2f(S[nl2][1] * sl2 - L1) : 0.f;
        const float p2 = vb && nB < m && m <= T ? exp2f(S[nl2][2] * sl2 - L0) : 0.f;
        const float p3 = vb && nB < m + 1 && m + 1 <= T ? exp2f(S[nl2][3] * sl2 - L1) : 0.f;
        pa[nl2][0] = pack_bf16x2(p0, p1);
        pa[nl2][1] = pack_bf16x2(p2, p3);
        ds[nl2][0] = pack_bf16x2(p0 * (dP[nl2][0] - D0), p1 * (dP[nl2][1] - D1));
        ds[nl2][1] = pack_bf16x2(p2 * (dP[nl2][2] - D0), p3 * (dP[nl2][3] - D1));
      }
#pragma unroll
      for (int kl = 0; kl < 2; ++kl) {
        const int qrow = 32 * half + 16 * kl + lrow + 8 * (lsel & 1);
        // dv [16 x 64] += P^T [16 x 32 queries] dO [32 queries x 64]
        {
          const uint32_t a0 = pa[2 * kl][0], a1 = pa[2 * kl][1], a2 = pa[2 * kl + 1][0], a3 = pa[2 * kl + 1][1];
#pragma unroll
          for (int nb2 = 0; nb2 < 4; ++nb2) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(obase + (uint32_t)(qrow * VS + 16 * nb2 + 8 * (lsel >> 1)) * 2, b0, b1, b2, b3);
            mma_bf16(dv[2 * nb2], a0, a1, a2, a3, b0, b1);
            mma_bf16(dv[2 * nb2 + 1], a0, a1, a2, a3, b2, b3);
          }
        }
        // [dk | dk^R] [16 x 96] += dS^T [16 x 32 queries] [q | q^R] [32 queries x 96]
        {
          const uint32_t a0 = ds[2 * kl][0], a1 = ds[2 * kl][1], a2 = ds[2 * kl + 1][0], a3 = ds[2 * kl + 1][1];
#pragma unroll
          for (int nb2 = 0; nb2 < 6; ++nb2) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(qbase + (uint32_t)(qrow * KS + 16 * nb2 + 8 * (lsel >> 1)) * 2, b0, b1, b2, b3);
            mma_bf16(dk[2 * nb2], a0, a1, a2, a3, b0, b1);
            mma_bf16(dk[2 * nb2 + 1], a0, a1, a2, a3, b2, b3);
          }
        }
      }
    }
    __syncthreads();  // this buffer's tiles are refilled two iterations on; the other's scalars now
    if (qt + 1 < nqt && tid < TB) {
      Ls[(buf ^ 1) * TB + tid] = nl;
      Ds[(buf ^ 1) * TB + tid] = nd;
    }
  }
  cp_wait<0>();

#pragma unroll
  for (int nb = 0; nb < 12; ++nb) {
    const int c = 8 * nb + 2 * q;
    if (c < DH) {
      if (va) *reinterpret_cast<uint32_t*>(p.dk + (rA * H + h) * DH + c) = pack_bf16x2(dk[nb][0] * sc, dk[nb][1] * sc);
      if (vb) *reinterpret_cast<uint32_t*>(p.dk + (rB * H + h) * DH + c) = pack_bf16x2(dk[nb][2] * sc, dk[nb][3] * sc);
    } else {
      if (va) *reinterpret_cast<float2*>(p.ws_dkrh + (rA * H + h) * DR + (c - DH)) = make_float2(dk[nb][0] * sc, dk[nb][1] * sc);
      if (vb) *reinterpret_cast<float2*>(p.ws_dkrh + (rB * H + h) * DR + (c - DH)) = make_float2(dk[nb][2] * sc, dk[nb][3] * sc);
    }
  }
#pragma unroll
  for (int nb = 0; nb < 8; ++nb) {
    const int c = 8 * nb + 2 * q;
    if (va) *reinterpret_cast<uint32_t*>(p.dv + (rA * H + h) * DH + c) = pack_bf16x2(dv[nb][0], dv[nb][1]);
    if (vb) *reinterpret_cast<uint32_t*>(p.dv + (rB * H + h) * DH + c) = pack_bf16x2(dv[nb][2], dv[nb][3]);
  }
}

// dk^R [b, t, :] = sum over heads of the per-head RoPE key gradients (fixed order)
__global__ void __launch_bounds__(256) dkr_reduce_kernel(const float* dkrh, float* dkr, int64_t rows, int H) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * DR) return;
  const int64_t row = idx / DR;
  const int c = (int)(idx % DR);
  float acc = 0.f;
  for (int h = 0; h < H; ++h) acc += dkrh[(row * H + h) * DR + c];
  dkr[idx] = acc;
}

}  // namespace tbw

cudaError_t launch_attn_bwd(const BwdArgs& a, cudaStream_t st) {
  static uint64_t done_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(done_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(tbw::bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tbw::SMEM_DQ);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tbw::bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tbw::SMEM_DKV);
    if (e != cudaSuccess) return e;
    if (dev < 64) done_mask |= 1ull << dev;
  }
  const int64_t rows = (int64_t)a.B * a.T;
  const int64_t nth = rows * a.H;
  tbw::bwd_prep_kernel<<<(unsigned)((nth + 255) / 256), 256, 0, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t nqb = (a.T + tbw::TB - 1) / tbw::TB;
  tbw::bwd_dq_kernel<<<(unsigned)(nqb * a.B * a.H), tbw::NT, tbw::SMEM_DQ, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t nkb = (a.T / a.s + tbw::TB - 1) / tbw::TB;
  if (nkb > 0) {
    tbw::bwd_dkv_kernel<<<(unsigned)(nkb * a.B * a.H), tbw::NT, tbw::SMEM_DKV, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  tbw::dkr_reduce_kernel<<<(unsigned)((rows * tbw::DR + 255) / 256), 256, 0, st>>>(a.ws_dkrh, a.dkr, rows, a.H);
  return cudaGetLastError();
}

}  // namespace mtla
