// Masked prefill with explicit per-head keys and values (the un-absorbed
// form), bf16, d_h = 64, d_R = 32.
//
// What it computes (MTLA paper notes, "Key designs: stride-aware causal mask"
// and "decoupled RoPE with temporal compression"): for query m (1-based) of
// sequence b and head h, with q_h = x W_Q^h, K_h = C_hat'_latent W_K^h,
// V_h = C_hat'_latent W_V^h and the merged RoPE keys k_hat^R' (the last d_R
// channels of C_hat'; the training shortcut of "decoupled RoPE with temporal
// compression" passes the uncompressed K^R instead),
//   score_n = (q_h . K_h,n + q^R_h . k_hat^R'_n) / sqrt(d_h),
//   o_h = sum_{n visible} softmax(score)_n V_h,n
// over the columns n == m and n = g s (g < ceil(m/s)).  Equal to the absorbed
// forward's o_h W_V^h by associativity (abstract page, Figure 1), at 2 (d_h +
// d_R) + 2 d_h = 320 flop per visible pair instead of 1088.
//
// Design: a flash-attention kernel on warp-level tensor-core MMAs (m16n8k16,
// bf16 in, fp32 accumulators).  A CTA is 64 consecutive queries of one head
// (16 per warp, Q fragments held in registers); it streams key tiles of 64
// completed groups (K_h and k_hat^R' rows of n = g s, and V_h rows) through
// shared memory with cp.async, double-buffered.  The own column n = m is
// taken first, from a shared-memory copy of the CTA's own rows, and seeds the
// online softmax.  Tiles past the staircase are never visited; columns past a
// row's last visible group are masked.  CTAs run heaviest first.  The log of
// each softmax denominator is written on request, for the backward pass.
#include "kernels.cuh"

namespace mtla {
namespace pua {

constexpr int DH = 64, DR = 32, DK = DH + DR;   // score width 96
constexpr int QB = 64;                          // queries per CTA
constexpr int KB = 64;                          // groups per key tile
constexpr int NW = 4, NT = 32 * NW;
constexpr int KS = DK + 8;                      // padded row stride of K rows (elements): conflict-free ldmatrix
constexpr int VS = DH + 8;                      // padded row stride of V rows
constexpr int KTILE = KB * KS, VTILE = KB * VS; // elements
constexpr int SMEM_ELEMS = 2 * (KTILE + VTILE) + QB * KS + QB * VS;
constexpr size_t SMEM = (size_t)SMEM_ELEMS * 2;

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g, bool valid) {
  // a chunk that is not valid is filled with zeros (src-size 0)
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr), "l"(g), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ uint32_t ld_u32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }

__global__ void __launch_bounds__(NT) prefill_unabs_kernel(const UnabsArgs p) {
  extern __shared__ __align__(16) __nv_bfloat16 smu[];
  __nv_bfloat16* Kt = smu;                       // [2][KB][KS]
  __nv_bfloat16* Vt = Kt + 2 * KTILE;            // [2][KB][VS]
  __nv_bfloat16* Ko = Vt + 2 * VTILE;            // [QB][KS] own rows' keys
  __nv_bfloat16* Vo = Ko + QB * KS;              // [QB][VS] own rows' values
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int T = p.T, H = p.H, s = p.s;
  const int nqb = (T + QB - 1) / QB;
  // heaviest first: the last query blocks of every (sequence, head) come first
  const int qb = nqb - 1 - (int)(blockIdx.x / (p.B * H));
  const int bh = (int)(blockIdx.x % (p.B * H));
  const int b = bh / H, h = bh % H;
  const int m0 = qb * QB + 1;                    // first query (1-based)
  const int m_last = m0 + QB - 1 < T ? m0 + QB - 1 : T;
  const int vis_max = (int)group_of(m_last, s) - 1;  // completed groups the last query sees
  const int nkt = (vis_max + KB - 1) / KB;
  const int64_t row0 = (int64_t)b * T;           // first position of the sequence
  const int n_groups = T / s;                    // completed groups of the prompt

  asm volatile("griddepcontrol.wait;" ::: "memory");

  // key tile kt: rows of groups kt KB .. + KB - 1 (column n = (g + 1) s)
  auto load_tile = [&](int kt, int buf) {
    const uint32_t kb = smem_u32(Kt + buf * KTILE), vb = smem_u32(Vt + buf * VTILE);
    for (int i = tid; i < KB * 20; i += NT) {
      const int r = i / 20, c = i % 20;
      const int grp = kt * KB + r;
      const bool valid = grp < n_groups;
      const int64_t pos = row0 + (valid ? (int64_t)(grp + 1) * s - 1 : 0);  // column n; a row of the sequence even when not read
      if (c < 8) {
        cp_async16(kb + (uint32_t)(r * KS + c * 8) * 2, p.k + (pos * H + h) * DH + c * 8, valid);
      } else if (c < 12) {
        cp_async16(kb + (uint32_t)(r * KS + DH + (c - 8) * 8) * 2, p.kr + pos * p.kr_stride + (c - 8) * 8, valid);
      } else {
        cp_async16(vb + (uint32_t)(r * VS + (c - 12) * 8) * 2, p.v + (pos * H + h) * DH + (c - 12) * 8, valid);
      }
    }
  };
  // the CTA's own rows (column n = m of each query)
  {
    const uint32_t kb = smem_u32(Ko), vb = smem_u32(Vo);
    for (int i = tid; i < QB * 20; i += NT) {
      const int r = i / 20, c = i % 20;
      const bool valid = m0 + r <= T;
      const int64_t pos = row0 + (valid ? m0 - 1 + r : 0);
      if (c < 8) cp_async16(kb + (uint32_t)(r * KS + c * 8) * 2, p.k + (pos * H + h) * DH + c * 8, valid);
      else if (c < 12)
        cp_async16(kb + (uint32_t)(r * KS + DH + (c - 8) * 8) * 2, p.kr + pos * p.kr_stride + (c - 8) * 8, valid);
      else cp_async16(vb + (uint32_t)(r * VS + (c - 12) * 8) * 2, p.v + (pos * H + h) * DH + (c - 12) * 8, valid);
    }
    cp_commit();
  }
  if (nkt > 0) load_tile(0, 0);
  cp_commit();

  // Q fragments (A of m16n8k16, row-major): rows r0 = 16 warp + g and r0 + 8,
  // columns 16 kk + 2q (+1) and 16 kk + 8 + 2q (+1) of [q_h | q^R_h]
  const int r0 = 16 * warp + g;
  const int ma = m0 + r0, mb = ma + 8;            // this thread's two queries (1-based)
  const bool va = ma <= T, vbq = mb <= T;
  uint32_t qf[6][4];
  {
    const __nv_bfloat16* qa = p.q + ((row0 + (va ? ma - 1 : 0)) * H + h) * DH;
    const __nv_bfloat16* qb_ = p.q + ((row0 + (vbq ? mb - 1 : 0)) * H + h) * DH;
    const __nv_bfloat16* ra = p.qr + ((row0 + (va ? ma - 1 : 0)) * H + h) * DR;
    const __nv_bfloat16* rb = p.qr + ((row0 + (vbq ? mb - 1 : 0)) * H + h) * DR;
#pragma unroll
    for (int kk = 0; kk < 6; ++kk) {
      const int c0 = 16 * kk + 2 * q, c1 = c0 + 8;
      auto at = [&](const __nv_bfloat16* qq, const __nv_bfloat16* rr, int c, bool v) -> uint32_t {
        if (!v) return 0u;
        return c < DH ? ld_u32(qq + c) : ld_u32(rr + (c - DH));
      };
      qf[kk][0] = at(qa, ra, c0, va);
      qf[kk][1] = at(qb_, rb, c0, vbq);
      qf[kk][2] = at(qa, ra, c1, va);
      qf[kk][3] = at(qb_, rb, c1, vbq);
    }
  }
  const float sl2 = p.scale_log2;
  float O[8][4];
#pragma unroll
  for (int nb = 0; nb < 8; ++nb) O[nb][0] = O[nb][1] = O[nb][2] = O[nb][3] = 0.f;

  // ---- the own column: q . k_own over this thread's 24 columns per row, summed over the row's 4 threads
  cp_wait<1>();
  __syncthreads();
  float mA, mB, lA, lB;
  {
    float da = 0.f, db = 0.f;
#pragma unroll
    for (int kk = 0; kk < 6; ++kk) {
      const int c0 = 16 * kk + 2 * q, c1 = c0 + 8;
      const __nv_bfloat16* ka = Ko + r0 * KS;
      const __nv_bfloat16* kb2 = Ko + (r0 + 8) * KS;
      const float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qf[kk][0]));
      const float2 b0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qf[kk][1]));
      const float2 a1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qf[kk][2]));
      const float2 b1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qf[kk][3]));
      const float2 ka0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(ka + c0));
      const float2 ka1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(ka + c1));
      const float2 kb0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kb2 + c0));
      const float2 kb1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kb2 + c1));
      da += a0.x * ka0.x + a0.y * ka0.y + a1.x * ka1.x + a1.y * ka1.y;
      db += b0.x * kb0.x + b0.y * kb0.y + b1.x * kb1.x + b1.y * kb1.y;
    }
    da += __shfl_xor_sync(0xffffffffu, da, 1);
    da += __shfl_xor_sync(0xffffffffu, da, 2);
    db += __shfl_xor_sync(0xffffffffu, db, 1);
    db += __shfl_xor_sync(0xffffffffu, db, 2);
    mA = da * sl2;
    mB = db * sl2;
    // p_own = exp2(own - max) = 1 with the own score as the first max; the
    // row's four threads keep partial sums (added at the end), so one of
    // them holds it
    lA = q == 0 ? 1.f : 0.f;
    lB = q == 0 ? 1.f : 0.f;
    const __nv_bfloat16* vA = Vo + r0 * VS;
    const __nv_bfloat16* vB = Vo + (r0 + 8) * VS;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vA + nb * 8 + 2 * q));
      const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vB + nb * 8 + 2 * q));
      O[nb][0] = x.x;
      O[nb][1] = x.y;
      O[nb][2] = y.x;
      O[nb][3] = y.y;
    }
  }
  const int visA = va ? (int)group_of(ma, s) - 1 : 0;  // completed groups each query sees
  const int visB = vbq ? (int)group_of(mb, s) - 1 : 0;

  // ldmatrix lane addressing: K rows (B of the score MMA, non-transposed) and
  // V rows (B of the value MMA, transposed)
  const int lrow = lane & 7, lsel = lane >> 3;
  for (int kt = 0; kt < nkt; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nkt) load_tile(kt + 1, buf ^ 1);
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    const uint32_t kbase = smem_u32(Kt + buf * KTILE), vbase = smem_u32(Vt + buf * VTILE);
    // S [16 x 64] = Q [16 x 96] K^T: 8 n-blocks of 8 keys
    float S[8][4];
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) S[nb][0] = S[nb][1] = S[nb][2] = S[nb][3] = 0.f;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int kk2 = 0; kk2 < 3; ++kk2) {
        // x4: k-steps 2 kk2 and 2 kk2 + 1 (b0, b1 each) for keys 8 nb .. 8 nb + 7
        uint32_t b0, b1, b2, b3;
        const uint32_t addr = kbase + (uint32_t)((8 * nb + lrow) * KS + 32 * kk2 + 8 * lsel) * 2;
        ldsm_x4(addr, b0, b1, b2, b3);
        mma_bf16(S[nb], qf[2 * kk2][0], qf[2 * kk2][1], qf[2 * kk2][2], qf[2 * kk2][3], b0, b1);
        mma_bf16(S[nb], qf[2 * kk2 + 1][0], qf[2 * kk2 + 1][1], qf[2 * kk2 + 1][2], qf[2 * kk2 + 1][3], b2, b3);
      }
    }
    // mask and scale: group index of column j of n-block nb is kt KB + 8 nb + 2q (+1)
    float mxA = -INFINITY, mxB = -INFINITY;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      const int gi = kt * KB + 8 * nb + 2 * q;
      S[nb][0] = gi < visA ? S[nb][0] * sl2 : -INFINITY;
      S[nb][1] = gi + 1 < visA ? S[nb][1] * sl2 : -INFINITY;
      S[nb][2] = gi < visB ? S[nb][2] * sl2 : -INFINITY;
      S[nb][3] = gi + 1 < visB ? S[nb][3] * sl2 : -INFINITY;
      mxA = fmaxf(mxA, fmaxf(S[nb][0], S[nb][1]));
      mxB = fmaxf(mxB, fmaxf(S[nb][2], S[nb][3]));
    }
    mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, 1));
    mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, 2));
    mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, 1));
    mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, 2));
    const float nA = fmaxf(mA, mxA), nB = fmaxf(mB, mxB);  // finite: the own column seeded the max
    const float aA = exp2f(mA - nA), aB = exp2f(mB - nB);
    mA = nA;
    mB = nB;
    float sA = 0.f, sB = 0.f;
    uint32_t pf[8][2];
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      const float p0 = exp2f(S[nb][0] - nA), p1 = exp2f(S[nb][1] - nA);
      const float p2 = exp2f(S[nb][2] - nB), p3 = exp2f(S[nb][3] - nB);
      sA += p0 + p1;
      sB += p2 + p3;
      pf[nb][0] = pack_bf16x2(p0, p1);
      pf[nb][1] = pack_bf16x2(p2, p3);
    }
    lA = lA * aA + sA;
    lB = lB * aB + sB;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      O[nb][0] *= aA;
      O[nb][1] *= aA;
      O[nb][2] *= aB;
      O[nb][3] *= aB;
    }
    // O [16 x 64] += P [16 x 64 keys] V [64 keys x 64]: A from the score
    // fragments of n-blocks 2 kk and 2 kk + 1, B = V^T by transposed ldmatrix
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint32_t a0 = pf[2 * kk][0], a1 = pf[2 * kk][1], a2 = pf[2 * kk + 1][0], a3 = pf[2 * kk + 1][1];
#pragma unroll
      for (int nb2 = 0; nb2 < 4; ++nb2) {
        // x4 trans: dims 16 nb2 .. + 15 (two n-blocks) for keys 16 kk .. + 15
        uint32_t b0, b1, b2, b3;
        const uint32_t addr = vbase + (uint32_t)((16 * kk + lrow + 8 * (lsel & 1)) * VS + 16 * nb2 + 8 * (lsel >> 1)) * 2;
        ldsm_x4_t(addr, b0, b1, b2, b3);
        mma_bf16(O[2 * nb2], a0, a1, a2, a3, b0, b1);
        mma_bf16(O[2 * nb2 + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();  // the buffer is refilled by the next iteration's prefetch
  }
  cp_wait<0>();

  // ---- normalise and store
  lA += __shfl_xor_sync(0xffffffffu, lA, 1);
  lA += __shfl_xor_sync(0xffffffffu, lA, 2);
  lB += __shfl_xor_sync(0xffffffffu, lB, 1);
  lB += __shfl_xor_sync(0xffffffffu, lB, 2);
  const float iA = 1.f / lA, iB = 1.f / lB;
  if (p.lse && q == 0) {
    // natural log of the denominator: the running max and sum are in log2 units of the scaled score
    if (va) p.lse[(row0 + ma - 1) * H + h] = (mA + log2f(lA)) * 0.69314718055994531f;
    if (vbq) p.lse[(row0 + mb - 1) * H + h] = (mB + log2f(lB)) * 0.69314718055994531f;
  }
  __nv_bfloat16* oA = p.out + ((row0 + ma - 1) * H + h) * DH;
  __nv_bfloat16* oB = p.out + ((row0 + mb - 1) * H + h) * DH;
#pragma unroll
  for (int nb = 0; nb < 8; ++nb) {
    if (va) *reinterpret_cast<uint32_t*>(oA + nb * 8 + 2 * q) = pack_bf16x2(O[nb][0] * iA, O[nb][1] * iA);
    if (vbq) *reinterpret_cast<uint32_t*>(oB + nb * 8 + 2 * q) = pack_bf16x2(O[nb][2] * iB, O[nb][3] * iB);
  }
}

}  // namespace pua

cudaError_t launch_prefill_unabs(const UnabsArgs& a, cudaStream_t st) {
  static uint64_t done_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(done_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(pua::prefill_unabs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pua::SMEM);
    if (e != cudaSuccess) return e;
    if (dev < 64) done_mask |= 1ull << dev;
  }
  const int64_t nqb = (a.T + pua::QB - 1) / pua::QB;
  pua::prefill_unabs_kernel<<<(unsigned)(nqb * a.B * a.H), pua::NT, pua::SMEM, st>>>(a);
  return cudaGetLastError();
}

}  // namespace mtla
