// Backward pass of the masked attention with explicit keys and values and the
// uncompressed RoPE keys (the training shortcut of the MTLA paper notes, "Key
// designs: decoupled RoPE with temporal compression", under the stride-aware
// causal mask of "Key designs: stride-aware causal mask") on the tensor cores:
// tcgen05 + TMEM, bf16, d_h = 64, d_R = 32.
//
// For query m, head h and visible column n (n == m, or n = g s < m), with the
// forward's lse and Delta_m = dO_m . O_m:
//   P = exp(score - lse),  dP = dO . v_n,  dS = P (dP - Delta_m),
//   dq_m = sum_n dS [k | k^R]_n / sqrt(d_h),
//   d[k | k^R]_n = sum_m dS [q | q^R]_m / sqrt(d_h),  dv_n = sum_m P dO_m.
// The lse fixes every probability, so neither kernel keeps a running max.
//
// dq kernel: an M tile is 128 queries of one (sequence, head).  Per tile of
// 64 group columns, S = Q K^T (K 96) and dP = dO V^T (K 64) go to TMEM; eight
// gradient warps turn them into bf16 dS in TMEM; dq += dS K (K 64 keys, N 96)
// takes dS as the TMEM A operand and the key tile as the MN-major B operand.
// A dot warp takes the own column (n == m), and writes the key and value
// gradients of the rows no later query sees (n mod s != 0); four epilogue
// warps fold the own column into dq and store it.
//
// dk/dv kernel: a work item is 128 group columns of one (sequence, head),
// their keys, values and own-position rows resident in shared memory.  Per
// tile of 64 queries (aligned to 64 positions), S^T = K Q^T and dP^T = V dO^T
// go to TMEM with the keys as rows; the gradient warps write bf16 P^T and dS^T
// back over them; dv += P^T dO and [dk | dk^R] += dS^T [q | q^R] take them as
// TMEM A operands and the query tile as the MN-major B operand.  The epilogue
// adds the own column's terms and stores dk, dv and the per-head dk^R.
#include "kernels.cuh"

namespace mtla {
namespace bwt {

constexpr int DH = 64, DR = 32;
constexpr int SMW = 8, EPW = 4;
constexpr int NT = 32 * (SMW + 4 + EPW);
constexpr int TMA_WARP = SMW, SMMA_WARP = SMW + 1, GMMA_WARP = SMW + 2, DOT_WARP = SMW + 3, EPI_WARP0 = SMW + 4;
static_assert(EPI_WARP0 % 4 == 0, "epilogue warp e reads TMEM lane quarter e");
constexpr uint32_t TMEM_COLS = 512;
constexpr int NSB = 2;  // S / dP buffers in TMEM

// 16-byte chunk ch of row `row` inside a plane-layout tile whose planes hold
// `rows` rows: plane ch / 4, 64-byte swizzle phase (row / 2) mod 4
__device__ __forceinline__ uint32_t plane_off(int rows, int row, int ch) {
  return (uint32_t)(ch >> 2) * (uint32_t)(rows * 64) + (uint32_t)row * 64u +
         ((((uint32_t)ch & 3u) ^ (((uint32_t)row >> 1) & 3u)) << 4);
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
      "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}
__device__ __forceinline__ int tile_index(int r, int x, int G) { return r * G + ((r & 1) ? G - 1 - x : x); }
// dot product of 8 bf16 pairs held in two uint4
__device__ __forceinline__ float dot8(const uint32_t (&a)[4], const uint32_t (&b)[4], float acc) {
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a[e]));
    const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b[e]));
    acc = fmaf(x.x, y.x, acc);
    acc = fmaf(x.y, y.y, acc);
  }
  return acc;
}
__device__ __forceinline__ void lds4(uint32_t addr, uint32_t (&v)[4]) {
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]) : "r"(addr));
}

// ===========================================================================
// dq kernel
// ===========================================================================
namespace dq {
constexpr int BM = 128, BN = 64;
constexpr int QPL = BM * 64, KPL = BN * 64;
constexpr int QTILE = 5 * QPL;   // [q | q^R] (3 planes), dO (2 planes)
constexpr int OWNB = 5 * QPL;    // own rows: k (2), k^R (1), v (2)
constexpr int STAGE = 5 * KPL;   // key tile: k (2), k^R (1), v (2)
constexpr int KS = 3;
constexpr uint32_t S_COL = 0, DP_COL = 128, DS_COL = 256, DQ_COL = 320;  // S, dP: 2 x 64; dS: 2 x 32; dq: 96
constexpr uint32_t IDESC_S = umma_idesc_bf16(BM, BN, false, false);
constexpr uint32_t IDESC_Q = umma_idesc_bf16(BM, 96, false, true);
constexpr size_t OFF_Q = 0;
constexpr size_t OFF_OWN = OFF_Q + QTILE;
constexpr size_t OFF_K = OFF_OWN + 2 * OWNB;
constexpr size_t OFF_XCH = OFF_K + (size_t)KS * STAGE;    // own-column dS and P per parity
constexpr size_t OFF_BAR = OFF_XCH + 4 * BM * 4;
constexpr int NBAR = 2 + 8 + 2 * KS + 3 * NSB + 3;
constexpr size_t OFF_TMEM = OFF_BAR + NBAR * 8;
constexpr size_t SMEM_USED = OFF_TMEM + 16;
static_assert(OFF_OWN % 1024 == 0 && OFF_K % 1024 == 0 && STAGE % 1024 == 0, "tile bases must be 1024-aligned");
static_assert(SMEM_USED + 1024 <= 232448, "one block's shared memory (227 KB)");

struct Tile {
  int b, h, m0, nkt;
};
__device__ __forceinline__ Tile tile_of(const TrainBwdTc& p, int o) {
  const int per_seq = (p.T + BM - 1) / BM;
  const int bh = o % (p.B * p.H);
  Tile t;
  t.b = bh / p.H;
  t.h = bh % p.H;
  t.m0 = (per_seq - 1 - o / (p.B * p.H)) * BM + 1;
  const int m_last = t.m0 + BM - 1 < p.T ? t.m0 + BM - 1 : p.T;
  t.nkt = ((int)group_of(m_last, p.s) - 1 + BN - 1) / BN;
  return t;
}

__global__ void __launch_bounds__(NT, 1) bwd_dq_tc_kernel(const __grid_constant__ TrainBwdMaps mp,
                                                          const TrainBwdTc p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* const q_full = bar + 0;
  uint64_t* const q_empty = bar + 1;           // the tile's last S / dP MMAs + the dot warp
  uint64_t* const own_full = bar + 2;          // [2]
  uint64_t* const own_empty = bar + 4;         // [2] the epilogue is done with them
  uint64_t* const dot_full = bar + 6;          // [2] own-column terms written
  uint64_t* const dot_empty = bar + 8;         // [2] the epilogue has read them
  uint64_t* const k_full = bar + 10;           // [KS]
  uint64_t* const k_empty = bar + 10 + KS;     // [KS] the tile's dq MMA has read it
  uint64_t* const s_full = bar + 10 + 2 * KS;  // [NSB] S and dP in TMEM
  uint64_t* const ds_full = s_full + NSB;      // [NSB] dS written (SMW arrivals)
  uint64_t* const ds_empty = s_full + 2 * NSB; // [NSB] the dq MMA has read dS (and so S, dP are free)
  uint64_t* const dq_full = s_full + 3 * NSB;
  uint64_t* const dq_empty = dq_full + 1;
  uint64_t* const mma_done = dq_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
  float* xds = reinterpret_cast<float*>(sm + OFF_XCH);           // [2][BM] own-column dS
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 2);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&own_full[b], 1);
      mbar_init(&own_empty[b], EPW);
      mbar_init(&dot_full[b], 1);
      mbar_init(&dot_empty[b], EPW);
    }
    for (int i = 0; i < KS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < NSB; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&ds_full[i], SMW);
      mbar_init(&ds_empty[i], 1);
    }
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, EPW);
    mbar_init(mma_done, 2);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == TMA_WARP && lane == 0) {
    prefetch_tmap(&mp.q128);
    prefetch_tmap(&mp.qr128);
    prefetch_tmap(&mp.do128);
    prefetch_tmap(&mp.k128);
    prefetch_tmap(&mp.kr128);
    prefetch_tmap(&mp.v128);
    prefetch_tmap(&mp.k_g64);
    prefetch_tmap(&mp.kr_g64);
    prefetch_tmap(&mp.v_g64);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");  // Delta and lse2 come from the previous launch
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t sQ = smem_u32(sm + OFF_Q);
  const uint32_t sOwn = smem_u32(sm + OFF_OWN);
  const uint32_t sK = smem_u32(sm + OFF_K);
  const int G = gridDim.x;
  const int n_tiles = p.B * p.H * ((p.T + BM - 1) / BM);
  const float sl2 = p.scale_log2, sc = p.scale;
  bool ok = true;

  if (warp == TMA_WARP) {
    if (lane == 0) {
      uint32_t tc = 0, kc = 0, q_issued = 0;
      for (int o; (o = tile_index(tc, blockIdx.x, G)) < n_tiles && ok; ++tc) {
        const Tile t = tile_of(p, o);
        const int row0 = t.b * p.T + (t.m0 - 1);
        const int sb2 = tc & 1;
        if (tc > 0 && !mbar_wait(q_empty, (tc - 1) & 1)) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, QTILE);
        tma_load_4d(sm + OFF_Q, &mp.q128, 0, t.h, row0, 0, q_full);
        tma_load_3d(sm + OFF_Q + 2 * QPL, &mp.qr128, 0, t.h, row0, q_full);
        tma_load_4d(sm + OFF_Q + 3 * QPL, &mp.do128, 0, t.h, row0, 0, q_full);
        q_issued = tc + 1;
        if (tc >= 2 && !mbar_wait(&own_empty[sb2], ((tc >> 1) & 1) ^ 1)) { ok = false; break; }
        uint8_t* ob = sm + OFF_OWN + (size_t)sb2 * OWNB;
        mbar_arrive_expect_tx(&own_full[sb2], OWNB);
        tma_load_4d(ob, &mp.k128, 0, t.h, row0, 0, &own_full[sb2]);
        tma_load_2d(ob + 2 * QPL, &mp.kr128, 0, row0, &own_full[sb2]);
        tma_load_4d(ob + 3 * QPL, &mp.v128, 0, t.h, row0, 0, &own_full[sb2]);
        for (int kt = 0; kt < t.nkt; ++kt, ++kc) {
          const int st = kc % KS;
          if (kc >= KS && !mbar_wait(&k_empty[st], ((kc / KS) & 1) ^ 1)) { ok = false; break; }
          uint8_t* kb = sm + OFF_K + (size_t)st * STAGE;
          mbar_arrive_expect_tx(&k_full[st], STAGE);
          tma_load_5d(kb, &mp.k_g64, 0, t.h, kt * BN, t.b, 0, &k_full[st]);
          tma_load_3d(kb + 2 * KPL, &mp.kr_g64, 0, kt * BN, t.b, &k_full[st]);
          tma_load_5d(kb + 3 * KPL, &mp.v_g64, 0, t.h, kt * BN, t.b, 0, &k_full[st]);
        }
      }
      if (!ok) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
      if (q_issued) mbar_wait(q_full, (q_issued - 1) & 1);
      for (uint32_t u = q_issued > 2 ? q_issued - 2 : 0; u < q_issued; ++u) mbar_wait(&own_full[u & 1], (u >> 1) & 1);
      for (uint32_t j = kc > (uint32_t)KS ? kc - KS : 0; j < kc; ++j) mbar_wait(&k_full[j % KS], (j / KS) & 1);
    }
  } else if (warp == DOT_WARP) {
    // own column (n == m) per row: s_own = [q | q^R] . [k | k^R], dp_own = dO . v,
    // P_own, dS_own; the key and value gradients of rows no later query sees
    for (uint32_t tc = 0;; ++tc) {
      const int o = tile_index(tc, blockIdx.x, G);
      if (o >= n_tiles) break;
      const Tile t = tile_of(p, o);
      const int sb2 = tc & 1;
      if (ok && !warp_wait(q_full, tc & 1)) ok = false;
      if (ok && !warp_wait(&own_full[sb2], (tc >> 1) & 1)) ok = false;
      if (ok && tc >= 2 && !warp_wait(&dot_empty[sb2], ((tc >> 1) & 1) ^ 1)) ok = false;
      const uint32_t ownb = sOwn + sb2 * OWNB;
      const int64_t lbase = ((int64_t)t.b * p.H + t.h) * p.Tp;
#pragma unroll 1
      for (int r = 0; r < BM / 32; ++r) {
        const int i = r * 32 + lane;
        const int m = t.m0 + i;
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int ch = 0; ch < 12; ++ch) {
          uint32_t a[4], b[4];
          lds4(sQ + plane_off(BM, i, ch), a);
          lds4(ownb + plane_off(BM, i, ch), b);
          s = dot8(a, b, s);
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t a[4], b[4];
          lds4(sQ + 3 * QPL + plane_off(BM, i, ch), a);
          lds4(ownb + 3 * QPL + plane_off(BM, i, ch), b);
          dp = dot8(a, b, dp);
        }
        const bool valid = m <= p.T;
        const float pown = valid ? ex2_approx(s * sl2 - p.lse2[lbase + m - 1]) : 0.f;
        const float ds = valid ? pown * (dp - p.delta[lbase + m - 1]) : 0.f;
        xds[sb2 * BM + i] = ds;
        if (valid && (m % p.s) != 0) {
          // no later query sees column m: its gradients are the own column's terms
          const size_t row = ((size_t)t.b * p.T + (m - 1)) * p.H + t.h;
          uint4* dk = reinterpret_cast<uint4*>(p.dk + row * DH);
          uint4* dv = reinterpret_cast<uint4*>(p.dv + row * DH);
          float4* dkr = reinterpret_cast<float4*>(p.dkrh + row * DR);
#pragma unroll
          for (int ch = 0; ch < 12; ++ch) {
            uint32_t a[4], w[4];
            lds4(sQ + plane_off(BM, i, ch), a);
            if (ch < 8) {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a[e]));
                w[e] = pack_bf16x2(ds * sc * x.x, ds * sc * x.y);
              }
              dk[ch] = make_uint4(w[0], w[1], w[2], w[3]);
            } else {
              float f[8];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a[e]));
                f[2 * e] = ds * sc * x.x;
                f[2 * e + 1] = ds * sc * x.y;
              }
              dkr[2 * (ch - 8)] = make_float4(f[0], f[1], f[2], f[3]);
              dkr[2 * (ch - 8) + 1] = make_float4(f[4], f[5], f[6], f[7]);
            }
          }
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            uint32_t a[4], w[4];
            lds4(sQ + 3 * QPL + plane_off(BM, i, ch), a);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a[e]));
              w[e] = pack_bf16x2(pown * x.x, pown * x.y);
            }
            dv[ch] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(q_empty);
        mbar_arrive(&dot_full[sb2]);
      }
    }
    if (!ok && lane == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
  } else if (warp == SMMA_WARP || warp == GMMA_WARP) {
    const bool scores = warp == SMMA_WARP;
    const uint64_t dq0 = umma_desc(sQ, 16, 512, 4);             // [q | q^R] planes, K-major
    const uint64_t do0 = umma_desc(sQ + 3 * QPL, 16, 512, 4);   // dO planes, K-major
    const uint64_t dk0 = umma_desc(sK, 16, 512, 4);             // key tile planes, K-major
    const uint64_t dv0 = umma_desc(sK + 3 * KPL, 16, 512, 4);   // value planes, K-major (rows = keys)
    const uint64_t dkm = umma_desc(sK, KPL, 512, 4);            // key tile as the MN-major B of dq += dS K
    uint32_t tc = 0, kc = 0;
    for (int o; (o = tile_index(tc, blockIdx.x, G)) < n_tiles && ok; ++tc) {
      const Tile t = tile_of(p, o);
      if (scores) {
        if (!warp_wait(q_full, tc & 1)) { ok = false; break; }
        for (int kt = 0; kt < t.nkt && ok; ++kt) {
          const uint32_t j = kc + kt;
          const int st = j % KS, sb = j % NSB;
          if (!warp_wait(&k_full[st], (j / KS) & 1)) { ok = false; break; }
          if (j >= NSB && !warp_wait(&ds_empty[sb], ((j / NSB) & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 6; ++kk) {
              const uint64_t ad = dq0 + (uint64_t)(((kk >> 1) * QPL + (kk & 1) * 32) >> 4);
              const uint64_t bd = dk0 + (uint64_t)((st * STAGE + (kk >> 1) * KPL + (kk & 1) * 32) >> 4);
              umma_bf16(tmem + S_COL + 64 * sb, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = do0 + (uint64_t)(((kk >> 1) * QPL + (kk & 1) * 32) >> 4);
              const uint64_t bd = dv0 + (uint64_t)((st * STAGE + (kk >> 1) * KPL + (kk & 1) * 32) >> 4);
              umma_bf16(tmem + DP_COL + 64 * sb, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
            }
            umma_commit(&s_full[sb]);
            if (kt + 1 == t.nkt) umma_commit(q_empty);
          }
          __syncwarp();
        }
        if (t.nkt == 0) {
          if (elect_one()) umma_commit(q_empty);
          __syncwarp();
        }
      } else {
        for (int kt = 0; kt < t.nkt && ok; ++kt) {
          const uint32_t j = kc + kt;
          const int sb = j % NSB, st = j % KS;
          if (!warp_wait(&ds_full[sb], (j / NSB) & 1)) { ok = false; break; }
          if (kt == 0 && tc > 0 && !warp_wait(dq_empty, (tc - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
              const uint32_t pa = tmem + DS_COL + 32 * sb + 8 * kk;
              const uint64_t bd = dkm + (uint64_t)((st * STAGE + kk * 16 * 64) >> 4);
              umma_bf16_ts(tmem + DQ_COL, pa, bd, IDESC_Q, (kt > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&k_empty[st]);
            umma_commit(&ds_empty[sb]);
          }
          __syncwarp();
        }
        if (ok && t.nkt == 0 && tc > 0 && !warp_wait(dq_empty, (tc - 1) & 1)) ok = false;
        if (ok) {
          if (elect_one()) umma_commit(dq_full);
          __syncwarp();
        }
      }
      kc += t.nkt;
    }
    if (!ok && lane == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
    if (elect_one()) umma_commit(mma_done);
    __syncwarp();
    warp_wait(mma_done, 0);
  } else if (warp >= EPI_WARP0) {
    // dq = (sum over the group columns + dS_own [k | k^R]_m) / sqrt(d_h)
    const int qe = warp - EPI_WARP0;
    const int i = qe * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(qe * 32) << 16);
    for (uint32_t tc = 0;; ++tc) {
      const int o = tile_index(tc, blockIdx.x, G);
      if (o >= n_tiles) break;
      const Tile t = tile_of(p, o);
      const int sb2 = tc & 1;
      if (ok && !warp_wait(&dot_full[sb2], (tc >> 1) & 1)) ok = false;
      if (ok && !warp_wait(&own_full[sb2], (tc >> 1) & 1)) ok = false;
      const float ds = xds[sb2 * BM + i];
      __syncwarp();
      if (lane == 0) mbar_arrive(&dot_empty[sb2]);
      if (ok && !warp_wait(dq_full, tc & 1)) ok = false;
      tc_fence_after();
      const uint32_t ownb = sOwn + sb2 * OWNB;
      const int m = t.m0 + i;
      const size_t row = ((size_t)t.b * p.T + (m - 1)) * p.H + t.h;
      // 32 columns at a time: dq (two blocks), then dq^R
#pragma unroll 1
      for (int c2 = 0; c2 < 3; ++c2) {
        uint32_t acc[32];
        if (t.nkt > 0) {
          tmem_ld32(lane_base + DQ_COL + 32 * c2, acc);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[e] = 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t kv[4];
          lds4(ownb + plane_off(BM, i, 4 * c2 + c4), kv);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 k = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kv[e]));
            const int c = c4 * 8 + e * 2;
            w[c4 * 4 + e] = pack_bf16x2((__uint_as_float(acc[c]) + ds * k.x) * sc, (__uint_as_float(acc[c + 1]) + ds * k.y) * sc);
          }
        }
        if (m <= p.T) {
          uint4* dst = c2 < 2 ? reinterpret_cast<uint4*>(p.dq + row * DH + 32 * c2) : reinterpret_cast<uint4*>(p.dqr + row * DR);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) dst[c4] = make_uint4(w[4 * c4], w[4 * c4 + 1], w[4 * c4 + 2], w[4 * c4 + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(dq_empty);
        mbar_arrive(&own_empty[sb2]);
      }
    }
    if (!ok && lane == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
  } else {
    // gradient warps: warp w owns TMEM lane quarter w % 4 and half w / 4 of
    // each tile's 64 columns; dS = P (dP - Delta), bf16, into the dS columns
    const int qw = warp & 3, hf = warp >> 2;
    const int i = qw * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    uint32_t tc = 0, kc = 0;
    for (int o; (o = tile_index(tc, blockIdx.x, G)) < n_tiles; ++tc) {
      const Tile t = tile_of(p, o);
      const int m = t.m0 + i;
      const bool valid = m <= p.T;
      const int64_t lbase = ((int64_t)t.b * p.H + t.h) * p.Tp;
      const float L = valid ? p.lse2[lbase + m - 1] : 0.f;
      const float Dl = valid ? p.delta[lbase + m - 1] : 0.f;
      const int vis = valid ? (int)group_of(m, p.s) - 1 : 0;
      for (int kt = 0; kt < t.nkt; ++kt) {
        const uint32_t j = kc + kt;
        const int sb = j % NSB;
        if (ok && !warp_wait(&s_full[sb], (j / NSB) & 1)) ok = false;
        tc_fence_after();
        uint32_t sr[32], dr[32];
        tmem_ld32(lane_base + S_COL + 64 * sb + 32 * hf, sr);
        tmem_ld32(lane_base + DP_COL + 64 * sb + 32 * hf, dr);
        tmem_wait_ld();
        const int nvis = vis - kt * BN - 32 * hf;
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float p0 = c < nvis ? ex2_approx(__uint_as_float(sr[c]) * sl2 - L) : 0.f;
          const float p1 = c + 1 < nvis ? ex2_approx(__uint_as_float(sr[c + 1]) * sl2 - L) : 0.f;
          pk[c >> 1] = pack_bf16x2(p0 * (__uint_as_float(dr[c]) - Dl), p1 * (__uint_as_float(dr[c + 1]) - Dl));
        }
        tmem_st16(lane_base + DS_COL + 32 * sb + 16 * hf, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ds_full[sb]);
      }
      kc += t.nkt;
    }
    if (!ok && lane == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}
}  // namespace dq

// ===========================================================================
// dk / dv kernel
// ===========================================================================
namespace dkv {
constexpr int BK = 128, QT = 64;
constexpr int KPL = BK * 64;                 // one 128-row plane (8192)
constexpr int QPL = QT * 64;                 // one 64-row plane (4096)
constexpr int ITEM = 10 * KPL;               // keys (3), values (2), own [q | q^R] (3), own dO (2)
constexpr int QBYTES = 5 * QPL + 2 * QT * 4; // query tile: [q | q^R] (3), dO (2), lse2, Delta
constexpr int QSTAGE = (QBYTES + 1023) / 1024 * 1024;
constexpr int KS = 4;
constexpr uint32_t S_COL = 0, DP_COL = 128, DV_COL = 256, DK_COL = 320;  // S^T, dP^T: 2 x 64; dv 64; dk 96
constexpr uint32_t IDESC_S = umma_idesc_bf16(BK, QT, false, false);
constexpr uint32_t IDESC_V = umma_idesc_bf16(BK, DH, false, true);
constexpr uint32_t IDESC_K = umma_idesc_bf16(BK, 96, false, true);
constexpr size_t OFF_ITEM = 0;
constexpr size_t OFF_Q = OFF_ITEM + ITEM;
constexpr size_t OFF_BAR = OFF_Q + (size_t)KS * QSTAGE;
constexpr int NBAR = 2 + 2 * KS + 3 * NSB + 3;
constexpr size_t OFF_TMEM = OFF_BAR + NBAR * 8;
constexpr size_t SMEM_USED = OFF_TMEM + 16;
static_assert(OFF_Q % 1024 == 0 && QSTAGE % 1024 == 0, "tile bases must be 1024-aligned");
static_assert(SMEM_USED + 1024 <= 232448, "one block's shared memory (227 KB)");

struct Item {
  int b, h, g0, k0, nqt;  // groups g0 + 1 .. g0 + BK; query tiles k0 .. k0 + nqt - 1 (64 positions each)
};
__device__ __forceinline__ Item item_of(const TrainBwdTc& p, int o) {
  Item it;
  const int bh = o % (p.B * p.H);
  it.b = bh / p.H;
  it.h = bh % p.H;
  it.g0 = (o / (p.B * p.H)) * BK;  // earliest groups (the most queries) first
  const int first = (it.g0 + 1) * p.s;  // 0-based position of the first query that sees group g0 + 1
  it.k0 = first / QT;
  it.nqt = first < p.T ? (p.T - 1) / QT - it.k0 + 1 : 0;
  return it;
}

__global__ void __launch_bounds__(NT, 1) bwd_dkv_tc_kernel(const __grid_constant__ TrainBwdKvMaps mp,
                                                           const TrainBwdTc p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* const item_full = bar + 0;
  uint64_t* const item_empty = bar + 1;         // the epilogue is done with the item's rows (EPW)
  uint64_t* const q_full = bar + 2;             // [KS]
  uint64_t* const q_empty = bar + 2 + KS;       // [KS] the tile's dv / dk MMAs have read it
  uint64_t* const s_full = bar + 2 + 2 * KS;    // [NSB] S^T and dP^T in TMEM
  uint64_t* const pds_full = s_full + NSB;      // [NSB] P^T and dS^T written (SMW)
  uint64_t* const pds_empty = s_full + 2 * NSB; // [NSB] the dv / dk MMAs have read them
  uint64_t* const acc_full = s_full + 3 * NSB;
  uint64_t* const acc_empty = acc_full + 1;     // (EPW)
  uint64_t* const mma_done = acc_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(item_full, 1);
    mbar_init(item_empty, EPW);
    for (int i = 0; i < KS; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < NSB; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&pds_full[i], SMW);
      mbar_init(&pds_empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, EPW);
    mbar_init(mma_done, 2);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == TMA_WARP && lane == 0) {
    prefetch_tmap(&mp.k_g);
    prefetch_tmap(&mp.kr_g);
    prefetch_tmap(&mp.v_g);
    prefetch_tmap(&mp.q_g);
    prefetch_tmap(&mp.qr_g);
    prefetch_tmap(&mp.do_g);
    prefetch_tmap(&mp.q64);
    prefetch_tmap(&mp.qr64);
    prefetch_tmap(&mp.do64);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");  // Delta and lse2 come from an earlier launch
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t sI = smem_u32(sm + OFF_ITEM);
  const uint32_t sQ = smem_u32(sm + OFF_Q);
  const int G = gridDim.x;
  const int n_groups = p.T / p.s;
  const int n_items = p.B * p.H * ((n_groups + BK - 1) / BK);
  const float sl2 = p.scale_log2, sc = p.scale;
  bool ok = true;

  if (warp == TMA_WARP) {
    if (lane == 0) {
      uint32_t ic = 0, qc = 0;
      for (int o; (o = tile_index(ic, blockIdx.x, G)) < n_items && ok; ++ic) {
        const Item it = item_of(p, o);
        if (ic > 0 && !mbar_wait(item_empty, (ic - 1) & 1)) { ok = false; break; }
        mbar_arrive_expect_tx(item_full, ITEM);
        tma_load_5d(sm + OFF_ITEM, &mp.k_g, 0, it.h, it.g0, it.b, 0, item_full);
        tma_load_3d(sm + OFF_ITEM + 2 * KPL, &mp.kr_g, 0, it.g0, it.b, item_full);
        tma_load_5d(sm + OFF_ITEM + 3 * KPL, &mp.v_g, 0, it.h, it.g0, it.b, 0, item_full);
        tma_load_5d(sm + OFF_ITEM + 5 * KPL, &mp.q_g, 0, it.h, it.g0, it.b, 0, item_full);
        tma_load_4d(sm + OFF_ITEM + 7 * KPL, &mp.qr_g, 0, it.h, it.g0, it.b, item_full);
        tma_load_5d(sm + OFF_ITEM + 8 * KPL, &mp.do_g, 0, it.h, it.g0, it.b, 0, item_full);
        const int64_t lbase = ((int64_t)it.b * p.H + it.h) * p.Tp;
        for (int q = 0; q < it.nqt; ++q, ++qc) {
          const int st = qc % KS;
          if (qc >= KS && !mbar_wait(&q_empty[st], ((qc / KS) & 1) ^ 1)) { ok = false; break; }
          const int m0 = (it.k0 + q) * QT;  // 0-based first position of the tile
          const int row = it.b * p.T + m0;
          uint8_t* qb = sm + OFF_Q + (size_t)st * QSTAGE;
          mbar_arrive_expect_tx(&q_full[st], QBYTES);
          tma_load_4d(qb, &mp.q64, 0, it.h, row, 0, &q_full[st]);
          tma_load_3d(qb + 2 * QPL, &mp.qr64, 0, it.h, row, &q_full[st]);
          tma_load_4d(qb + 3 * QPL, &mp.do64, 0, it.h, row, 0, &q_full[st]);
          bulk_load(qb + 5 * QPL, p.lse2 + lbase + m0, QT * 4, &q_full[st]);
          bulk_load(qb + 5 * QPL + QT * 4, p.delta + lbase + m0, QT * 4, &q_full[st]);
        }
      }
      if (!ok) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
      if (ic) mbar_wait(item_full, (ic - 1) & 1);
      for (uint32_t j = qc > (uint32_t)KS ? qc - KS : 0; j < qc; ++j) mbar_wait(&q_full[j % KS], (j / KS) & 1);
    }
  } else if (warp == SMMA_WARP || warp == GMMA_WARP) {
    const bool scores = warp == SMMA_WARP;
    const uint64_t dka = umma_desc(sI, 16, 512, 4);              // keys [k | k^R], K-major (rows = keys)
    const uint64_t dva = umma_desc(sI + 3 * KPL, 16, 512, 4);    // values, K-major
    const uint64_t dqb = umma_desc(sQ, 16, 512, 4);              // query tile [q | q^R], K-major
    const uint64_t dob = umma_desc(sQ + 3 * QPL, 16, 512, 4);    // query tile dO, K-major
    const uint64_t dqm = umma_desc(sQ, QPL, 512, 4);             // [q | q^R] as the MN-major B of dk
    const uint64_t dom = umma_desc(sQ + 3 * QPL, QPL, 512, 4);   // dO as the MN-major B of dv
    uint32_t ic = 0, qc = 0;
    for (int o; (o = tile_index(ic, blockIdx.x, G)) < n_items && ok; ++ic) {
      const Item it = item_of(p, o);
      if (scores) {
        if (!warp_wait(item_full, ic & 1)) { ok = false; break; }
        for (int q = 0; q < it.nqt && ok; ++q) {
          const uint32_t j = qc + q;
          const int st = j % KS, sb = j % NSB;
          if (!warp_wait(&q_full[st], (j / KS) & 1)) { ok = false; break; }
          if (j >= NSB && !warp_wait(&pds_empty[sb], ((j / NSB) & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 6; ++kk) {
              const uint64_t ad = dka + (uint64_t)(((kk >> 1) * KPL + (kk & 1) * 32) >> 4);
              const uint64_t bd = dqb + (uint64_t)((st * QSTAGE + (kk >> 1) * QPL + (kk & 1) * 32) >> 4);
              umma_bf16(tmem + S_COL + 64 * sb, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = dva + (uint64_t)(((kk >> 1) * KPL + (kk & 1) * 32) >> 4);
              const uint64_t bd = dob + (uint64_t)((st * QSTAGE + (kk >> 1) * QPL + (kk & 1) * 32) >> 4);
              umma_bf16(tmem + DP_COL + 64 * sb, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
            }
            umma_commit(&s_full[sb]);
          }
          __syncwarp();
        }
      } else {
        for (int q = 0; q < it.nqt && ok; ++q) {
          const uint32_t j = qc + q;
          const int st = j % KS, sb = j % NSB;
          if (!warp_wait(&pds_full[sb], (j / NSB) & 1)) { ok = false; break; }
          if (q == 0 && ic > 0 && !warp_wait(acc_empty, (ic - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < QT / 16; ++kk) {
              const uint64_t bo = dom + (uint64_t)((st * QSTAGE + kk * 16 * 64) >> 4);
              umma_bf16_ts(tmem + DV_COL, tmem + S_COL + 64 * sb + 8 * kk, bo, IDESC_V, (q > 0 || kk > 0) ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < QT / 16; ++kk) {
              const uint64_t bq = dqm + (uint64_t)((st * QSTAGE + kk * 16 * 64) >> 4);
              umma_bf16_ts(tmem + DK_COL, tmem + DP_COL + 64 * sb + 8 * kk, bq, IDESC_K, (q > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&q_empty[st]);
            umma_commit(&pds_empty[sb]);
          }
          __syncwarp();
        }
        if (ok && it.nqt == 0 && ic > 0 && !warp_wait(acc_empty, (ic - 1) & 1)) ok = false;
        if (ok) {
          if (elect_one()) umma_commit(acc_full);
          __syncwarp();
        }
      }
      qc += it.nqt;
    }
    if (!ok && lane == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
    if (elect_one()) umma_commit(mma_done);
    __syncwarp();
    warp_wait(mma_done, 0);
  } else if (warp >= EPI_WARP0) {
    // key row i: the own column's terms (query m = n), then dv, [dk | dk^R]
    const int qe = warp - EPI_WARP0;
    const int i = qe * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(qe * 32) << 16);
    for (uint32_t ic = 0;; ++ic) {
      const int o = tile_index(ic, blockIdx.x, G);
      if (o >= n_items) break;
      const Item it = item_of(p, o);
      const int g = it.g0 + 1 + i;
      const bool valid = g <= n_groups;
      const int n = g * p.s;  // 1-based position of the key column
      if (ok && !warp_wait(item_full, ic & 1)) ok = false;
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int ch = 0; ch < 12; ++ch) {
        uint32_t a[4], b[4];
        lds4(sI + plane_off(BK, i, ch), a);
        lds4(sI + 5 * KPL + plane_off(BK, i, ch), b);
        s = dot8(a, b, s);
      }
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint32_t a[4], b[4];
        lds4(sI + 3 * KPL + plane_off(BK, i, ch), a);
        lds4(sI + 8 * KPL + plane_off(BK, i, ch), b);
        dp = dot8(a, b, dp);
      }
      const int64_t lbase = ((int64_t)it.b * p.H + it.h) * p.Tp;
      const float pown = valid ? ex2_approx(s * sl2 - p.lse2[lbase + n - 1]) : 0.f;
      const float ds = valid ? pown * (dp - p.delta[lbase + n - 1]) : 0.f;
      if (ok && !warp_wait(acc_full, ic & 1)) ok = false;
      tc_fence_after();
      const size_t row = ((size_t)it.b * p.T + (valid ? n - 1 : 0)) * p.H + it.h;
      // dv = sum_m P^T dO + P_own dO_n, 32 channels at a time
#pragma unroll 1
      for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t acc[32];
        if (it.nqt > 0) {
          tmem_ld32(lane_base + DV_COL + 32 * c2, acc);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[e] = 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t x[4];
          lds4(sI + 8 * KPL + plane_off(BK, i, 4 * c2 + c4), x);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 d = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x[e]));
            const int c = c4 * 8 + e * 2;
            w[c4 * 4 + e] = pack_bf16x2(__uint_as_float(acc[c]) + pown * d.x, __uint_as_float(acc[c + 1]) + pown * d.y);
          }
        }
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.dv + row * DH + 32 * c2);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) dst[c4] = make_uint4(w[4 * c4], w[4 * c4 + 1], w[4 * c4 + 2], w[4 * c4 + 3]);
        }
      }
      // [dk | dk^R] = (sum_m dS^T [q | q^R] + dS_own [q | q^R]_n) / sqrt(d_h)
#pragma unroll 1
      for (int c2 = 0; c2 < 3; ++c2) {
        uint32_t acc[32];
        if (it.nqt > 0) {
          tmem_ld32(lane_base + DK_COL + 32 * c2, acc);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[e] = 0u;
        }
        float f[32];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t x[4];
          lds4(sI + 5 * KPL + plane_off(BK, i, 4 * c2 + c4), x);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 d = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x[e]));
            const int c = c4 * 8 + e * 2;
            f[c] = (__uint_as_float(acc[c]) + ds * d.x) * sc;
            f[c + 1] = (__uint_as_float(acc[c + 1]) + ds * d.y) * sc;
          }
        }
        if (valid) {
          if (c2 < 2) {
            uint4* dst = reinterpret_cast<uint4*>(p.dk + row * DH + 32 * c2);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
              dst[c4] = make_uint4(pack_bf16x2(f[8 * c4], f[8 * c4 + 1]), pack_bf16x2(f[8 * c4 + 2], f[8 * c4 + 3]),
                                   pack_bf16x2(f[8 * c4 + 4], f[8 * c4 + 5]), pack_bf16x2(f[8 * c4 + 6], f[8 * c4 + 7]));
          } else {
            float4* dst = reinterpret_cast<float4*>(p.dkrh + row * DR);
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) dst[c4] = make_float4(f[4 * c4], f[4 * c4 + 1], f[4 * c4 + 2], f[4 * c4 + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(acc_empty);
        mbar_arrive(item_empty);
      }
    }
    if (!ok && lane == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
  } else if (warp < SMW) {
    // gradient warps: key row i (TMEM lane), half hf of the tile's 64 query
    // columns.  P^T and dS^T (bf16) go back over the first 32 columns of the
    // S^T and dP^T buffers once both halves have loaded theirs (pair barrier).
    const int qw = warp & 3, hf = warp >> 2;
    const int i = qw * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    uint32_t ic = 0, qc = 0;
    for (int o; (o = tile_index(ic, blockIdx.x, G)) < n_items; ++ic) {
      const Item it = item_of(p, o);
      const int g = it.g0 + 1 + i;
      const int n = g <= n_groups ? g * p.s : 0x7fffffff;  // a column past the groups is seen by no query
      for (int q = 0; q < it.nqt; ++q) {
        const uint32_t j = qc + q;
        const int st = j % KS, sb = j % NSB;
        if (ok && !warp_wait(&s_full[sb], (j / NSB) & 1)) ok = false;
        if (ok && !warp_wait(&q_full[st], (j / KS) & 1)) ok = false;
        tc_fence_after();
        uint32_t sr[32], dr[32];
        tmem_ld32(lane_base + S_COL + 64 * sb + 32 * hf, sr);
        tmem_ld32(lane_base + DP_COL + 64 * sb + 32 * hf, dr);
        tmem_wait_ld();
        tc_fence_before();
        named_bar(1 + qw, 64);
        tc_fence_after();
        const float* L = reinterpret_cast<const float*>(sm + OFF_Q + (size_t)st * QSTAGE + 5 * QPL) + 32 * hf;
        const float* Dd = L + QT;
        const int m0 = (it.k0 + q) * QT + 1 + 32 * hf;  // query of column 0 of this half (1-based)
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const int m = m0 + c;
          const bool v0 = n < m && m <= p.T, v1 = n < m + 1 && m + 1 <= p.T;
          const float p0 = v0 ? ex2_approx(__uint_as_float(sr[c]) * sl2 - L[c]) : 0.f;
          const float p1 = v1 ? ex2_approx(__uint_as_float(sr[c + 1]) * sl2 - L[c + 1]) : 0.f;
          pk[c >> 1] = pack_bf16x2(p0, p1);
          // (Delta past the sequence is padding: masked columns must not read it)
          dk[c >> 1] = pack_bf16x2(v0 ? p0 * (__uint_as_float(dr[c]) - Dd[c]) : 0.f,
                                   v1 ? p1 * (__uint_as_float(dr[c + 1]) - Dd[c + 1]) : 0.f);
        }
        tmem_st16(lane_base + S_COL + 64 * sb + 16 * hf, pk);
        tmem_st16(lane_base + DP_COL + 64 * sb + 16 * hf, dk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pds_full[sb]);
      }
      qc += it.nqt;
    }
    if (!ok && lane == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
  }
  // (the dot warp has no role here)

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}
}  // namespace dkv

cudaLaunchAttribute pdl_attr() {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

}  // namespace bwt

size_t bwd_dq_tc_smem() { return bwt::dq::SMEM_USED + 1024; }

size_t bwd_dkv_tc_smem() { return bwt::dkv::SMEM_USED + 1024; }

cudaError_t launch_bwd_dkv_tc(const TrainBwdKvMaps& mp, const TrainBwdTc& p, int grid, cudaStream_t st) {
  const size_t smem = bwd_dkv_tc_smem();
  static uint64_t done_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(done_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(bwt::dkv::bwd_dkv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev < 64) done_mask |= 1ull << dev;
  }
  cudaLaunchAttribute attr[1] = {bwt::pdl_attr()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(bwt::NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, bwt::dkv::bwd_dkv_tc_kernel, mp, p);
}

cudaError_t launch_bwd_dq_tc(const TrainBwdMaps& mp, const TrainBwdTc& p, int grid, cudaStream_t st) {
  const size_t smem = bwd_dq_tc_smem();
  static uint64_t done_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(done_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(bwt::dq::bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev < 64) done_mask |= 1ull << dev;
  }
  cudaLaunchAttribute attr[1] = {bwt::pdl_attr()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(bwt::NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, bwt::dq::bwd_dq_tc_kernel, mp, p);
}

}  // namespace mtla
