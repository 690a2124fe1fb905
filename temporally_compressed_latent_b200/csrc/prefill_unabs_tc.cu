// Masked attention with explicit per-head keys and values (the un-absorbed
// form, and the training shortcut's forward) on the 5th-generation tensor
// cores: tcgen05 + TMEM, bf16, d_h = 64, d_R = 32.
//
// What it computes (MTLA paper notes, "Key designs: stride-aware causal mask"
// and "decoupled RoPE with temporal compression"): for query m (1-based) of
// sequence b and head h, over the columns n == m and n = g s (g < ceil(m/s)),
//   score_n = ([q | q^R]_m . [k | k^R]_n) / sqrt(d_h),
//   out = sum_n softmax(score)_n v_n,  lse = log sum_n exp(score_n),
// where k^R_n is the merged k_hat^R'_n (the last d_R channels of C_hat') for
// the prefill, or the uncompressed K^R_n for the training shortcut.
//
// Design (B200):
//  * An M tile is 128 consecutive queries of one (sequence, head); a key tile
//    is 64 completed groups of the same head.  The queries [q | q^R], the
//    keys [k | k^R] (96 wide) and the values v (64 wide) land by TMA as
//    [rows x 64 B] planes with the 64-byte swizzle: the canonical K-major
//    operand layout of the score MMA, and the MN-major layout of v as the
//    value MMA's B operand.  The group columns are read straight out of
//    k, v and k^R through tensor maps whose row stride is s positions, so
//    no compressed copy is made.  The own rows (k, k^R, v of the tile's 128
//    positions) come by TMA into a buffer per M-tile parity.
//  * Scores S = Q K^T (M 128, N 64, K 96) and values O += P V (M 128, N 64,
//    K 64) are tcgen05.mma ops with fp32 accumulators in TMEM (four 64-column
//    S / P buffers and the 64 columns of O).  A score warp and a value warp
//    issue them, each as soon as its inputs are ready.
//  * Eight softmax warps, two per TMEM lane quarter: one takes the even key
//    tiles, the other the odd ones, all 64 columns each, with its own running
//    max and sum and its own O accumulator in TMEM (d_h = 64 makes a second
//    O cheap), rescaled only when the max grows by more than 2^8; the two
//    never wait for each other, and the epilogue merges them.  bf16 P is
//    written back over the tile's S columns, where the value MMA reads it.
//    A dot warp takes the own-column scores while the key tiles run; four
//    epilogue warps fold the own column in, normalise, and write out and lse.
//  * One TMA warp, two MMA warps, mbarrier pipelines; a persistent grid visits
//    the M tiles heaviest first, in rounds of alternating direction.
#include "kernels.cuh"

namespace mtla {
namespace utc {

constexpr int DH = 64, DR = 32;
constexpr int BM = 128;                // queries per M tile
constexpr int BN = 64;                 // groups per key tile
constexpr int QPL = BM * 64;           // bytes of one 128-row plane (8192)
constexpr int KPL = BN * 64;           // bytes of one 64-row plane (4096)
constexpr int QBYTES = 3 * QPL;        // [q | q^R]: 3 planes
constexpr int OWNB = 5 * QPL;          // own rows: k (2 planes), k^R (1), v (2)
constexpr int STAGE = 5 * KPL;         // key tile: k (2), k^R (1), v (2): 20480
constexpr int KS = 4;                  // key-tile stages
constexpr int SMW = 8;                 // softmax warps: two per TMEM lane quarter
constexpr int EPW = 4;                 // epilogue warps
constexpr int NT = 32 * (SMW + 4 + EPW);
constexpr int TMA_WARP = SMW, SMMA_WARP = SMW + 1, PMMA_WARP = SMW + 2, DOT_WARP = SMW + 3, EPI_WARP0 = SMW + 4;
static_assert(EPI_WARP0 % 4 == 0, "epilogue warp e reads TMEM lane quarter e");
constexpr uint32_t TMEM_COLS = 512;
constexpr int NSB = 4;                 // S / P buffers in TMEM (64 columns each)
constexpr uint32_t O_COL = 256;         // two O accumulators: even tiles at O_COL, odd tiles at O_COL + 64
__host__ __device__ constexpr uint32_t s_col(int b) { return 64u * (uint32_t)b; }
constexpr uint32_t IDESC_S = umma_idesc_bf16(BM, BN, false, false);
constexpr uint32_t IDESC_O = umma_idesc_bf16(BM, DH, false, true);

constexpr size_t OFF_Q = 0;
constexpr size_t OFF_OWN = OFF_Q + QBYTES;               // two own-row buffers (M tile parity)
constexpr size_t OFF_K = OFF_OWN + 2 * OWNB;             // KS stages
constexpr size_t OFF_XCH = OFF_K + (size_t)KS * STAGE;   // row maxima, sums, final maxima, own-row scores
constexpr size_t OFF_BAR = OFF_XCH + (4 + 4 + 2 + 2) * BM * 4;
constexpr int NBAR = 2 + 12 + 2 * KS + 3 * NSB + 3;
constexpr size_t OFF_TMEM = OFF_BAR + NBAR * 8;
constexpr size_t SMEM_USED = OFF_TMEM + 16;
static_assert(OFF_OWN % 1024 == 0 && OFF_K % 1024 == 0 && STAGE % 1024 == 0 && OWNB % 1024 == 0,
              "tile bases must be 1024-aligned");
static_assert(SMEM_USED + 1024 <= 232448, "one block's shared memory (227 KB)");

struct Params {
  int B, T, H, s;
  int n_mtiles;            // B * H * ceil(T / BM)
  float scale_log2;        // log2(e) / sqrt(d_h)
  __nv_bfloat16* out;      // [B, T, H, d_h]
  float* lse;              // nullable [B, T, H]
  int32_t* dev_err;
};

// 16-byte chunk ch of row `row` inside a plane-layout tile whose planes hold
// `rows` rows: plane ch / 4, 64-byte swizzle phase (row / 2) mod 4
__device__ __forceinline__ uint32_t plane_off(int rows, int row, int ch) {
  return (uint32_t)(ch >> 2) * (uint32_t)(rows * 64) + (uint32_t)row * 64u +
         ((((uint32_t)ch & 3u) ^ (((uint32_t)row >> 1) & 3u)) << 4);
}

// 2^x with the hardware approximation (relative error about 2^-22; results
// below 2^-126 flush to zero, 2^-inf = 0): the probabilities' exponentials
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
      "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}


// mbarrier wait by every lane of a warp, warp-uniform result (the tcgen05
// loads and stores that follow are warp-collective)
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

// M tile of block x in round r: numbered heaviest first, rounds alternate direction
__device__ __forceinline__ int tile_index(int r, int x, int G) { return r * G + ((r & 1) ? G - 1 - x : x); }

struct Tile {
  int b, h, m0, nkt;
};
// The last M tile of a (sequence, head) is ragged when T is not a multiple of
// BM: its rows past query T read finite values (the next sequence's rows, or
// the TMA fill past the last one) and are never stored.
__device__ __forceinline__ Tile tile_of(const Params& p, int o) {
  const int per_seq = (p.T + BM - 1) / BM;
  const int bh = o % (p.B * p.H);
  Tile t;
  t.b = bh / p.H;
  t.h = bh % p.H;
  const int mb = per_seq - 1 - o / (p.B * p.H);
  t.m0 = mb * BM + 1;
  const int m_last = t.m0 + BM - 1 < p.T ? t.m0 + BM - 1 : p.T;
  const int vis_max = (int)group_of(m_last, p.s) - 1;  // groups seen by the tile's last query
  t.nkt = (vis_max + BN - 1) / BN;
  return t;
}

struct Maps {
  CUtensorMap q, qr;           // queries: 4-D {32, H, B T, 2 planes}; RoPE queries: 3-D {32, H, B T}
  CUtensorMap k_own, v_own;    // like q, on k and v
  CUtensorMap kr_own;          // 2-D {32, B T} (row stride kr_stride)
  CUtensorMap k_grp, v_grp;    // 5-D {32, H, groups, B, 2 planes}: rows n = g s
  CUtensorMap kr_grp;          // 3-D {32, groups, B}
};

__global__ void __launch_bounds__(NT, 1) prefill_unabs_tc_kernel(const __grid_constant__ Maps mp, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* const q_full = bar + 0;
  uint64_t* const q_empty = bar + 1;            // the tile's last score MMA + the dot warp
  uint64_t* const own_full = bar + 2;           // [2] own rows of M tile parity b landed
  uint64_t* const own_empty = bar + 4;          // [2] the epilogue is done with them
  uint64_t* const dot_full = bar + 6;           // [2] own-column scores written
  uint64_t* const dot_empty = bar + 8;          // [2] the epilogue has read them
  uint64_t* const stat_full = bar + 10;         // [2] a tile's row maxima and sums written
  uint64_t* const stat_empty = bar + 12;        // [2] the epilogue has read them
  uint64_t* const k_full = bar + 14;            // [KS]
  uint64_t* const k_empty = bar + 14 + KS;      // [KS]
  uint64_t* const s_full = bar + 14 + 2 * KS;   // [NSB]
  uint64_t* const p_full = s_full + NSB;        // [NSB]
  uint64_t* const p_empty = s_full + 2 * NSB;   // [NSB]: the value MMA has read P
  uint64_t* const o_full = s_full + 3 * NSB;
  uint64_t* const o_empty = o_full + 1;
  uint64_t* const mma_done = o_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
  float* xm = reinterpret_cast<float*>(sm + OFF_XCH);                   // [2 M-tile parity][2 tile parity][BM]: maxima
  float* xl = reinterpret_cast<float*>(sm + OFF_XCH + 4 * BM * 4);      // [2][2][BM]: row sums
  float* xdot = reinterpret_cast<float*>(sm + OFF_XCH + 8 * BM * 4);    // [2 M-tile parity][BM]: own-column scores
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 2);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&own_full[b], 1);
      mbar_init(&own_empty[b], EPW);
      mbar_init(&dot_full[b], 1);
      mbar_init(&dot_empty[b], EPW);
      mbar_init(&stat_full[b], SMW);
      mbar_init(&stat_empty[b], EPW);
    }
    for (int i = 0; i < KS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < NSB; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], SMW / 2);  // the four warps of the tile's parity
      mbar_init(&p_empty[i], 1);
    }
    mbar_init(o_full, 1);
    mbar_init(o_empty, EPW);
    mbar_init(mma_done, 2);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == TMA_WARP && lane == 0) {
    prefetch_tmap(&mp.q);
    prefetch_tmap(&mp.qr);
    prefetch_tmap(&mp.k_own);
    prefetch_tmap(&mp.v_own);
    prefetch_tmap(&mp.kr_own);
    prefetch_tmap(&mp.k_grp);
    prefetch_tmap(&mp.v_grp);
    prefetch_tmap(&mp.kr_grp);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");  // k and v may come from the previous launch
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t sQ = smem_u32(sm + OFF_Q);
  const uint32_t sOwn = smem_u32(sm + OFF_OWN);
  const uint32_t sK = smem_u32(sm + OFF_K);
  const int G = gridDim.x;
  bool ok = true;

  if (warp == TMA_WARP) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      uint32_t tc = 0, kc = 0, q_issued = 0;
      for (int o; (o = tile_index(tc, blockIdx.x, G)) < p.n_mtiles && ok; ++tc) {
        const Tile t = tile_of(p, o);
        const int row0 = t.b * p.T + (t.m0 - 1);  // first position of the tile in [B T]
        const int sb2 = tc & 1;
        if (tc > 0 && !mbar_wait(q_empty, (tc - 1) & 1)) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, QBYTES);
        tma_load_4d(sm + OFF_Q, &mp.q, 0, t.h, row0, 0, q_full);
        tma_load_3d(sm + OFF_Q + 2 * QPL, &mp.qr, 0, t.h, row0, q_full);
        q_issued = tc + 1;
        // own rows into the buffer of this tile's parity, once the epilogue of
        // tile tc - 2 is done with it
        if (tc >= 2 && !mbar_wait(&own_empty[sb2], ((tc >> 1) & 1) ^ 1)) { ok = false; break; }
        uint8_t* ob = sm + OFF_OWN + (size_t)sb2 * OWNB;
        mbar_arrive_expect_tx(&own_full[sb2], OWNB);
        tma_load_4d(ob, &mp.k_own, 0, t.h, row0, 0, &own_full[sb2]);
        tma_load_2d(ob + 2 * QPL, &mp.kr_own, 0, row0, &own_full[sb2]);
        tma_load_4d(ob + 3 * QPL, &mp.v_own, 0, t.h, row0, 0, &own_full[sb2]);
        for (int kt = 0; kt < t.nkt; ++kt, ++kc) {
          const int st = kc % KS;
          if (kc >= KS && !mbar_wait(&k_empty[st], ((kc / KS) & 1) ^ 1)) { ok = false; break; }
          uint8_t* kb = sm + OFF_K + (size_t)st * STAGE;
          mbar_arrive_expect_tx(&k_full[st], STAGE);
          tma_load_5d(kb, &mp.k_grp, 0, t.h, kt * BN, t.b, 0, &k_full[st]);
          tma_load_3d(kb + 2 * KPL, &mp.kr_grp, 0, kt * BN, t.b, &k_full[st]);
          tma_load_5d(kb + 3 * KPL, &mp.v_grp, 0, t.h, kt * BN, t.b, 0, &k_full[st]);
        }
      }
      if (!ok) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
      // drain: no copy may still be writing shared memory when the block exits
      if (q_issued) mbar_wait(q_full, (q_issued - 1) & 1);
      for (uint32_t u = q_issued > 2 ? q_issued - 2 : 0; u < q_issued; ++u) mbar_wait(&own_full[u & 1], (u >> 1) & 1);
      for (uint32_t j = kc > (uint32_t)KS ? kc - KS : 0; j < kc; ++j) mbar_wait(&k_full[j % KS], (j / KS) & 1);
    }
  } else if (warp == DOT_WARP) {
    // ======================= own-column scores =======================
    // [q | q^R]_m . [k | k^R]_m for the 128 rows (lane: rows lane + 32 r)
    for (uint32_t tc = 0; tile_index(tc, blockIdx.x, G) < p.n_mtiles; ++tc) {
      const int sb2 = tc & 1;
      if (ok && !warp_wait(q_full, tc & 1)) ok = false;
      if (ok && !warp_wait(&own_full[sb2], (tc >> 1) & 1)) ok = false;
      if (ok && tc >= 2 && !warp_wait(&dot_empty[sb2], ((tc >> 1) & 1) ^ 1)) ok = false;
      const uint32_t ownb = sOwn + sb2 * OWNB;
#pragma unroll 1
      for (int r = 0; r < BM / 32; ++r) {
        const int i = r * 32 + lane;
        float dot = 0.f;
#pragma unroll
        for (int ch = 0; ch < 12; ++ch) {  // 96 elements: 12 chunks of 8
          uint32_t qv[4], kv[4];
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(qv[0]), "=r"(qv[1]), "=r"(qv[2]), "=r"(qv[3])
                       : "r"(sQ + plane_off(BM, i, ch)));
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(kv[0]), "=r"(kv[1]), "=r"(kv[2]), "=r"(kv[3])
                       : "r"(ownb + plane_off(BM, i, ch)));
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qv[e]));
            const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kv[e]));
            dot = fmaf(a.x, c.x, dot);
            dot = fmaf(a.y, c.y, dot);
          }
        }
        xdot[sb2 * BM + i] = dot;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(q_empty);
        mbar_arrive(&dot_full[sb2]);
      }
    }
    if (!ok && lane == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
  } else if (warp == SMMA_WARP || warp == PMMA_WARP) {
    // ======================= MMA issuers =======================
    // The score warp issues S(j) as soon as its key tile has landed and its
    // TMEM buffer is free; the value warp issues O += P(j) V(j) as soon as
    // the softmax has written P(j).  All 32 lanes run the loop (warp-uniform
    // waits); one elected lane issues the MMAs and their commits.  A K step
    // or a stage moves only the descriptors' start-address field (shared
    // addresses are below 2^18: no carry).
    const bool scores = warp == SMMA_WARP;
    const uint64_t dq0 = umma_desc(sQ, 16, 512, 4);
    const uint64_t dk0 = umma_desc(sK, 16, 512, 4);
    const uint64_t dv0 = umma_desc(sK + 3 * KPL, KPL, 512, 4);  // v planes: MN-major, plane stride KPL
    uint32_t tc = 0, kc = 0;
    for (int o; (o = tile_index(tc, blockIdx.x, G)) < p.n_mtiles && ok; ++tc) {
      const Tile t = tile_of(p, o);
      if (scores) {
        if (!warp_wait(q_full, tc & 1)) { ok = false; break; }
        for (int kt = 0; kt < t.nkt && ok; ++kt) {
          const uint32_t j = kc + kt;
          const int st = j % KS, sb = j % NSB;
          if (!warp_wait(&k_full[st], (j / KS) & 1)) { ok = false; break; }
          if (j >= NSB && !warp_wait(&p_empty[sb], ((j / NSB) & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 6; ++kk) {  // K = 96: 6 steps of 16, two per plane
              const uint64_t ad = dq0 + (uint64_t)(((kk >> 1) * QPL + (kk & 1) * 32) >> 4);
              const uint64_t bd = dk0 + (uint64_t)((st * STAGE + (kk >> 1) * KPL + (kk & 1) * 32) >> 4);
              umma_bf16(tmem + s_col(sb), ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
            }
            umma_commit(&s_full[sb]);
            if (kt + 1 == t.nkt) umma_commit(q_empty);  // the tile's scores no longer read Q
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
          const int pb = j % NSB, st = j % KS;
          if (!warp_wait(&p_full[pb], (j / NSB) & 1)) { ok = false; break; }
          if (kt == 0 && tc > 0 && !warp_wait(o_empty, (tc - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
              const uint32_t pa = tmem + s_col(pb) + 8 * kk;  // two bf16 per column: 8 columns per K step
              const uint64_t bd = dv0 + (uint64_t)((st * STAGE + kk * 16 * 64) >> 4);
              umma_bf16_ts(tmem + O_COL + 64 * (j & 1), pa, bd, IDESC_O, (kt > 1 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&k_empty[st]);
            umma_commit(&p_empty[pb]);
          }
          __syncwarp();
        }
        // a tile without key tiles still waits for the epilogue of tile tc - 1
        // before it completes o_full (o_full must not complete twice ahead of it)
        if (ok && t.nkt == 0 && tc > 0 && !warp_wait(o_empty, (tc - 1) & 1)) ok = false;
        if (ok) {
          if (elect_one()) umma_commit(o_full);
          __syncwarp();
        }
      }
      kc += t.nkt;
    }
    if (!ok && lane == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
    if (elect_one()) umma_commit(mma_done);  // every MMA of both warps completes before TMEM is released
    __syncwarp();
    warp_wait(mma_done, 0);
  } else if (warp >= EPI_WARP0) {
    // ======================= epilogue warps =======================
    // warp EPI_WARP0 + e: rows 32 e .. 32 e + 31 (TMEM lane quarter e), all 64
    // channels: out = (alpha O + p_own v_m) / (alpha l + p_own), the own
    // column as one more key; lse from the same terms.
    const int qe = warp - EPI_WARP0;
    const int i = qe * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(qe * 32) << 16);
    const float sl2 = p.scale_log2;
    uint32_t tc = 0, kc = 0;
    for (int o; (o = tile_index(tc, blockIdx.x, G)) < p.n_mtiles; ++tc) {
      const Tile t = tile_of(p, o);
      const int sb2 = tc & 1;
      // O accumulator q was written by this M tile iff one of its key tiles j has j mod 2 == q
      const bool w0 = t.nkt >= 2 || (t.nkt == 1 && (kc & 1) == 0);
      const bool w1 = t.nkt >= 2 || (t.nkt == 1 && (kc & 1) == 1);
      kc += t.nkt;
      if (ok && !warp_wait(&stat_full[sb2], (tc >> 1) & 1)) ok = false;
      if (ok && !warp_wait(&dot_full[sb2], (tc >> 1) & 1)) ok = false;
      if (ok && !warp_wait(&own_full[sb2], (tc >> 1) & 1)) ok = false;
      // the two groups' running max and sum (even and odd j), merged with the own column
      const float m_e = xm[(sb2 * 2 + 0) * BM + i], m_o = xm[(sb2 * 2 + 1) * BM + i];
      const float l_e = xl[(sb2 * 2 + 0) * BM + i], l_o = xl[(sb2 * 2 + 1) * BM + i];
      const float xs = xdot[sb2 * BM + i] * sl2;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&stat_empty[sb2]);
        mbar_arrive(&dot_empty[sb2]);
      }
      const float mf = fmaxf(fmaxf(m_e, m_o), xs);
      const float a_e = m_e == -INFINITY ? 0.f : exp2f(m_e - mf);
      const float a_o = m_o == -INFINITY ? 0.f : exp2f(m_o - mf);
      const float pown = exp2f(xs - mf);
      const float den = l_e * a_e + l_o * a_o + pown;
      const float inv = 1.f / den;
      if (ok && !warp_wait(o_full, tc & 1)) ok = false;
      tc_fence_after();
      const int m = t.m0 + i;  // this row's query (1-based)
      const uint32_t vown = sOwn + sb2 * OWNB + 3 * QPL;
      const size_t row = ((size_t)t.b * p.T + (m <= p.T ? m - 1 : 0)) * p.H + t.h;
      uint4* dst = reinterpret_cast<uint4*>(p.out + row * DH);
#pragma unroll 1
      for (int c2 = 0; c2 < 2; ++c2) {  // 32 channels at a time
        uint32_t oe[32], oo[32];
        if (w0) tmem_ld32(lane_base + O_COL + 32 * c2, oe);
        if (w1) tmem_ld32(lane_base + O_COL + 64 + 32 * c2, oo);
        tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t cv[4], res[4];
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(cv[0]), "=r"(cv[1]), "=r"(cv[2]), "=r"(cv[3])
                       : "r"(vown + plane_off(BM, i, 4 * c2 + ch)));
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cv[e]));
            const int k = ch * 8 + e * 2;
            // (an accumulator the M tile never wrote counts as zero)
            const float e0 = w0 ? __uint_as_float(oe[k]) : 0.f, e1 = w0 ? __uint_as_float(oe[k + 1]) : 0.f;
            const float o0 = w1 ? __uint_as_float(oo[k]) : 0.f, o1 = w1 ? __uint_as_float(oo[k + 1]) : 0.f;
            res[e] = pack_bf16x2((e0 * a_e + o0 * a_o + pown * c.x) * inv, (e1 * a_e + o1 * a_o + pown * c.y) * inv);
          }
          if (m <= p.T) dst[4 * c2 + ch] = make_uint4(res[0], res[1], res[2], res[3]);
        }
      }
      // the last read of O in TMEM: the next M tile's value MMAs may start
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(o_empty);
        mbar_arrive(&own_empty[sb2]);
      }
      if (m <= p.T && p.lse) p.lse[row] = (mf + log2f(den)) * 0.69314718055994531f;
    }
    if (!ok && lane == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
  } else {
    // ======================= softmax warps =======================
    // warp w: TMEM lane quarter w % 4 and the key tiles j (counted over the
    // block's whole run) with j mod 2 == w / 4, all 64 columns of each, with
    // its own running max and sum and its own O accumulator (columns O_COL +
    // 64 (w / 4)); the epilogue merges the two.  The two warps of a lane
    // quarter never wait for each other; buffer j mod 4 is always used by the
    // same warps, so they take its mbarrier phases in order.
    const int qw = warp & 3, par = warp >> 2;
    const int i = qw * 32 + lane;              // row of the M tile = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    const uint32_t ocol = O_COL + 64 * par;
    const float sl2 = p.scale_log2;
    uint32_t tc = 0, kc = 0;
    for (int o; (o = tile_index(tc, blockIdx.x, G)) < p.n_mtiles; ++tc) {
      const Tile t = tile_of(p, o);
      const int m = t.m0 + i;
      const int vis = (int)group_of(m, p.s) - 1;  // completed groups the query sees
      float m_run = -INFINITY, l = 0.f;
      bool first = true;  // this warp's first key tile of the M tile
      for (int kt = 0; kt < t.nkt; ++kt) {
        const uint32_t j = kc + kt;
        if ((int)(j & 1) != par) continue;
        const int sb = j % NSB;
        if (ok && !warp_wait(&s_full[sb], (j / NSB) & 1)) ok = false;
        tc_fence_after();
        uint32_t sr[64];  // the tile's 64 scores, both loads in flight
        tmem_ld32(lane_base + s_col(sb), *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(lane_base + s_col(sb) + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_wait_ld();
        const int nvis = vis - kt * BN;
        float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 64; ++c) {  // masked and scaled in place
          const float xc = c < nvis ? __uint_as_float(sr[c]) * sl2 : -INFINITY;
          sr[c] = __float_as_uint(xc);
          mq[c & 3] = fmaxf(mq[c & 3], xc);
        }
        const float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
        const bool grow = mx > m_run + 8.f;
        const bool resc = grow && m_run != -INFINITY;
        if (!first && __any_sync(0xffffffffu, resc)) {
          // rescale this parity's O once its previous value MMA (tile j - 2) has landed
          const uint32_t jp = j - 2;
          if (ok && !warp_wait(&p_empty[jp % NSB], (jp / NSB) & 1)) ok = false;
          tc_fence_after();
          const float a = resc ? exp2f(m_run - mx) : 1.f;
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {  // 16 columns at a time (the scores stay live)
            uint32_t ov[16];
            tmem_ld16(lane_base + ocol + 16 * c4, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * a);
            tmem_st16(lane_base + ocol + 16 * c4, ov);
          }
          tmem_wait_st();
          l *= a;
        }
        if (grow) m_run = mx;
        first = false;
        const float mref = m_run == -INFINITY ? 0.f : m_run;
        float lq[4] = {0.f, 0.f, 0.f, 0.f};
        // bf16 P over the tile's first 32 S columns (this warp alone read them)
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float p0 = ex2_approx(__uint_as_float(sr[32 * h2 + c]) - mref);
            const float p1 = ex2_approx(__uint_as_float(sr[32 * h2 + c + 1]) - mref);
            lq[(c >> 1) & 3] += p0 + p1;
            pk[c >> 1] = pack_bf16x2(p0, p1);
          }
          tmem_st16(lane_base + s_col(sb) + 16 * h2, pk);
        }
        l += (lq[0] + lq[1]) + (lq[2] + lq[3]);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[sb]);
      }
      const int sb2 = tc & 1;
      if (ok && tc >= 2 && !warp_wait(&stat_empty[sb2], ((tc >> 1) & 1) ^ 1)) ok = false;
      xl[(sb2 * 2 + par) * BM + i] = l;
      xm[(sb2 * 2 + par) * BM + i] = m_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(&stat_full[sb2]);
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

cudaLaunchAttribute pdl_attr() {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

}  // namespace utc

size_t prefill_unabs_tc_smem() { return utc::SMEM_USED + 1024; }

cudaError_t launch_prefill_unabs_tc(const UnabsTcLaunch& a, int grid, cudaStream_t st) {
  const size_t smem = prefill_unabs_tc_smem();
  static uint64_t done_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(done_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(utc::prefill_unabs_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev < 64) done_mask |= 1ull << dev;
  }
  utc::Maps mp;
  mp.q = a.q;
  mp.qr = a.qr;
  mp.k_own = a.k_own;
  mp.v_own = a.v_own;
  mp.kr_own = a.kr_own;
  mp.k_grp = a.k_grp;
  mp.v_grp = a.v_grp;
  mp.kr_grp = a.kr_grp;
  utc::Params p;
  p.B = a.B;
  p.T = a.T;
  p.H = a.H;
  p.s = a.s;
  p.n_mtiles = a.B * a.H * ((a.T + utc::BM - 1) / utc::BM);
  p.scale_log2 = a.scale_log2;
  p.out = a.out;
  p.lse = a.lse;
  p.dev_err = a.dev_err;
  cudaLaunchAttribute attr[1] = {utc::pdl_attr()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(utc::NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, utc::prefill_unabs_tc_kernel, mp, p);
}

}  // namespace mtla
