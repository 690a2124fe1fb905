// Stride-aware masked parallel forward on the 5th-generation tensor cores
// (tcgen05 + TMEM), bf16 with H = 8, r = 256, d_R = 32.
//
// What it computes (MTLA paper notes, "Key designs: stride-aware causal mask"
// and "decoupled RoPE with temporal compression"; Figure 2(c) of the abstract
// page): query m (1-based) of sequence b, head h, attends the columns n of the
// running merge C_hat' with n == m, or n < m and n mod s == 0.  The columns
// n = g s (g < ceil(m/s)) are the completed groups, i.e. the compressed cache
// rows C_hat_g; the only other column is the query's own partial row C_hat'_m.
// So: out[m, h] = softmax over {C_hat_1 .. C_hat_{ceil(m/s)-1}, C_hat'_m} of
// (q_abs . c_hat + q_rope . k_hat^R) / sqrt(d_h), weighting the latent parts.
//
// Design (B200):
//  * An M tile is 16 consecutive queries x 8 heads = 128 rows (the heads share
//    every key, so each key tile is loaded once for all of them); a key tile is
//    64 completed groups, read straight out of C_hat' through a 4-D tensor map
//    whose row stride is s rows.  Queries, keys and the 16 own rows land as
//    nine [rows x 64 B] planes with the 64-byte swizzle: the canonical K-major
//    operand layout for the score MMA and, for the latent planes, the
//    MN-major operand layout for the value MMA (the key tile is also V).
//    The own rows are read from global memory (L1 / L2): four key stages fill
//    the shared memory that a copy of them would take.
//  * Scores S = Q K^T (M 128, N 64, K 288) and values O += P V (M 128, N 256,
//    K 64) are tcgen05.mma ops with fp32 accumulators in TMEM (four 64-column
//    S / P buffers, O 256 columns: all 512 columns).  A score warp and a value
//    warp issue them, each as soon as its inputs are ready, so the tensor pipe
//    holds the next group before the current one ends.  Only complete groups
//    up to the staircase are visited, so no tile is empty.
//  * Eight softmax warps, two per TMEM lane quarter: warps w and w + 4 own
//    the same 32 (query, head) rows (TMEM lanes) and split the key tile's 64
//    columns and O's 256 columns between them, so each SMSP runs two of them.
//    Per tile the pair exchanges row maxima through shared memory (a 64-thread
//    named barrier) and makes the same lazy-rescale decision (O is rescaled in
//    TMEM only when the running max grows by more than 2^8); the row sums stay
//    per half until the epilogue.  The own-row score is taken when the M tile
//    starts, so the query tile is free for the next M tile as soon as its last
//    score MMA completes.  Masking, online softmax, and bf16 P written
//    back into the tile's S columns of TMEM (tcgen05.st), from where the value
//    MMA reads it as its A operand: no shared-memory round trip and no proxy
//    fence.  The epilogue adds the own-row term and writes bf16 out.
//  * One TMA warp, two MMA warps, mbarrier pipelines; a persistent grid visits
//    the M tiles heaviest first, in rounds of alternating direction.
#include "kernels.cuh"

namespace mtla {
namespace ptc {

constexpr int H = 8, R = 256, DR = 32, D = R + DR;
constexpr int QM = 16;                 // query positions per M tile
constexpr int BM = QM * H;             // 128 rows
constexpr int BN = 64;                 // groups per key tile
constexpr int NPL = D / 32;            // 9 planes of 32 elements
constexpr int QPL = BM * 64;           // bytes of one query plane (8192)
constexpr int KPL = BN * 64;           // bytes of one key plane (4096)
constexpr int SPL = QM * 64;           // bytes of one own-row plane (1024)
constexpr int QBYTES = NPL * QPL;      // 73728
constexpr int KBYTES = NPL * KPL;      // 36864
constexpr int SBYTES = NPL * SPL;      // 9216
constexpr int KS = 3;                  // key-tile stages
constexpr int SMW = 8;                 // softmax warps: two per TMEM lane quarter
constexpr int EPW = 4;                 // epilogue warps: one per TMEM lane quarter
constexpr int NT = 32 * (SMW + 4 + EPW);  // + TMA warp, score-MMA warp, value-MMA warp, own-row warp, epilogue
constexpr int TMA_WARP = SMW, SMMA_WARP = SMW + 1, PMMA_WARP = SMW + 2, DOT_WARP = SMW + 3, EPI_WARP0 = SMW + 4;
static_assert(EPI_WARP0 % 4 == 0, "epilogue warp e reads TMEM lane quarter e");
constexpr uint32_t TMEM_COLS = 512;
constexpr int NSB = 4;                 // S / P buffers in TMEM (64 columns each)
constexpr uint32_t O_COL = 256;
__host__ __device__ constexpr uint32_t s_col(int b) { return 64u * (uint32_t)b; }
static_assert(NSB * 64 <= (int)O_COL, "S buffers below O");
constexpr uint32_t IDESC_S = umma_idesc_bf16(BM, BN, false, false);
constexpr uint32_t IDESC_O = umma_idesc_bf16(BM, R, false, true);

constexpr int OST_BYTES = 32 * 64;     // output staging of one epilogue warp: 32 rows x 32 channels bf16

constexpr size_t OFF_Q = 0;
constexpr size_t OFF_SELF = OFF_Q + QBYTES;              // two own-row buffers (M tile parity)
constexpr size_t OFF_K = OFF_SELF + 2 * SBYTES;          // KS stages
constexpr size_t OFF_OST = OFF_K + (size_t)KS * KBYTES;  // EPW output staging blocks
constexpr size_t OFF_XCH = OFF_OST + (size_t)EPW * OST_BYTES;  // row maxima, sums, final maxima, own-row scores
constexpr size_t OFF_BAR = OFF_XCH + 2 * 2 * BM * 4 + 2 * 2 * BM * 4 + 2 * BM * 4 + 2 * BM * 4;
constexpr int NBAR = 2 + 12 + 2 * KS + 3 * NSB + 3;
constexpr size_t OFF_TMEM = OFF_BAR + NBAR * 8;
constexpr size_t SMEM_USED = OFF_TMEM + 16;
static_assert(OFF_K % 1024 == 0 && OFF_SELF % 1024 == 0 && OFF_OST % 1024 == 0, "tile bases must be 1024-aligned");

size_t smem_bytes() { return SMEM_USED + 1024; }
static_assert(SMEM_USED + 1024 <= 232448, "one block's shared memory (227 KB)");

struct Params {
  int B, T, s;
  int n_mtiles;            // B * T / QM
  float scale_log2;        // log2(e) / sqrt(d_h)
  __nv_bfloat16* out;      // [B, T, H, R]
  int32_t* dev_err;
};


// 16-byte chunk ch (0..35) of row `row` inside a plane-layout tile whose planes
// hold `rows` rows: plane ch / 4, 64-byte swizzle phase (row / 2) mod 4
__device__ __forceinline__ uint32_t plane_off(int rows, int row, int ch) {
  return (uint32_t)(ch >> 2) * (uint32_t)(rows * 64) + (uint32_t)row * 64u +
         ((((uint32_t)ch & 3u) ^ (((uint32_t)row >> 1) & 3u)) << 4);
}

// work of an M tile, heaviest first: index o -> (b, first query m0 1-based, key tiles)
struct Tile {
  int b, m0, nkt;
};
// 2^x with the hardware approximation (relative error about 2^-22; results
// below 2^-126 flush to zero, 2^-inf = 0): the probabilities' exponentials
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 16 consecutive 32-bit TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
      "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}


// mbarrier wait taken by every lane of a warp, with a warp-uniform result:
// the tcgen05.ld / st that follow are warp-collective, so no lane may leave
// the common path on its own
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

// M tile that block x takes in its round r: tiles are numbered heaviest
// first and the rounds alternate direction (x, then G - 1 - x), so each block
// gets a heavy and a light tile in turn and all blocks end close together;
// increasing in r for every block
__device__ __forceinline__ int tile_index(int r, int x, int G) { return r * G + ((r & 1) ? G - 1 - x : x); }

// A sequence's last M tile is ragged when T is not a multiple of QM: its rows
// past query T read finite values (the next sequence's rows, or the TMA fill
// past the last one) and are never stored.
__device__ __forceinline__ Tile tile_of(const Params& p, int o) {
  const int per_seq = (p.T + QM - 1) / QM;
  Tile t;
  t.b = o % p.B;
  const int mb = per_seq - 1 - o / p.B;
  t.m0 = mb * QM + 1;
  const int m_last = t.m0 + QM - 1 < p.T ? t.m0 + QM - 1 : p.T;
  const int vis_max = (int)group_of(m_last, p.s) - 1;  // groups seen by the tile's last query
  t.nkt = (vis_max + BN - 1) / BN;
  return t;
}

__global__ void __launch_bounds__(NT, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap rmap,
                  const __grid_constant__ CUtensorMap smap, const __grid_constant__ CUtensorMap kmap,
                  const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* const q_full = bar + 0;
  uint64_t* const q_empty = bar + 1;            // the tile's last score MMA + the own-row warp
  uint64_t* const self_full = bar + 2;          // [2] own rows of M tile parity b landed
  uint64_t* const self_empty = bar + 4;         // [2] the epilogue is done with them
  uint64_t* const dot_full = bar + 6;           // [2] own-row scores written
  uint64_t* const dot_empty = bar + 8;          // [2] the epilogue has read them
  uint64_t* const stat_full = bar + 10;         // [2] the softmax has written a tile's row maxima and sums
  uint64_t* const stat_empty = bar + 12;        // [2] the epilogue has read them
  uint64_t* const k_full = bar + 14;            // [KS]
  uint64_t* const k_empty = bar + 14 + KS;      // [KS]
  uint64_t* const s_full = bar + 14 + 2 * KS;   // [NSB]
  uint64_t* const p_full = s_full + NSB;        // [NSB]
  uint64_t* const p_empty = s_full + 2 * NSB;   // [NSB]: the value MMA has read P (and so the buffer is free)
  uint64_t* const o_full = s_full + 3 * NSB;
  uint64_t* const o_empty = o_full + 1;
  uint64_t* const mma_done = o_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
  float* xmax = reinterpret_cast<float*>(sm + OFF_XCH);                 // [2 parity][2 halves][BM]
  float* xl = reinterpret_cast<float*>(sm + OFF_XCH + 4 * BM * 4);      // [2 parity][2 halves][BM]: row sums
  float* xdot = reinterpret_cast<float*>(sm + OFF_XCH + 8 * BM * 4);    // [2 parity][BM]: own-row scores
  float* xm = reinterpret_cast<float*>(sm + OFF_XCH + 10 * BM * 4);     // [2 parity][BM]: final row maxima
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 2);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&self_full[b], 1);
      mbar_init(&self_empty[b], EPW);
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
      mbar_init(&p_full[i], SMW);
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
    prefetch_tmap(&qmap);
    prefetch_tmap(&rmap);
    prefetch_tmap(&smap);
    prefetch_tmap(&kmap);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t sQ = smem_u32(sm + OFF_Q);
  const uint32_t sSelf = smem_u32(sm + OFF_SELF);
  const uint32_t sK = smem_u32(sm + OFF_K);
  const int G = gridDim.x;
  bool ok = true;

  if (warp == TMA_WARP) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      uint32_t tc = 0, kc = 0, q_issued = 0;
      for (int o; (o = tile_index(tc, blockIdx.x, G)) < p.n_mtiles && ok; ++tc) {
        const Tile t = tile_of(p, o);
        const int qrow0 = ((t.b * p.T) + (t.m0 - 1)) * H;  // first row of [B*T*H, .]
        const int crow0 = t.b * p.T + (t.m0 - 1);         // first own row of [B*T, .]
        const int sb2 = tc & 1;
        if (tc > 0 && !mbar_wait(q_empty, (tc - 1) & 1)) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, QBYTES);
        tma_load_3d(sm + OFF_Q, &qmap, 0, qrow0, 0, q_full);
        tma_load_2d(sm + OFF_Q + 8 * QPL, &rmap, 0, qrow0, q_full);
        q_issued = tc + 1;
        // own rows into the buffer of this tile's parity, once the epilogue of
        // tile tc - 2 is done with it
        if (tc >= 2 && !mbar_wait(&self_empty[sb2], ((tc >> 1) & 1) ^ 1)) { ok = false; break; }
        mbar_arrive_expect_tx(&self_full[sb2], SBYTES);
        tma_load_3d(sm + OFF_SELF + sb2 * SBYTES, &smap, 0, crow0, 0, &self_full[sb2]);
        for (int kt = 0; kt < t.nkt; ++kt, ++kc) {
          const int st = kc % KS;
          if (kc >= KS && !mbar_wait(&k_empty[st], ((kc / KS) & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[st], KBYTES);
          tma_load_4d(sm + OFF_K + st * KBYTES, &kmap, 0, kt * BN, 0, t.b, &k_full[st]);
        }
      }
      if (!ok) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
      // drain: no copy may still be writing shared memory when the block exits
      if (q_issued) mbar_wait(q_full, (q_issued - 1) & 1);
      for (uint32_t u = q_issued > 2 ? q_issued - 2 : 0; u < q_issued; ++u) mbar_wait(&self_full[u & 1], (u >> 1) & 1);
      for (uint32_t j = kc > (uint32_t)KS ? kc - KS : 0; j < kc; ++j) mbar_wait(&k_full[j % KS], (j / KS) & 1);
    }
  } else if (warp == DOT_WARP) {
    // ======================= own-row scores =======================
    // x_self = q_abs . c_hat'_m + q^R . k_hat^R'_m for the 128 rows of the M
    // tile (lane: rows lane + 32 r), from the query tile and the own rows in
    // shared memory, while the key tiles run.  Then this warp is done with Q.
    for (uint32_t tc = 0; tile_index(tc, blockIdx.x, G) < p.n_mtiles; ++tc) {
      const int sb2 = tc & 1;
      if (ok && !warp_wait(q_full, tc & 1)) ok = false;
      if (ok && !warp_wait(&self_full[sb2], (tc >> 1) & 1)) ok = false;
      // the epilogue of tile tc - 2 has read this parity's scores
      if (ok && tc >= 2 && !warp_wait(&dot_empty[sb2], ((tc >> 1) & 1) ^ 1)) ok = false;
      const uint32_t selfb = sSelf + sb2 * SBYTES;
#pragma unroll 1
      for (int r = 0; r < BM / 32; ++r) {
        const int i = r * 32 + lane;
        const int srow = i / H;
        float dot = 0.f;
#pragma unroll 4
        for (int ch = 0; ch < D / 8; ++ch) {
          uint32_t qv[4], cv[4];
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(qv[0]), "=r"(qv[1]), "=r"(qv[2]), "=r"(qv[3])
                       : "r"(sQ + plane_off(BM, i, ch)));
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(cv[0]), "=r"(cv[1]), "=r"(cv[2]), "=r"(cv[3])
                       : "r"(selfb + plane_off(QM, srow, ch)));
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qv[e]));
            const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cv[e]));
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
    // Two warps feed the one tensor pipe: the score warp issues S(j) as soon
    // as its key tile has landed and its TMEM buffer is free, the value warp
    // issues O += P(j) V(j) as soon as the softmax has written P(j), so the
    // pipe holds the next group before the current one ends.  Each warp runs
    // its loop with all 32 lanes (warp-uniform operands); one elected lane
    // issues the MMAs and the commits that track them.  Operand descriptors
    // are built once; a K step or a stage moves only the 14-bit start-address
    // field (shared addresses are below 2^18, no carry).
    const bool scores = warp == SMMA_WARP;
    const uint64_t dq0 = umma_desc(sQ, 16, 512, 4);
    const uint64_t dk0 = umma_desc(sK, 16, 512, 4);
    const uint64_t dv0 = umma_desc(sK, KPL, 512, 4);
    uint32_t tc = 0, kc = 0;
    for (int o; (o = tile_index(tc, blockIdx.x, G)) < p.n_mtiles && ok; ++tc) {
      const Tile t = tile_of(p, o);
      if (scores) {
        // S(j) = Q K(j)^T into buffer j mod NSB, once the value MMA of tile
        // j - NSB has read that buffer (which also means its scores were read)
        if (!warp_wait(q_full, tc & 1)) { ok = false; break; }
        for (int kt = 0; kt < t.nkt && ok; ++kt) {
          const uint32_t j = kc + kt;
          const int st = j % KS, sb = j % NSB;
          if (!warp_wait(&k_full[st], (j / KS) & 1)) { ok = false; break; }
          if (j >= NSB && !warp_wait(&p_empty[sb], ((j / NSB) & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t ad = dq0 + (uint64_t)(((kk >> 1) * QPL + (kk & 1) * 32) >> 4);
              const uint64_t bd = dk0 + (uint64_t)((st * KBYTES + (kk >> 1) * KPL + (kk & 1) * 32) >> 4);
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
        // O += P(j) V(j): P from TMEM over the tile's S columns, V = the
        // latent planes of its key tile.  Its completion frees the key stage
        // (the scores of tile j completed before the softmax wrote P(j)).
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
              const uint64_t bd = dv0 + (uint64_t)((st * KBYTES + kk * 16 * 64) >> 4);
              umma_bf16_ts(tmem + O_COL, pa, bd, IDESC_O, (kt > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&k_empty[st]);
            umma_commit(&p_empty[pb]);
          }
          __syncwarp();
        }
        // a tile without key tiles still waits for the epilogue of tile
        // tc - 1 before it completes o_full: otherwise o_full could complete
        // twice before the epilogue waits on the earlier phase
        if (ok && t.nkt == 0 && tc > 0 && !warp_wait(o_empty, (tc - 1) & 1)) ok = false;
        if (ok) {
          if (elect_one()) umma_commit(o_full);
          __syncwarp();
        }
      }
      kc += t.nkt;
    }
    if (!ok && lane == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
    // every MMA of both warps has completed before TMEM is released
    if (elect_one()) umma_commit(mma_done);
    __syncwarp();
    warp_wait(mma_done, 0);
  } else if (warp >= EPI_WARP0) {
    // ======================= epilogue warps =======================
    // warp EPI_WARP0 + e owns rows 32 e .. 32 e + 31 (TMEM lane quarter e) and
    // all 256 channels: out = (alpha O + p_self c_hat'_m) / (alpha l + p_self)
    // with the own row as one more key, in bf16.  It runs while the softmax
    // warps start the next M tile; that tile's value MMAs wait until O has
    // been read.  O is read 64 channels at a time; each 32 x 32 block goes
    // through a staging block in shared memory (64-byte swizzle, no bank
    // conflicts either way) so that every store writes 64 contiguous bytes
    // of 8 rows.
    const int qe = warp - EPI_WARP0;
    const int i = qe * 32 + lane;
    const int srow = i / H;
    const uint32_t lane_base = tmem + ((uint32_t)(qe * 32) << 16);
    const uint32_t ost = smem_u32(sm + OFF_OST + (size_t)qe * OST_BYTES);
    const float sl2 = p.scale_log2;
    uint32_t tc = 0;
    for (int o; (o = tile_index(tc, blockIdx.x, G)) < p.n_mtiles; ++tc) {
      const Tile t = tile_of(p, o);
      const int sb2 = tc & 1;
      if (ok && !warp_wait(&stat_full[sb2], (tc >> 1) & 1)) ok = false;
      if (ok && !warp_wait(&dot_full[sb2], (tc >> 1) & 1)) ok = false;
      if (ok && !warp_wait(&self_full[sb2], (tc >> 1) & 1)) ok = false;
      const float m_run = xm[sb2 * BM + i];
      const float lt = xl[(sb2 * 2 + 0) * BM + i] + xl[(sb2 * 2 + 1) * BM + i];
      const float xs = xdot[sb2 * BM + i] * sl2;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&stat_empty[sb2]);
        mbar_arrive(&dot_empty[sb2]);
      }
      const float mf = fmaxf(m_run, xs);
      const float alpha = m_run == -INFINITY ? 0.f : exp2f(m_run - mf);
      const float pself = exp2f(xs - mf);
      const float inv = 1.f / (lt * alpha + pself);
      if (ok && !warp_wait(o_full, tc & 1)) ok = false;
      tc_fence_after();
      const uint32_t selfb = sSelf + sb2 * SBYTES;
      // this warp's 32 output rows, and the row / 16-byte piece each lane
      // stores in the transposed pass
      __nv_bfloat16* const obase = p.out + ((size_t)((t.b * p.T) + (t.m0 - 1)) * H + 32 * qe) * R;
      const int tr = lane >> 2, tq = lane & 3;
#pragma unroll 1
      for (int c2 = 0; c2 < R / 64; ++c2) {
        uint32_t ov[64];
        if (t.nkt > 0) {
          tmem_ld32(lane_base + O_COL + c2 * 64, *reinterpret_cast<uint32_t(*)[32]>(&ov[0]));
          tmem_ld32(lane_base + O_COL + c2 * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&ov[32]));
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 64; ++e) ov[e] = 0u;
        }
        if (c2 == R / 64 - 1) {
          // the last read of O in TMEM: the next M tile's value MMAs may start
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_empty);
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int ch = 2 * c2 + hh;          // 32-channel block
          uint32_t res[16];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t cv[4];
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(cv[0]), "=r"(cv[1]), "=r"(cv[2]), "=r"(cv[3])
                         : "r"(selfb + plane_off(QM, srow, ch * 4 + q4)));
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cv[e]));
              const int k = hh * 32 + q4 * 8 + e * 2;
              const float v0 = (__uint_as_float(ov[k]) * alpha + pself * c.x) * inv;
              const float v1 = (__uint_as_float(ov[k + 1]) * alpha + pself * c.y) * inv;
              res[q4 * 4 + e] = pack_bf16x2(v0, v1);
            }
          }
          __syncwarp();                        // the previous block's transposed reads are done
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const uint32_t off = (uint32_t)lane * 64u + ((((uint32_t)q4) ^ (((uint32_t)lane >> 1) & 3u)) << 4);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(ost + off), "r"(res[4 * q4]),
                         "r"(res[4 * q4 + 1]), "r"(res[4 * q4 + 2]), "r"(res[4 * q4 + 3]) : "memory");
          }
          __syncwarp();
#pragma unroll
          for (int k8 = 0; k8 < 4; ++k8) {
            const int r = 8 * k8 + tr;         // row of the block this lane stores
            if (t.m0 + 4 * qe + k8 > p.T) break;  // query past the prompt (ragged last tile)
            uint32_t w[4];
            const uint32_t off = (uint32_t)r * 64u + ((((uint32_t)tq) ^ (((uint32_t)r >> 1) & 3u)) << 4);
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                         : "r"(ost + off));
            *reinterpret_cast<uint4*>(obase + (size_t)r * R + ch * 32 + tq * 8) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&self_empty[sb2]);
    }
    if (!ok && lane == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
  } else {
    // ======================= softmax warps =======================
    // warp w: TMEM lane quarter w % 4 (rows 32 (w % 4) .. +31) and half w / 4
    // of the key tile's 64 columns and of O's 256 columns.  Warps w and w + 4
    // own the same rows and agree on the running max every tile (64-thread
    // named barrier per pair; the exchange buffers alternate with the tile, so
    // neither can overwrite a value its partner has not read).  A wait that
    // times out only stops further waiting: every warp still takes every pair
    // barrier, so a pair never waits for a warp that left.
    const int qw = warp & 3, hf = warp >> 2;
    const int i = qw * 32 + lane;              // row of the M tile = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    const float sl2 = p.scale_log2;
    uint32_t tc = 0, kc = 0;
    for (int o; (o = tile_index(tc, blockIdx.x, G)) < p.n_mtiles; ++tc) {
      const Tile t = tile_of(p, o);
      const int m = t.m0 + i / H;              // this row's query (1-based)
      const int vis = (int)group_of(m, p.s) - 1;  // completed groups it sees
      float m_run = -INFINITY, l = 0.f;        // l: this half's sum
      for (int kt = 0; kt < t.nkt; ++kt) {
        const uint32_t j = kc + kt;
        const int sb = j % NSB, xb = j & 1;    // TMEM buffer; exchange-buffer parity
        if (ok && !warp_wait(&s_full[sb], (j / NSB) & 1)) ok = false;
        tc_fence_after();
        uint32_t sr[32];
        tmem_ld32(lane_base + s_col(sb) + 32 * hf, sr);
        tmem_wait_ld();
        // mask (group kt*BN + 32 hf + c + 1 visible iff <= vis) and scale
        const int nvis = vis - kt * BN - 32 * hf;
        float x[32];
        float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // four independent chains
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = c < nvis ? __uint_as_float(sr[c]) * sl2 : -INFINITY;
          mq[c & 3] = fmaxf(mq[c & 3], x[c]);
        }
        const float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
        xmax[(xb * 2 + hf) * BM + i] = mx;
        tc_fence_before();
        named_bar(1 + qw, 64);
        tc_fence_after();
        const float rmx = fmaxf(mx, xmax[(xb * 2 + (hf ^ 1)) * BM + i]);
        // the running max moves by more than 2^8: rescale l and, once the
        // previous value MMA has landed, this half of the row of O in TMEM
        // (warp-collective: the whole warp rescales when any row needs it)
        const bool grow = rmx > m_run + 8.f;
        const bool resc = grow && m_run != -INFINITY;
        if (kt > 0 && __any_sync(0xffffffffu, resc)) {
          const uint32_t jp = j - 1;
          if (ok && !warp_wait(&p_empty[jp % NSB], (jp / NSB) & 1)) ok = false;
          tc_fence_after();
          const float a = resc ? exp2f(m_run - rmx) : 1.f;
#pragma unroll 1
          for (int ch = 0; ch < R / 64; ++ch) {
            uint32_t ov[32];
            const uint32_t col = O_COL + 128 * hf + 32 * ch;
            tmem_ld32(lane_base + col, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * a);
            tmem_st32(lane_base + col, ov);
          }
          tmem_wait_st();
          l *= a;
        }
        if (grow) m_run = rmx;
        // probabilities (relative to the possibly stale max, at most 2^8)
        // (a row with nothing visible yet keeps m_run = -inf; its x are all -inf)
        const float mref = m_run == -INFINITY ? 0.f : m_run;
        uint32_t pk[16];
        float lq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float p0 = ex2_approx(x[c] - mref);
          const float p1 = ex2_approx(x[c + 1] - mref);
          lq[(c >> 1) & 3] += p0 + p1;
          pk[c >> 1] = pack_bf16x2(p0, p1);
        }
        l += (lq[0] + lq[1]) + (lq[2] + lq[3]);
        // this half of P row i into TMEM over the tile's S columns (both halves'
        // S are loaded: the pair barrier above), bf16 pairs, for the value MMA
        tmem_st16(lane_base + s_col(sb) + 16 * hf, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[sb]);
      }
      // ---- hand the tile to the epilogue warps: this half's row sum and the
      // running max (both halves hold the same), once the epilogue of tile
      // tc - 2 has read this parity's slots
      const int sb2 = tc & 1;
      if (ok && tc >= 2 && !warp_wait(&stat_empty[sb2], ((tc >> 1) & 1) ^ 1)) ok = false;
      xl[(sb2 * 2 + hf) * BM + i] = l;
      if (hf == 0) xm[sb2 * BM + i] = m_run;
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

}  // namespace ptc

cudaError_t launch_prefill_tc(const ptc::Params& p, const CUtensorMap& qmap, const CUtensorMap& rmap,
                              const CUtensorMap& smap, const CUtensorMap& kmap, int grid, cudaStream_t st) {
  const size_t smem = ptc::smem_bytes();
  static uint64_t done_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(done_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(ptc::prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev < 64) done_mask |= 1ull << dev;
  }
  ptc::prefill_tc_kernel<<<grid, ptc::NT, smem, st>>>(qmap, rmap, smap, kmap, p);
  return cudaGetLastError();
}

cudaError_t launch_prefill_tc_args(const PrefillTcLaunch& a, const CUtensorMap& qmap, const CUtensorMap& rmap,
                                   const CUtensorMap& smap, const CUtensorMap& kmap, int grid, cudaStream_t st) {
  ptc::Params p;
  p.B = a.B;
  p.T = a.T;
  p.s = a.s;
  p.n_mtiles = a.B * ((a.T + ptc::QM - 1) / ptc::QM);
  p.scale_log2 = a.scale_log2;
  p.out = reinterpret_cast<__nv_bfloat16*>(a.out);
  p.dev_err = a.dev_err;
  return launch_prefill_tc(p, qmap, rmap, smap, kmap, grid, st);
}

}  // namespace mtla
