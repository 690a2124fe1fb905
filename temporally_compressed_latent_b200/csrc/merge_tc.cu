// Running merge C_hat' of a prompt on the 5th-generation tensor cores, for bf16
// caches with r = 256, d_R = 32 and a stride s <= 32.
//
// What it computes (MTLA paper notes, "Key designs: hyper-network temporal
// merging" and "stride-aware causal mask"; Figure 2(c) of the abstract page):
// for every token n (0-based) of sequence b, with group j = n / s + 1,
//   w_n     = sigmoid((c_n W_c + b_c) * P[j-1])          (channel-wise, D = 288)
//   C'_n    = sum of w_i * [c_i ; k^R_i] over the tokens i <= n of n's group,
// stored as c_partial[b, n]; the last token of every group (or of the prompt)
// also writes its C'_n as compressed-cache row j - 1.
//
// Design (B200):
//  * The gate pre-activations are a dense contraction (256 latents in, 288
//    channels out per token), so they run as tcgen05.mma with fp32
//    accumulators in TMEM, transposed: D[channel, token] = W_c^T c^T.  The
//    channels sit on the TMEM lanes, so an epilogue thread owns one channel;
//    the running merge inside a group is a sum along the thread's own
//    columns.
//  * The 288 channels form three tiles of 96, one per CTA (MMA rows 96..127
//    are padding).  Each CTA rounds its 96 columns of W_c to bf16 once, the
//    cache's own precision, and keeps them in TMEM as the MMA's A operand
//    (two bf16 of K per column); the latents are bf16 already and the sums
//    are fp32.  The TMA warp streams the first tiles while W_c is placed.
//  * A token tile is floor(128 / s) * s tokens of one sequence, so groups
//    never cross tiles.  Every input of the epilogue arrives by TMA: the
//    latent tile (four K blocks of 128 rows x 64 latents, 128-byte swizzle,
//    eight stages: two tiles in flight), which the MMA reads and the
//    epilogue reads again for the gated entries before releasing it; the
//    RoPE keys of the tile (RoPE channel tile only, two buffers); the P rows
//    of the tile's groups for the CTA's channels (one buffer).  A CTA takes a
//    contiguous range of tiles ordered by position, then sequence, so
//    consecutive tiles mostly share their P rows and P is loaded again only
//    when the position changes.  The three channel tiles of a token tile run
//    in neighbouring CTAs, so the second and third reads of the latent tile
//    hit L2.
//  * The epilogue stages C_hat' rows and the closing rows in shared memory.
//    With a stride that divides 16 each warp stages its own 32 channels of
//    its 32 rows and sends them by TMA stores (maps [B][T][D] and
//    [B][groups][D], clipping rows past the prompt's end), so no warp waits
//    for another; otherwise a quarter's three warps stage its rows together
//    and write them with 16-byte stores after a barrier.
//  * Roles (16 warps, four per SM sub-partition): twelve epilogue warps, four
//    per live TMEM lane quarter, each over a group-aligned quarter of the
//    tile's tokens; the padding quarter's warps take the TMA producer and the
//    MMA issuer (one elected lane issues).  The accumulator is double-buffered
//    in TMEM so a tile's epilogue overlaps the next tile's MMAs.  Per chunk of
//    16 tokens the epilogue loads everything first, then forms the gates and
//    gated entries (independent across tokens), then the group sums and the
//    staged stores.  Strides 1, 2, 3, 4, 8 and 16 have their own instances,
//    in which the positions and divisions are constants (and, for the
//    strides that divide 16, every chunk starts a group).
#include "kernels.cuh"

namespace mtla {
namespace mtc {

constexpr int R = 256, DR = 32, D = R + DR;
constexpr int CT = 3;                 // channel tiles
constexpr int NCT = D / CT;           // channels per tile: 96
constexpr int M = 128;                // MMA rows: the tile's channels, then padding
constexpr int NTOK = 128;             // MMA columns: token slots per tile
constexpr int KB = R / 64;            // K blocks of 64 latents (128-byte rows): 4
constexpr int BBLK = NTOK * 128;      // one K block of the latent tile: 16384 B
constexpr int KS = 2 * KB;            // latent stages: two tiles
constexpr int KRBLK = NTOK * DR * 2;  // one tile of RoPE keys: 8192 B
constexpr int NWARPS = 16, NT = 32 * NWARPS;
constexpr int NEPI = 4 * (NCT / 32);  // epilogue warps: four per live lane quarter (12)
constexpr int TMA_WARP = 3, MMA_WARP = 7;  // warps of the padding quarter
constexpr uint32_t TMEM_COLS = 512, ACC_STRIDE = 128, W_COL = 256;  // W^T: 128 columns (K / 2)
constexpr uint32_t IDESC = umma_idesc_bf16(M, NTOK, false, false);
constexpr int PROW = NCT * 4;                    // one staged P row (fp32): 384 B
constexpr int OROW = NCT * 2;                    // one staged output row (bf16): 192 B
constexpr int P_BYTES_MAX = NTOK * PROW;         // P rows of a tile at s = 1: 49152 B
constexpr int P_BYTES_S2 = (NTOK / 2) * PROW;    // at s >= 2 (at most 64 groups): 24576 B

constexpr size_t OFF_B = 0;
constexpr size_t OFF_KR = OFF_B + (size_t)KS * BBLK;
constexpr size_t OFF_X = OFF_KR + 2 * (size_t)KRBLK;  // P rows; at s >= 2 the closing rows follow them
constexpr size_t OFF_OUT = OFF_X + P_BYTES_MAX;
constexpr size_t OFF_BAR = OFF_OUT + (size_t)NTOK * OROW;
constexpr int NBAR = 2 * KS + 2 + 2 + 2 + 2 + 2 + 1;
constexpr size_t OFF_TMEM = OFF_BAR + NBAR * 8;
constexpr size_t SMEM_USED = OFF_TMEM + 16;
static_assert(BBLK % 1024 == 0 && OFF_KR % 1024 == 0 && OFF_X % 1024 == 0 && OFF_OUT % 1024 == 0,
              "stage and staging alignment");
static_assert(P_BYTES_S2 + (NTOK / 2) * OROW <= P_BYTES_MAX, "closing rows fit beside the P rows");
static_assert(NCT * CT == D && NCT <= M && NCT % 32 == 0 && OROW % 16 == 0 && PROW % 16 == 0, "channel tiles");

size_t smem_bytes() { return SMEM_USED + 1024; }

struct Params {
  int B, s, tt, tiles_per_seq, n_tiles;
  int64_t T, n_groups;
  const float* W_c;
  const float* b_c;
  __nv_bfloat16* cp;
  __nv_bfloat16* cache;
  int32_t* dev_err;
};

// mbarrier wait by every lane of a warp with a warp-uniform result (the
// tcgen05.ld that follow are warp-collective)
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

// 16 consecutive 32-bit TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr) : "memory");
}

// The gated entry v * sigmoid(z) = v / (1 + 2^(-z log2 e)).  The caller
// passes y = -z log2 e, formed as one fused multiply-add of the accumulator
// with -P log2 e and (b_c P)(-log2 e) (both once per group); the base-2
// exponential and the reciprocal are the hardware approximations (relative
// error near 2^-22 each), far below the bf16 rounding of what they scale.
// The fp32 paths of the library keep the correctly rounded sigmoid.
__device__ __forceinline__ float gated(float v, float y) {
  float e, r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(y));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.f + e));
  return v * r;
}
constexpr float kNegLog2e = -1.4426950408889634f;

// first column of part `part` (0..4) of a tile of tt tokens: group-aligned quarters
__device__ __forceinline__ int part_start(int part, int tt, int s) { return part >= 4 ? tt : ((part * tt / 4) / s) * s; }

// Tile u of the ordering by position, then sequence: (sequence, tile in it).
__device__ __forceinline__ void tile_of(int u, int B, int& b, int& tb) {
  tb = u / B;
  b = u - tb * B;
}

// S: the stride when it has its own instance (1, 2, 3, 4, 8, 16: positions
// and divisions fold to constants), else 0
template <int S>
__global__ void __launch_bounds__(NT, 1) merge_tc_kernel(const __grid_constant__ MergeMaps mp, const Params p) {
  // a tiled TMA store reads shared memory from a 128-byte aligned address:
  // each warp's staged rows (2 KB) and closing rows ((32 / S) x 64 B) must
  // start on one, and twelve of each fit the staging regions
  static_assert(S == 0 || 16 % S != 0 ||
                    (NTOK == 128 && OFF_OUT % 128 == 0 && (OFF_X + P_BYTES_S2) % 128 == 0 &&
                     ((32 / S) * 64) % 128 == 0 && 12 * 2048 <= NTOK * OROW &&
                     12 * (32 / S) * 64 <= P_BYTES_MAX - P_BYTES_S2),
                "TMA store sources of the warps");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* const k_full = bar;                // [KS]
  uint64_t* const k_empty = bar + KS;          // [KS]
  uint64_t* const acc_full = bar + 2 * KS;     // [2]
  uint64_t* const acc_empty = bar + 2 * KS + 2;  // [2]
  uint64_t* const kr_full = bar + 2 * KS + 4;    // [2]
  uint64_t* const kr_empty = bar + 2 * KS + 6;   // [2]
  uint64_t* const p_full = bar + 2 * KS + 8;
  uint64_t* const p_empty = bar + 2 * KS + 9;
  uint64_t* const mma_done = bar + 2 * KS + 10;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ct = blockIdx.x % CT;              // channel tile
  const int G = gridDim.x / CT;                // CTAs per channel tile
  const int j = blockIdx.x / CT;
  const int u_beg = (int)((int64_t)j * p.n_tiles / G), u_end = (int)((int64_t)(j + 1) * p.n_tiles / G);
  const bool has_rope = (ct + 1) * NCT > R;    // this channel tile holds the RoPE channels
  const int s = S > 0 ? S : p.s, tt = p.tt, gpt = tt / s;  // groups per tile
  const int q = warp & 3, part = warp >> 2;    // TMEM lane quarter; quarter of the tile's tokens
  const bool epi = q * 32 < NCT;               // an epilogue warp
  const int chl = q * 32 + lane;               // its channel inside the tile
  const int ch = ct * NCT + chl;               // and in the row of D channels

  // W^T, this warp's 32 TMEM columns (latents 64 part .. +63, two per
  // column) of its quarter's lanes: requested before anything else, while
  // the memory system is idle (all 64 loads in flight at once)
  float wv[64];
  if (epi) {
#pragma unroll
    for (int k = 0; k < 64; ++k) wv[k] = __ldg(p.W_c + (size_t)(64 * part + k) * D + ch);
  }

  if (tid == 0) {
    for (int i = 0; i < KS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], NEPI);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], NEPI);
      mbar_init(&kr_full[i], 1);
      mbar_init(&kr_empty[i], 4);              // the four warps of the RoPE lane quarter
    }
    mbar_init(p_full, 1);
    mbar_init(p_empty, NEPI);
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == TMA_WARP && lane == 0) {
    prefetch_tmap(&mp.c);
    prefetch_tmap(&mp.kr);
    prefetch_tmap(&mp.p);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  bool ok = true;

  if (warp == TMA_WARP) {
    // ======================= TMA producer (starts at once) =======================
    if (lane == 0) {
      uint32_t kc = 0, tc = 0, np = 0, kr_n = 0;
      int prev_tb = -1;
      for (int u = u_beg; u < u_end && ok; ++u, ++tc) {
        int b, tb;
        tile_of(u, p.B, b, tb);
        const int32_t row = (int32_t)((int64_t)b * p.T + (int64_t)tb * tt);
        // the latent stages first (the MMA waits on them), then the RoPE
        // keys, then the P rows when the position changes (their buffer is
        // free only once the epilogue has finished the previous tile)
        for (int kb = 0; kb < KB; ++kb, ++kc) {
          const int st = kc % KS;
          if (kc >= KS && !mbar_wait(&k_empty[st], ((kc / KS) & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[st], BBLK);
          // slots past the tile's tokens load rows that are never used
          tma_load_2d(sm + OFF_B + st * BBLK, &mp.c, kb * 64, row, &k_full[st]);
        }
        if (!ok) break;
        if (has_rope) {
          const int kb2 = tc & 1;
          if (tc >= 2 && !mbar_wait(&kr_empty[kb2], ((tc >> 1) & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&kr_full[kb2], KRBLK);
          tma_load_2d(sm + OFF_KR + kb2 * KRBLK, &mp.kr, 0, row, &kr_full[kb2]);
          ++kr_n;
        }
        if (tb != prev_tb) {  // the P rows of this position's groups
          if (np > 0 && !mbar_wait(p_empty, (np - 1) & 1)) { ok = false; break; }
          mbar_arrive_expect_tx(p_full, (uint32_t)(gpt * PROW));
          tma_load_2d(sm + OFF_X, &mp.p, ct * NCT, tb * gpt, p_full);
          ++np;
          prev_tb = tb;
        }
      }
      if (!ok) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
      // drain: no copy may still be writing shared memory when the block exits
      for (uint32_t i = kc > (uint32_t)KS ? kc - KS : 0; i < kc; ++i) mbar_wait(&k_full[i % KS], (i / KS) & 1);
      for (uint32_t i = kr_n > 2u ? kr_n - 2 : 0; i < kr_n; ++i) mbar_wait(&kr_full[i & 1], (i >> 1) & 1);
      if (np > 0) mbar_wait(p_full, (np - 1) & 1);
    }
  } else if (warp == MMA_WARP) {
    // ======================= MMA issuer =======================
    // The whole warp runs the loop (warp-uniform operands); one elected lane
    // issues the MMAs and the commits that track them.  The epilogue releases
    // the latent stages (it reads them too).
    named_bar(1, 32 * (NEPI + 1));  // W^T is in TMEM
    tc_fence_after();
    const uint32_t sB = smem_u32(sm + OFF_B);
    uint32_t kc = 0, tc = 0;
    for (int u = u_beg; u < u_end && ok; ++u, ++tc) {
      const int ab = tc & 1;
      if (tc >= 2 && !warp_wait(&acc_empty[ab], ((tc >> 1) & 1) ^ 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t dcol = tmem + ab * ACC_STRIDE;
      for (int kb = 0; kb < KB; ++kb, ++kc) {
        const int st = kc % KS;
        if (!warp_wait(&k_full[st], (kc / KS) & 1)) { ok = false; break; }
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = umma_desc(sB + st * BBLK + kk * 32, 16, 1024, 2);
            umma_bf16_ts(dcol, tmem + W_COL + (kb * 4 + kk) * 8, bd, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) umma_commit(&acc_full[ab]);
      __syncwarp();
    }
    if (!ok && lane == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
    // every MMA of this warp has completed before TMEM is released
    if (elect_one()) umma_commit(mma_done);
    __syncwarp();
    warp_wait(mma_done, 0);
  } else if (epi) {
    // ================= epilogue: gate, gated entry, group sums =================
    const bool rope = ch >= R;                       // warp-uniform
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    {
      // W^T into TMEM (its loads were issued at the kernel's start)
      uint32_t wp[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) wp[k] = pack_bf16x2(wv[2 * k], wv[2 * k + 1]);
      tmem_st32(lane_base + W_COL + 32 * part, wp);
      tmem_wait_st();
      tc_fence_before();
    }
    named_bar(1, 32 * (NEPI + 1));

    const float bc = __ldg(p.b_c + ch);
    const int cb = part_start(part, tt, s), ce = part_start(part + 1, tt, s);
    const uint32_t sB = smem_u32(sm + OFF_B);
    // this channel's byte inside a swizzled 128-byte latent row (K block ch / 64)
    const uint32_t c_kb = (uint32_t)(ch >> 6), c_chunk = (uint32_t)((ch & 63) >> 3), c_in = (uint32_t)(ch & 7) * 2;
    // byte of this channel's 16-byte piece in a latent row r of an 8-row
    // swizzle atom: (c_chunk ^ r) * 16, for r = 0..7
    uint32_t xo[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) xo[r] = (c_chunk ^ (uint32_t)r) << 4;
    const uint32_t p_addr = smem_u32(sm + OFF_X) + (uint32_t)chl * 4;
    const uint32_t o_base = smem_u32(sm + OFF_OUT), g_base = smem_u32(sm + OFF_X + P_BYTES_S2);
    const int ptid = q * 32 + lane;                  // thread of this quarter of the tokens (0..95)
    // With a stride that divides 16 every quarter of a tile is 32 rows, and
    // each warp stages its own 32 channels of them ([32 rows][32 channels],
    // 2 KB; the closing rows likewise) and sends them with its own TMA
    // stores: no warp waits for another.  Otherwise the quarter's three warps
    // stage [rows][96 channels] together and store the rows with 16-byte
    // stores after a barrier.
    constexpr bool kTmaRows = S > 0 && 16 % S == 0;
    constexpr uint32_t o_pitch = kTmaRows ? 64u : (uint32_t)OROW;  // bytes per staged row
    const int ew = part * 3 + q;                     // epilogue warp index, 0..11
    const int cb0 = part_start(part, tt, s);         // the quarter's first column
    const uint32_t o_w = o_base + (uint32_t)ew * 2048u;
    const uint32_t g_w = g_base + (uint32_t)ew * (uint32_t)((32 / s) * 64);
    // staged element of column col (group gl) for this thread's channel
    const uint32_t o_row0 = kTmaRows ? o_w - (uint32_t)cb0 * 64u + (uint32_t)lane * 2u : o_base + (uint32_t)chl * 2u;
    const uint32_t g_row0 =
        kTmaRows ? g_w - (uint32_t)(cb0 / s) * 64u + (uint32_t)lane * 2u : g_base + (uint32_t)chl * 2u;
    uint32_t tc = 0, np = 0;
    int prev_tb = -1;
    for (int u = u_beg; u < u_end && ok; ++u, ++tc) {
      const int ab = tc & 1, sb = (tc & 1) * KB;      // accumulator; the tile's first stage
      int b, tb;
      tile_of(u, p.B, b, tb);
      int nb, ntb = -1;                               // the next tile's position (P still needed?)
      if (u + 1 < u_end) tile_of(u + 1, p.B, nb, ntb);
      const int64_t n0 = (int64_t)tb * tt;           // first token of the tile (a group start)
      const int64_t left = p.T - n0;
      const int hi = (int)(left < ce ? left : ce);   // this warp's columns: [cb, hi)
      const uint32_t par = (tc >> 1) & 1;
      if (tb != prev_tb) {
        ++np;
        prev_tb = tb;
      }
      // the accumulator; the P rows; the stage holding this channel's K
      // block (latent channels) or the tile's RoPE keys
      ok = warp_wait(&acc_full[ab], par) && warp_wait(p_full, (np - 1) & 1) &&
           (rope ? warp_wait(&kr_full[tc & 1], par) : warp_wait(&k_full[sb + c_kb], par));
      tc_fence_after();
      const uint32_t crow = rope ? smem_u32(sm + OFF_KR + (tc & 1) * KRBLK) + (uint32_t)(ch - R) * 2
                                 : sB + (sb + c_kb) * BBLK + c_in;
      float run = 0.f, pe = 0.f;
      // (TMA rows) the staged rows of this quarter are written again only
      // after the stores issued at the previous tile have read them: waited
      // for just before the first staged write, after that chunk's loads
      // and gate math
      bool need_free = kTmaRows && tc > 0;
      for (int cc = (cb / 16) * 16; cc < hi && ok; cc += 16) {
        // pass 1: the chunk's accumulators, entries and P values (loads only)
        uint32_t g[16];
        tmem_ld16(lane_base + ab * ACC_STRIDE + cc, g);
        float v[16], pc[16];
        const int pos0 = (S > 0 && 16 % S == 0) ? 0 : cc % s, gl0 = cc / s;
        // chunks start at multiples of 16 columns, so column cc + k sits in
        // row k & 7 of swizzle atom cc / 8 + k / 8
        const uint32_t cbase = rope ? crow + (uint32_t)cc * (DR * 2) : crow + (uint32_t)(cc >> 3) * 1024;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          uint16_t raw;
          const uint32_t a = rope ? cbase + (uint32_t)k * (DR * 2)
                                  : cbase + (uint32_t)(k >> 3) * 1024 + (uint32_t)(k & 7) * 128 + xo[k & 7];
          asm volatile("ld.shared.u16 %0, [%1];" : "=h"(raw) : "r"(a));
          v[k] = __bfloat162float(__ushort_as_bfloat16(raw));
        }
        {
          // the P entry of each column's group (rows past the tile's groups
          // hold the TMA's zero fill or an earlier tile's rows: unused)
          int pos = pos0, gl = gl0;
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            if (pos == 0) asm volatile("ld.shared.f32 %0, [%1];" : "=f"(pe) : "r"(p_addr + (uint32_t)(gl < gpt ? gl : 0) * PROW));
            pc[k] = pe;
            if (++pos == s) {
              pos = 0;
              ++gl;
            }
          }
        }
        tmem_wait_ld();
        // pass 2: the gate and the gated entry, independent across columns
        // (the group's two factors are formed at its first column)
        {
          int pos = pos0;
          float pa = 0.f, pb = 0.f;
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            if (k == 0 || pos == 0) {
              pa = pc[k] * kNegLog2e;
              pb = bc * pa;
            }
            v[k] = gated(v[k], fmaf(__uint_as_float(g[k]), pa, pb));
            if (++pos == s) pos = 0;
          }
        }
        if (need_free) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          need_free = false;
        }
        // pass 3: the running sums inside groups and the staged stores; a
        // chunk inside this warp's columns that does not hold the prompt's
        // last token needs no per-column checks
        int pos = pos0, gl = gl0;
        if (cc >= cb && cc + 16 <= hi && cc + 16 < left) {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            run = pos == 0 ? v[k] : __fadd_rn(run, v[k]);
            const unsigned short o = __bfloat16_as_ushort(__float2bfloat16_rn(run));
            asm volatile("st.shared.u16 [%0], %1;" ::"r"(o_row0 + (uint32_t)(cc + k) * o_pitch), "h"(o));
            if (s > 1 && pos == s - 1)
              asm volatile("st.shared.u16 [%0], %1;" ::"r"(g_row0 + (uint32_t)gl * o_pitch), "h"(o));
            if (++pos == s) {
              pos = 0;
              ++gl;
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int col = cc + k;
            run = pos == 0 ? v[k] : __fadd_rn(run, v[k]);
            if (col >= cb && col < hi) {
              const unsigned short o = __bfloat16_as_ushort(__float2bfloat16_rn(run));
              asm volatile("st.shared.u16 [%0], %1;" ::"r"(o_row0 + (uint32_t)col * o_pitch), "h"(o));
              if (s > 1 && (pos == s - 1 || col == left - 1))
                asm volatile("st.shared.u16 [%0], %1;" ::"r"(g_row0 + (uint32_t)gl * o_pitch), "h"(o));
            }
            if (++pos == s) {
              pos = 0;
              ++gl;
            }
          }
        }
      }
      // the accumulator and this tile's stages have been read; the P rows
      // too when the next tile needs others
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&acc_empty[ab]);
        for (int kb = 0; kb < KB; ++kb) mbar_arrive(&k_empty[sb + kb]);
        if (rope) mbar_arrive(&kr_empty[tc & 1]);
        if (ntb >= 0 && ntb != tb) mbar_arrive(p_empty);
      }
      if (need_free) {  // a warp without columns in this tile
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
      }
      if constexpr (kTmaRows) {
        // this warp's staged rows are complete: its first lane sends them
        // (the maps clip rows past the prompt's end); a failed wait ends
        // only this warp's loop (the others' waits are bounded)
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && ok && hi > cb) {
          tma_store_3d(&mp.out, sm + OFF_OUT + ew * 2048, ct * NCT + q * 32, (int32_t)(n0 + cb), b);
          if (p.cache)
            tma_store_3d(&mp.cache, s == 1 ? sm + OFF_OUT + ew * 2048 : sm + OFF_X + P_BYTES_S2 + ew * ((32 / s) * 64),
                         ct * NCT + q * 32, (int32_t)((n0 + cb) / s), b);
          bulk_commit();
        }
        if (!ok) break;
      } else {
        // the three warps of this quarter of the tokens write its staged rows
        // [cb, hi) (and their closing rows) with 16-byte stores: 12 per row
        named_bar(4 + part, 96);
        const int64_t row0 = (int64_t)b * p.T + n0;
        const int nrow = hi > cb ? hi - cb : 0;
        // thread ptid takes the 16-byte piece ptid % 12 of every eighth row
        const int c16 = ptid % 12, r_first = ptid / 12;
        for (int r = cb + r_first; r < hi; r += 8) {
          uint4 w;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                       : "r"(o_base + (uint32_t)r * OROW + c16 * 16));
          *reinterpret_cast<uint4*>(p.cp + (row0 + r) * D + ct * NCT + c16 * 8) = w;
        }
        if (p.cache && nrow > 0) {
          // closing rows: the groups of columns cb .. hi-1 (a partial last
          // group closes at the prompt's last token)
          const int gb = cb / s, ge = (hi - 1) / s + 1;
          const uint32_t src = s == 1 ? o_base : g_base;
          const int64_t grow0 = (int64_t)b * p.n_groups + n0 / s;
          for (int r = gb + r_first; r < ge; r += 8) {
            uint4 w;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                         : "r"(src + (uint32_t)r * OROW + c16 * 16));
            *reinterpret_cast<uint4*>(p.cache + (grow0 + r) * D + ct * NCT + c16 * 8) = w;
          }
        }
        // the next tile writes the staged rows again only after this
        // barrier; it also ORs the three warps' failed waits, so they leave
        // the loop at the same tile
        uint32_t failed;
        asm volatile(
            "{\n .reg .pred f;\n setp.eq.u32 f, %1, 0;\n bar.red.or.pred f, %2, 96, f;\n selp.u32 %0, 1, 0, f;\n}"
            : "=r"(failed) : "r"(ok ? 1u : 0u), "r"(4 + part) : "memory");
        if (failed) {
          ok = false;
          break;
        }
      }
    }
    if (kTmaRows && lane == 0) bulk_wait_all();  // no store may still read shared memory at exit
    if (!ok && lane == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace mtc

cudaError_t launch_merge_tc(const PrefillArgs& a, int B, const MergeMaps& m, int sms, cudaStream_t st) {
  mtc::Params p;
  p.B = B;
  p.T = a.T;
  p.s = a.s;
  p.tt = (mtc::NTOK / a.s) * a.s;
  p.tiles_per_seq = (int)cdiv(a.T, p.tt);
  p.n_tiles = B * p.tiles_per_seq;
  p.n_groups = cdiv(a.T, a.s);
  p.W_c = a.W_c;
  p.b_c = a.b_c;
  p.cp = static_cast<__nv_bfloat16*>(a.c_partial);
  p.cache = static_cast<__nv_bfloat16*>(a.cache_out);
  p.dev_err = a.dev_err;
  const size_t smem = mtc::smem_bytes();
  int per_tile = sms / mtc::CT > 0 ? sms / mtc::CT : 1;  // CTAs per channel tile
  if (p.n_tiles < per_tile) per_tile = p.n_tiles;
  auto go = [&](auto kernel, int slot) -> cudaError_t {
    // the shared-memory opt-in, once per instance and device
    static uint64_t done_mask[7] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !(done_mask[slot] & (1ull << dev))) {
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      if (dev < 64) done_mask[slot] |= 1ull << dev;
    }
    kernel<<<mtc::CT * per_tile, mtc::NT, smem, st>>>(m, p);
    return cudaGetLastError();
  };
  switch (a.s) {
    case 1: return go(mtc::merge_tc_kernel<1>, 1);
    case 2: return go(mtc::merge_tc_kernel<2>, 2);
    case 4: return go(mtc::merge_tc_kernel<4>, 3);
    case 8: return go(mtc::merge_tc_kernel<8>, 4);
    case 16: return go(mtc::merge_tc_kernel<16>, 5);
    case 3: return go(mtc::merge_tc_kernel<3>, 6);
    default: return go(mtc::merge_tc_kernel<0>, 0);
  }
}

}  // namespace mtla
