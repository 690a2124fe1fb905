// Split-L tensor-core decode step for bf16 caches with H = 8, r = 256, d_R = 32:
// one kernel for the merge of the new tokens and the attention, one for the
// split combine and the lengths.
//
// What it computes (MTLA paper notes, "Key designs: decoupled RoPE with
// temporal compression"; Figure 2(a) of the abstract page): for every
// sequence b and head h, o_h = sum_j softmax_j((q_abs_h . c_hat_j +
// q^R_h . k_hat^R_j) / sqrt(d_h)) c_hat_j over the ceil(t/s) cache rows, the
// partial tail row included; optionally the new token is first merged into
// the tail row ("Key designs: hyper-network temporal merging").
//
// Design (B200):
//  * The H heads share one latent cache, so every cache row (576 B) is read
//    from HBM exactly once for all heads.  The rows of all sequences are cut
//    into equal shares for a persistent grid of two blocks per SM (split-L,
//    balanced to the row; a merged sequence weighs MERGE_COST extra rows).
//    Every block reads all lengths and derives the same partition.
//  * One producer warp streams 64-row tiles HBM -> shared memory with 3-D TMA
//    boxes {32 elements, 64 rows, 9 planes}: the tensor map orders the row's
//    nine 32-element segments as the outer dimension, so a tile lands as nine
//    [64 rows x 64 B] planes with the 64-byte swizzle, whose XOR phase then
//    depends on the row only (every ldmatrix address is a per-lane base plus a
//    constant).  A ragged last tile uses {32, 8, 1} boxes.  NS stages per
//    block, mbarrier completion.
//  * Four consumer warps each own 16 rows of a tile.  Scores S^T = rows . Q^T
//    (M = rows, N = the 8 heads, K = 288) and values O^T += C_hat^T . P^T
//    (M = 256 latent channels, N = 8 heads, K = rows) run on the tensor cores
//    with bf16 operands and fp32 accumulators; the score fragment becomes the
//    value-MMA operand with one in-register 8x8 transpose (movmatrix).  Each
//    warp keeps its own online-softmax state, so no block barrier is needed
//    per tile.
//  * The merge's gate contraction Linear(c_t) (r x D per token) is cut into
//    units of a few tokens x 32 channels that the consumer warps of the
//    blocks run while their first tiles are in flight.  A unit writes its
//    gated entries w * [c_t ; k^R_t] (fp32) to the workspace and counts itself
//    in its tokens' counters.  Every block visits its share's sequences last
//    to first, so a tail row is the last tile of its sequence's segment; the
//    warp holding it waits (bounded) until the nine units of the token are
//    in, patches the appended or updated row into its tile and writes it to
//    the cache.
//  * At the end of each of its sequences a block's four warps combine their
//    online-softmax states through shared memory.  A sequence held by one
//    block is written out; otherwise the block writes one part (max, sum,
//    unnormalised output per head).  A second kernel, launched behind it with
//    programmatic dependent launch (its blocks are resident and waiting
//    before the first ends), combines the parts of every split sequence, one
//    block per (sequence, head), from a per-sequence summary the first kernel
//    writes, advances t_processed / cache_len and resets the gate counters.
#include "kernels.cuh"

namespace mtla {
namespace dtc {

// every region starts on a 128-byte boundary (the queries are read with
// 16-byte vector loads, the mbarriers need 8)
constexpr size_t kAlign = 128;
__host__ __device__ constexpr size_t rup(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
constexpr int kCombHeads = 4;  // heads per pass of the block combine
constexpr int QSTR = D / 2 + 4;  // words per query row in shared memory (148: conflict-free)
constexpr size_t kCombBytes = (size_t)NCW * kCombHeads * OSTR * 4;
static_assert((size_t)H * QSTR * 4 <= kCombBytes, "query buffer must fit the combine buffer");
static_assert((size_t)4 * 8 * 32 * 4 <= kCombBytes, "gate partial sums must fit the combine buffer");
constexpr size_t kOffComb = rup((size_t)NS * STAGE);
constexpr size_t kOffCombMl = kOffComb + rup(kCombBytes);
constexpr size_t kOffPrefix = kOffCombMl + rup((size_t)NCW * H * 2 * 4 + (size_t)(NCW + 2) * H * 4);
constexpr size_t kOffMeta = kOffPrefix + rup((size_t)(MAXB + 1) * 8);
constexpr size_t kOffQx = kOffMeta + rup((size_t)MAXB * 4);
constexpr size_t kOffBar = kOffQx + rup((size_t)H * QSTR * 4);
constexpr size_t kOffFlags = kOffBar + rup(2 * NS * 8);
constexpr size_t kSmemUsed = kOffFlags + rup(16 * 4);
static_assert(kOffQx % 16 == 0 && kOffBar % 8 == 0, "shared-memory regions must stay aligned");
static_assert(128 * 8 <= kCombBytes, "scan scratch must fit the combine buffer");
// two blocks (each with 1 KB of alignment slack and 1 KB the system reserves) fit one SM's 228 KB
static_assert(2 * (kSmemUsed + 1024 + 1024) <= 233472, "shared memory per SM");

size_t smem_bytes() { return kSmemUsed + 1024; }  // + slack to align the base to 1024

WsLayout ws_layout(int B, int grid) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  WsLayout l;
  l.counters = up((size_t)B * 4);                    // gate counters
  l.seq_info = l.counters;                           // [B] partition summary
  l.e = up(l.seq_info + (size_t)B * 16);             // [B][D] fp32 gated entries
  l.ml = up(l.e + (size_t)B * D * 4);                // parts: (max, sum) per head, two slots per block
  l.o = up(l.ml + (size_t)2 * grid * H * 2 * 4);     // parts: unnormalised outputs
  l.total = l.o + (size_t)2 * grid * H * R * 4;
  return l;
}

size_t workspace_bytes(int B, int grid) { return ws_layout(B, grid).total; }

// byte offset, inside a tile, of row `row`, 16-byte chunk `ch` (0..35): plane
// ch / 4 holds the row's 64-byte segment, TMA's 64-byte swizzle XORs chunk
// bits [4:5] with address bits [7:8], i.e. with (row / 2) mod 4
__host__ __device__ __forceinline__ uint32_t swz_off(int row, int ch) {
  return (uint32_t)(ch >> 2) * SEGB + (uint32_t)row * 64u + ((((uint32_t)ch & 3u) ^ (((uint32_t)row >> 1) & 3u)) << 4);
}

// per-sequence summary in shared memory: rows after the call (bits 0..28),
// whether the new token opens its row (bit 29), whether it is merged (bit 30)
constexpr uint32_t kMetaRows = (1u << 29) - 1;
constexpr uint32_t kMetaOpens = 1u << 29;
constexpr uint32_t kMetaMergeOk = 1u << 30;

struct Smem {
  uint8_t* stages;
  float* comb_o;
  float* comb_ml;
  int64_t* prefix;
  uint32_t* meta;
  int64_t* scan;
  uint32_t* qx;       // [H][QSTR] queries of the share's second sequence (prefetched)
  uint64_t* full_bar;
  uint64_t* empty_bar;
  int32_t* flags;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* p = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.stages = p;
  s.comb_o = reinterpret_cast<float*>(p + kOffComb);
  s.comb_ml = reinterpret_cast<float*>(p + kOffCombMl);
  s.prefix = reinterpret_cast<int64_t*>(p + kOffPrefix);
  s.meta = reinterpret_cast<uint32_t*>(p + kOffMeta);
  // the prologue's scan scratch shares the combine buffer, first used after it
  s.scan = reinterpret_cast<int64_t*>(p + kOffComb);
  s.qx = reinterpret_cast<uint32_t*>(p + kOffQx);
  s.full_bar = reinterpret_cast<uint64_t*>(p + kOffBar);
  s.empty_bar = s.full_bar + NS;
  s.flags = reinterpret_cast<int32_t*>(p + kOffFlags);
  return s;
}

// first index i in [0, n) with a[i] > x (n if none)
__device__ __forceinline__ int upper_bound_i64(const int64_t* a, int n, int64_t x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] > x) hi = mid; else lo = mid + 1;
  }
  return lo;
}

constexpr int PRO_T = NT;               // every warp takes part in the prologue
constexpr int CON_T = 32 * NCW;        // threads of the consumer warps

// 16-byte asynchronous global -> shared copies (completion per thread)
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ int64_t rows_of(const uint32_t* meta, int b) { return (int64_t)(meta[b] & kMetaRows); }

// Block c of the G_eff blocks that share C cost positions starts at floor(c C / G_eff).
// floor(c C / G) in double precision: c C < 2^53 is exact, and a quotient
// that is not an integer lies at least 1/G from one, far beyond the rounding
// error (below 2^-3 ulp of 2^40), so truncation gives the integer quotient
// without a 64-bit integer division
__device__ __forceinline__ int64_t share_start(int c, int64_t C, int G) {
  return C > 0 ? (int64_t)(((double)c * (double)C) / (double)G) : 0;
}
// The block whose share holds cost position x (0 <= x < C): shares are not
// empty because G_eff <= C.
__device__ __forceinline__ int block_of(int64_t x, int64_t C, int G) {
  int c = (int)(((double)x * (double)G) / (double)C);
  if (c > G - 1) c = G - 1;
  if (c < 0) c = 0;
  while (c > 0 && share_start(c, C, G) > x) --c;
  while (c + 1 < G && share_start(c + 1, C, G) <= x) ++c;
  return c;
}
// The first sequence with rows in the share [lo, hi), B if the share is empty.
__device__ __forceinline__ int first_seq(const int64_t* prefix, const uint32_t* meta, int B, int64_t lo, int64_t hi) {
  if (lo >= hi) return B;
  int b = upper_bound_i64(prefix, B + 1, lo) - 1;
  if (b < 0) b = 0;
  if (b < B && lo - prefix[b] >= rows_of(meta, b)) ++b;
  return b;
}

// Sequence b after this call: its rows, whether its new token is merged and
// opens a row, and the device-error bits the checks raise.
struct SeqState {
  int64_t t;        // processed tokens after the call
  int64_t L;        // cache rows after the call
  bool merge_ok;
  bool opens;
  int err;
};
__device__ __forceinline__ SeqState seq_state(const Params& p, int b, bool with_merge) {
  const int s = p.a.s;
  const int64_t t0 = p.a.t_processed[b];
  const int64_t off = p.a.seq_offset[b], cap = p.a.seq_capacity[b];
  SeqState st;
  st.t = t0 + (with_merge ? 1 : 0);
  st.L = st.t > 0 ? group_of(st.t, s) : 0;
  st.merge_ok = with_merge;
  st.opens = st.t > 0 && opens_row(st.t, s);
  st.err = 0;
  if (t0 < 0 || off < 0 || cap < 0 || off > p.a.cache_rows || cap > p.a.cache_rows - off) {
    st.err |= MTLA_DEVERR_CAPACITY;
    st.L = 0;
    st.merge_ok = false;
  } else if (st.L > cap) {
    st.err |= MTLA_DEVERR_CAPACITY;
    st.L = cap;
    st.merge_ok = false;
  }
  if (st.L > (int64_t)kMetaRows) {  // beyond what one call can address
    st.err |= MTLA_DEVERR_CAPACITY;
    st.L = 0;
    st.merge_ok = false;
  }
  if (st.merge_ok && group_of(st.t, s) > p.m.J_max) {
    st.err |= MTLA_DEVERR_PE_RANGE;
    st.merge_ok = false;
  }
  return st;
}

// Bounded wait (about one second) until *cnt reaches `target`; acquire order
// for the reads that follow.  False on timeout.
__device__ __forceinline__ bool wait_count(const uint32_t* cnt, uint32_t target) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
  if (v >= target) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    for (int i = 0; i < 64; ++i) {
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
      if (v >= target) return true;
    }
    if (global_ns() - t0 > kWaitNs) return false;
    __nanosleep(64);
  }
}

// Release form of the counters' atomic (no full fence needed).
__device__ __forceinline__ void red_add_release(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// One gate unit: tokens b0 .. b0 + TPU - 1, channels k0 .. k0 + 31 of the
// merge gate (MTLA paper notes, "Key designs: hyper-network temporal
// merging"): w = sigmoid((c_t W_c + b_c) * P[j - 1]) and the gated entry
// w * [c_t ; k^R_t], written to ws_e.  The four consumer warps run it: warp w
// takes input rows 64 w .. 64 w + 63 of the contraction, lanes are channels,
// and every load of the unit is issued at once (gate_issue, then the P row
// once t_processed has arrived); a block's first unit is issued right after
// the kernel starts, beside the length loads and before the tile stream
// floods the memory system.  The warps' partial sums meet in shared memory
// and are added in a fixed order (deterministic).  The unit then counts
// itself in each of its tokens' gate counters (release: the entries are
// visible to the reader that sees the count).
template <int TPU>
struct GateIn {
  static constexpr int NF = (TPU + NCW - 1) / NCW;  // tokens warp w finishes: w, w + 4
  float wv[64];           // W_c rows 64 w .. 64 w + 63, channel k
  float cv[2][TPU];       // the tokens' latents of rows 64 w + lane and 64 w + 32 + lane
  float fb[NF], fp[NF], fx[NF];  // b_c[k], P[j - 1][k] and the entry [c_t ; k^R_t][k] of a finished token
  int32_t t0[NF];         // its t_processed before the call
};

template <int TPU>
__device__ __forceinline__ void gate_issue(const Params& p, int k0, int b0, GateIn<TPU>& g) {
  const int ctid = threadIdx.x, w = ctid >> 5, lane = ctid & 31;
  const int k = k0 + lane, i0 = w * 64;
  const __nv_bfloat16* cn = reinterpret_cast<const __nv_bfloat16*>(p.m.c_new);
#pragma unroll
  for (int i = 0; i < 64; ++i) g.wv[i] = __ldg(p.m.W_c + (size_t)(i0 + i) * D + k);
#pragma unroll
  for (int half = 0; half < 2; ++half)
#pragma unroll
    for (int u = 0; u < TPU; ++u)
      g.cv[half][u] = b0 + u < p.B ? __bfloat162float(cn[(size_t)(b0 + u) * R + i0 + 32 * half + lane]) : 0.f;
#pragma unroll
  for (int f = 0; f < GateIn<TPU>::NF; ++f) {
    const int b = b0 + w + NCW * f;
    g.fb[f] = g.fp[f] = g.fx[f] = 0.f;
    g.t0[f] = -1;
    if (w + NCW * f < TPU && b < p.B) {
      g.fb[f] = __ldg(p.m.b_c + k);
      g.fx[f] = __bfloat162float(k < R ? cn[(size_t)b * R + k]
                                       : reinterpret_cast<const __nv_bfloat16*>(p.m.kR_new)[(size_t)b * DR + (k - R)]);
      g.t0[f] = p.a.t_processed[b];
    }
  }
}

// The P row of each finished token's group j = ceil((t0 + 1) / s); a group
// outside the table is not loaded (that token is not merged: PE_RANGE).
template <int TPU>
__device__ __forceinline__ void gate_issue_p(const Params& p, int k0, GateIn<TPU>& g) {
  const int k = k0 + (threadIdx.x & 31);
#pragma unroll
  for (int f = 0; f < GateIn<TPU>::NF; ++f) {
    if (g.t0[f] < 0) continue;
    const int64_t j = group_of((int64_t)g.t0[f] + 1, p.a.s);
    if (j <= p.m.J_max) g.fp[f] = __ldg(p.m.P + (j - 1) * D + k);
  }
}

template <int TPU>
__device__ __forceinline__ void gate_finish(const Params& p, const Smem& sm, int k0, int b0, const GateIn<TPU>& g) {
  const int ctid = threadIdx.x, w = ctid >> 5, lane = ctid & 31;
  float* part = sm.comb_o;  // [4 warps][TPU][32]
  const int k = k0 + lane;
  float acc[TPU];
#pragma unroll
  for (int u = 0; u < TPU; ++u) acc[u] = 0.f;
#pragma unroll
  for (int i = 0; i < 64; ++i)
#pragma unroll
    for (int u = 0; u < TPU; ++u) acc[u] = fmaf(__shfl_sync(0xffffffffu, g.cv[i >> 5][u], i & 31), g.wv[i], acc[u]);
#pragma unroll
  for (int u = 0; u < TPU; ++u) part[(w * TPU + u) * 32 + lane] = acc[u];
  named_bar(1, CON_T);
#pragma unroll
  for (int f = 0; f < GateIn<TPU>::NF; ++f) {
    const int u = w + NCW * f;
    const int b = b0 + u;
    if (u >= TPU || b >= p.B || !(sm.meta[b] & kMetaMergeOk)) continue;
    float gs = 0.f;
#pragma unroll
    for (int ww = 0; ww < NCW; ++ww) gs += part[(ww * TPU + u) * 32 + lane];
    const float gv = gs + g.fb[f];
    const float wt = sigmoidf_(__fmul_rn(gv, g.fp[f]));
    p.ws_e[(size_t)b * D + k] = __fmul_rn(wt, g.fx[f]);
  }
  named_bar(1, CON_T);  // every entry of the unit is written (and `part` may be reused)
  if (ctid < TPU) {
    const int b = b0 + ctid;
    if (b < p.B && (sm.meta[b] & kMetaMergeOk)) red_add_release(p.gate_cnt + b, 1u);
  }
}

template <int TPU>
__device__ __forceinline__ int gate_unit_count(int B) { return ((B + TPU - 1) / TPU) * GATE_CHUNKS; }

template <int TPU>
__global__ void __launch_bounds__(NT, 2)
decode_tc_kernel(const __grid_constant__ CUtensorMap map64, const __grid_constant__ CUtensorMap map8,
                 const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const Smem sm = carve(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = p.B, G = gridDim.x, cta = blockIdx.x;
  const bool with_merge = p.with_merge != 0;
  const int64_t mcost = with_merge ? p.merge_cost : 0;

  // the next launch on the stream may be scheduled as soon as blocks retire;
  // it waits for this grid before reading anything (griddepcontrol.wait)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sm.full_bar[i], 1);
      mbar_init(&sm.empty_bar[i], NCW);
    }
    fence_mbar_init();
  }
  if (warp == PRODUCER_WARP && lane == 0) {
    prefetch_tmap(&map64);
    prefetch_tmap(&map8);
  }
  // the previous launch may write everything read below: lengths, the cache,
  // the workspace's counters, this step's inputs
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // this block's first gate unit: its loads go out now, beside the lengths
  const int n_units = with_merge ? gate_unit_count<TPU>(B) : 0;
  const bool first_unit = tid < CON_T && cta < n_units;
  const int gk0 = (cta % GATE_CHUNKS) * GATE_CH, gb0 = (cta / GATE_CHUNKS) * TPU;
  GateIn<TPU> gi;
  if (first_unit) gate_issue<TPU>(p, gk0, gb0, gi);

  // ---- 1. rows per sequence and the cost prefix (identical in every block)
  const int per = (B + 127) / 128;
  if (tid < 128) {
    int64_t sum = 0;
    for (int b = tid * per; b < B && b < (tid + 1) * per; ++b) {
      const SeqState st = seq_state(p, b, with_merge);
      if (st.err && cta == 0) set_err(p.a.dev_err, st.err);
      sm.meta[b] = (uint32_t)st.L | (st.merge_ok ? kMetaMergeOk : 0u) | (st.opens ? kMetaOpens : 0u);
      sum += st.L + mcost;
    }
    sm.scan[tid] = sum;
  }
  if (first_unit) gate_issue_p<TPU>(p, gk0, gi);
  named_bar(2, PRO_T);
  if (warp == 0) {
    // exclusive scan of the 128 partial sums (4 per lane)
    int64_t v[4], run = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) { v[i] = sm.scan[lane * 4 + i]; run += v[i]; }
    int64_t incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    int64_t ex = incl - run;
#pragma unroll
    for (int i = 0; i < 4; ++i) { const int64_t t = v[i]; sm.scan[lane * 4 + i] = ex; ex += t; }
    if (lane == 31) sm.prefix[B] = ex;  // total cost
  }
  named_bar(2, PRO_T);
  const int64_t C = sm.prefix[B];
  // shares of the first G_eff blocks (no share is empty); the rest hold none
  const int Ge = C < (int64_t)G ? (int)C : G;
  // this block's share: cost positions [my_lo, my_hi).  While the prefix is
  // written, the threads that own the sequences holding its first and last
  // positions record them: its first sequence with rows (B if none) and the
  // sequence of its last position
  const int64_t my_lo = cta < Ge ? share_start(cta, C, Ge) : 0;
  const int64_t my_hi = cta < Ge ? share_start(cta + 1, C, Ge) : 0;
  if (tid < 128) {
    int64_t run = sm.scan[tid];
    for (int b = tid * per; b < B && b < (tid + 1) * per; ++b) {
      sm.prefix[b] = run;
      const int64_t next = run + rows_of(sm.meta, b) + mcost;
      if (my_lo < my_hi) {
        if (run <= my_lo && my_lo < next) sm.flags[0] = my_lo - run >= rows_of(sm.meta, b) ? b + 1 : b;
        if (run <= my_hi - 1 && my_hi - 1 < next) sm.flags[1] = b;
      }
      run = next;
    }
  }
  named_bar(2, PRO_T);
  // the share's sequences are visited last to first so that a sequence's tail
  // row (whose gated entry other blocks compute meanwhile) is the last tile
  // of its segment
  const int b_first = my_lo < my_hi ? sm.flags[0] : B;
  const int b_last = my_lo < my_hi ? sm.flags[1] : -1;

  // ======================= producer warp =======================
  if (warp == PRODUCER_WARP) {
    if (lane == 0 && my_lo < my_hi) {
      uint32_t job = 0;
      bool ok = true;
      for (int b = b_last; b >= b_first && ok; --b) {
        const int64_t Lb = rows_of(sm.meta, b);
        const int64_t r_lo = (my_lo > sm.prefix[b] ? my_lo : sm.prefix[b]) - sm.prefix[b];
        const int64_t r_end = sm.prefix[b] + Lb < my_hi ? sm.prefix[b] + Lb : my_hi;
        const int64_t r_hi = r_end - sm.prefix[b];
        if (r_lo >= r_hi) continue;
        const int64_t row0 = p.a.seq_offset[b];
        for (int64_t u = r_lo; u < r_hi && ok; u += UNIT) {
          const int st = job % NS;
          if (job >= NS && !mbar_wait(&sm.empty_bar[st], ((job / NS) & 1) ^ 1)) { ok = false; break; }
          const int64_t nrows = r_hi - u < UNIT ? r_hi - u : UNIT;
          uint8_t* dst = sm.stages + st * STAGE;
          if (nrows == UNIT) {
            mbar_arrive_expect_tx(&sm.full_bar[st], STAGE);
            tma_load_3d(dst, &map64, 0, (int32_t)(row0 + u), 0, &sm.full_bar[st]);
          } else {
            // 8-row boxes of one plane each, into the same plane layout
            const int nsub = (int)((nrows + SUB - 1) / SUB);
            mbar_arrive_expect_tx(&sm.full_bar[st], (uint32_t)(nsub * SUB * ROWB));
            for (int i = 0; i < nsub; ++i)
              for (int c = 0; c < D / 32; ++c)
                tma_load_3d(dst + c * SEGB + i * SUB * 64, &map8, 0, (int32_t)(row0 + u + i * SUB), c,
                            &sm.full_bar[st]);
          }
          ++job;
        }
      }
      if (!ok) set_err(p.a.dev_err, MTLA_DEVERR_TIMEOUT);
      // drain: no copy may still be writing this block's shared memory at exit
      const uint32_t first = job > (uint32_t)NS ? job - NS : 0;
      for (uint32_t j = first; j < job; ++j) mbar_wait(&sm.full_bar[j % NS], (j / NS) & 1);
    }
    return;
  }

  // ======================= consumer warps =======================
  const int cw = warp, ctid = tid;  // 0..127
  const int g = lane >> 2, q = lane & 3;
  const float sl2 = p.scale_log2;

  // the share's second sequence (in visiting order): its queries are fetched
  // now, so that they do not queue behind the tile stream later
  int b_second = -1;
  {
    int found = 0;
    for (int b = b_last; b >= b_first && found < 2; --b) {
      const int64_t lo_b = my_lo > sm.prefix[b] ? my_lo : sm.prefix[b];
      const int64_t hi_b = sm.prefix[b] + rows_of(sm.meta, b) < my_hi ? sm.prefix[b] + rows_of(sm.meta, b) : my_hi;
      if (lo_b >= hi_b) continue;
      if (++found == 2) b_second = b;
    }
  }
  if (b_second >= 0) {
    const __nv_bfloat16* qa = reinterpret_cast<const __nv_bfloat16*>(p.o.q_abs) + (size_t)b_second * H * R;
    const __nv_bfloat16* qr = reinterpret_cast<const __nv_bfloat16*>(p.o.q_rope) + (size_t)b_second * H * DR;
    for (int i = ctid; i < H * (D / 8); i += 128) {
      const int h = i / (D / 8), c = i % (D / 8);  // 16-byte chunk c of head h's row
      const __nv_bfloat16* src = c < R / 8 ? qa + h * R + c * 8 : qr + h * DR + (c - R / 8) * 8;
      cp_async16(smem_u32(sm.qx) + (uint32_t)(h * QSTR + c * 4) * 4u, src);
    }
    cp_async_commit();
  }


  // the partition as the combine kernel needs it (block c takes sequences
  // c, c + G, ...): rows, merged, the first part's slot and the number of
  // parts (blocks cf .. cl hold its rows; block cf's part is in slot 2 cf or
  // 2 cf + 1, block c > cf's in slot 2 c)
  for (int b = cta + G * ctid; b < B; b += G * CON_T) {
    const uint32_t mt = sm.meta[b];
    const int64_t Lb = (int64_t)(mt & kMetaRows);
    int first = 0, n = 0;
    if (Lb > 0) {
      const int cf = block_of(sm.prefix[b], C, Ge), cl = block_of(sm.prefix[b] + Lb - 1, C, Ge);
      const int fs = first_seq(sm.prefix, sm.meta, B, share_start(cf, C, Ge), share_start(cf + 1, C, Ge));
      first = 2 * cf + (fs == b ? 0 : 1);
      n = cl - cf + 1;
    }
    p.seq_info[b] = make_int4((int)Lb, (mt & kMetaMergeOk) ? 1 : 0, first, n);
  }

  // this block's gate units (the first one's inputs have arrived meanwhile)
  if (first_unit) gate_finish<TPU>(p, sm, gk0, gb0, gi);
  for (int u = cta + G; u < n_units; u += G) {
    const int k0 = (u % GATE_CHUNKS) * GATE_CH, b0 = (u / GATE_CHUNKS) * TPU;
    gate_issue<TPU>(p, k0, b0, gi);
    gate_issue_p<TPU>(p, k0, gi);
    gate_finish<TPU>(p, sm, k0, b0, gi);
  }

  // per-lane ldmatrix rows: scores (A = rows, K-major) and values (A = C_hat^T, trans)
  const int w_lo = 16 * cw;
  const int arow = w_lo + (lane & 7) + ((lane >> 3) & 1) * 8;
  const int ach = lane >> 4;
  const int vrow = w_lo + (lane & 7) + (lane >> 4) * 8;
  const int vch = (lane >> 3) & 1;
  // ldmatrix offsets inside a tile: chunk 2 kk + ach of row arow sits in plane
  // kk / 2 at swz_off(arow, ach) (kk even) or swz_off(arow, 2 + ach) (kk odd)
  const uint32_t offA0 = swz_off(arow, ach), offA1 = swz_off(arow, 2 + ach);
  const uint32_t offV0 = swz_off(vrow, vch), offV1 = swz_off(vrow, 2 + vch);
  uint32_t job = 0;
  bool ok = true;
  int seg = 0;

  for (int b = b_last; b >= b_first; --b) {
    const int64_t Lb = rows_of(sm.meta, b);
    const int64_t r_lo = (my_lo > sm.prefix[b] ? my_lo : sm.prefix[b]) - sm.prefix[b];
    const int64_t r_end = sm.prefix[b] + Lb < my_hi ? sm.prefix[b] + Lb : my_hi;
    const int64_t r_hi = r_end - sm.prefix[b];
    if (r_lo >= r_hi) continue;
    const uint32_t mt = sm.meta[b];
    const bool merge_here = (mt & kMetaMergeOk) && r_hi == Lb;

    // [q_abs ; q_rope] of the 8 heads into shared memory (rows padded to
    // QSTR words so the B-fragment loads below are free of bank conflicts):
    // the prefetched buffer for the second sequence, else loaded now into the
    // combine buffer, which is only used after the segment's last tile
    const bool pre = (seg == 1 && b == b_second);
    if (pre) {
      cp_async_wait_all();
      named_bar(1, CON_T);
    } else {
      named_bar(1, CON_T);  // every warp is done with the buffer (previous queries, gate sums)
      const uint32_t* qa = reinterpret_cast<const uint32_t*>(
          reinterpret_cast<const __nv_bfloat16*>(p.o.q_abs) + (size_t)b * H * R);
      const uint32_t* qr = reinterpret_cast<const uint32_t*>(
          reinterpret_cast<const __nv_bfloat16*>(p.o.q_rope) + (size_t)b * H * DR);
      uint32_t* qs = reinterpret_cast<uint32_t*>(sm.comb_o);
      for (int i = ctid; i < H * (D / 2); i += 128) {
        const int h = i / (D / 2), w = i % (D / 2);
        qs[h * QSTR + w] = w < R / 2 ? __ldg(qa + h * (R / 2) + w) : __ldg(qr + h * (DR / 2) + (w - R / 2));
      }
      named_bar(1, CON_T);
    }
    // B operand of the score MMA for head g: words 8kk + q and 8kk + q + 4 of its row
    const uint32_t qrow = smem_u32(pre ? reinterpret_cast<float*>(sm.qx) : sm.comb_o) + (uint32_t)(g * QSTR + q) * 4u;
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    float O[16][4];
#pragma unroll
    for (int mb = 0; mb < 16; ++mb) O[mb][0] = O[mb][1] = O[mb][2] = O[mb][3] = 0.f;

    for (int64_t u = r_lo; u < r_hi; u += UNIT) {
      const bool is_tail = merge_here && u + UNIT >= r_hi;

      const int st = job % NS;
      if (ok && !mbar_wait(&sm.full_bar[st], (job / NS) & 1)) ok = false;
      uint8_t* tile_ptr = sm.stages + st * STAGE;
      const uint32_t tile = smem_u32(tile_ptr);
      const int rows = (int)(r_hi - u < UNIT ? r_hi - u : UNIT);
      if (w_lo < rows) {
        bool wrote = false;
        if (w_lo + 16 > rows) {
          // rows past the segment's end: zero them (they may hold anything)
          for (int i = lane; i < (w_lo + 16 - rows) * 36; i += 32) {
            const int rr = rows + i / 36, ch = i % 36;
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(tile + swz_off(rr, ch)), "r"(0u)
                         : "memory");
          }
          wrote = true;
        }
        if (is_tail) {
          const int lr = (int)(Lb - 1 - u);
          if (lr >= w_lo && lr < w_lo + 16) {
            // the nine gate units of b's new token are in (bounded wait; they
            // ran first thing in their blocks), then the appended or updated
            // row: in the tile for the attention and in the cache
            bool ready = true;
            if (lane == 0) ready = wait_count(p.gate_cnt + b, GATE_CHUNKS);
            ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
            __syncwarp();
            if (!ready) {
              ok = false;
            } else {
              const bool opens = (mt & kMetaOpens) != 0;
              const float4* e4 = reinterpret_cast<const float4*>(p.ws_e + (size_t)b * D);
              uint4* crow = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.a.cache) +
                                                     (p.a.seq_offset[b] + Lb - 1) * p.a.row_stride);
              for (int ch = lane; ch < 36; ch += 32) {
                const float4 ea = __ldcg(e4 + 2 * ch), eb = __ldcg(e4 + 2 * ch + 1);
                const float e[8] = {ea.x, ea.y, ea.z, ea.w, eb.x, eb.y, eb.z, eb.w};
                uint32_t old[4];
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(old[0]), "=r"(old[1]), "=r"(old[2]),
                             "=r"(old[3]) : "r"(tile + swz_off(lr, ch)));
                uint32_t nv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const float2 o2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&old[i]));
                  const float v0 = opens ? e[2 * i] : __fadd_rn(o2.x, e[2 * i]);
                  const float v1 = opens ? e[2 * i + 1] : __fadd_rn(o2.y, e[2 * i + 1]);
                  nv[i] = pack_bf16x2(v0, v1);
                }
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(tile + swz_off(lr, ch)), "r"(nv[0]),
                             "r"(nv[1]), "r"(nv[2]), "r"(nv[3]) : "memory");
                crow[ch] = make_uint4(nv[0], nv[1], nv[2], nv[3]);
              }
            }
            wrote = true;
          }
        }
        if (wrote) fence_proxy_async_smem();
        __syncwarp();

        // scores S^T (16 rows x 8 heads) = rows . [q_abs ; q_rope]^T, two
        // independent accumulator chains
        float sacc[2][4];
#pragma unroll
        for (int i = 0; i < 2; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 18; ++kk) {
          uint32_t a0, a1, a2, a3, b0, b1;
          ldsm_x4(tile + (kk >> 1) * SEGB + ((kk & 1) ? offA1 : offA0), a0, a1, a2, a3);
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(b0) : "r"(qrow + kk * 32u));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(b1) : "r"(qrow + kk * 32u + 16u));
          mma_bf16(sacc[kk & 1], a0, a1, a2, a3, b0, b1);
        }
        const bool v0 = (w_lo + g) < rows, v1 = (w_lo + g + 8) < rows;
        const float xA0 = v0 ? (sacc[0][0] + sacc[1][0]) * sl2 : -INFINITY;
        const float xB0 = v0 ? (sacc[0][1] + sacc[1][1]) * sl2 : -INFINITY;
        const float xA1 = v1 ? (sacc[0][2] + sacc[1][2]) * sl2 : -INFINITY;
        const float xB1 = v1 ? (sacc[0][3] + sacc[1][3]) * sl2 : -INFINITY;
        float mxA = fmaxf(xA0, xA1), mxB = fmaxf(xB0, xB1);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, o));
          mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, o));
        }
        const float nA = fmaxf(mA, mxA), nB = fmaxf(mB, mxB);  // finite: row w_lo is valid
        const float aA = exp2f(mA - nA), aB = exp2f(mB - nB);
        const float pA0 = exp2f(xA0 - nA), pB0 = exp2f(xB0 - nB);
        const float pA1 = exp2f(xA1 - nA), pB1 = exp2f(xB1 - nB);
        lA = lA * aA + pA0 + pA1;
        lB = lB * aB + pB0 + pB1;
        mA = nA;
        mB = nB;
        if (__any_sync(0xffffffffu, aA != 1.f || aB != 1.f)) {  // some head's max moved
#pragma unroll
          for (int mb = 0; mb < 16; ++mb) {
            O[mb][0] *= aA;
            O[mb][1] *= aB;
            O[mb][2] *= aA;
            O[mb][3] *= aB;
          }
        }
        // P^T fragments (k = rows, n = heads) by an 8x8 transpose of the score fragment
        const uint32_t pb0 = movmatrix_t(pack_bf16x2(pA0, pB0));
        const uint32_t pb1 = movmatrix_t(pack_bf16x2(pA1, pB1));
        // values O^T (256 channels x 8 heads) += C_hat^T . P^T
#pragma unroll
        for (int mb = 0; mb < 16; ++mb) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(tile + (mb >> 1) * SEGB + ((mb & 1) ? offV1 : offV0), a0, a1, a2, a3);
          mma_bf16(O[mb], a0, a1, a2, a3, pb0, pb1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty_bar[st]);
      ++job;
    }

    // ---- segment end
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      lA += __shfl_xor_sync(0xffffffffu, lA, o);
      lB += __shfl_xor_sync(0xffffffffu, lB, o);
    }
    // the four warps combine through shared memory: a sequence held by this
    // block alone is normalised and written out; the block's share of a split
    // sequence becomes one part (its max, sum and unnormalised output per
    // head)
    const bool whole = r_lo == 0 && r_hi == Lb;
    const int part = 2 * cta + (b == b_first ? 0 : 1);
    named_bar(1, CON_T);  // every warp is done with the query buffer
    if (g == 0) {
      sm.comb_ml[(cw * H + 2 * q) * 2 + 0] = mA;
      sm.comb_ml[(cw * H + 2 * q) * 2 + 1] = lA;
      sm.comb_ml[(cw * H + 2 * q + 1) * 2 + 0] = mB;
      sm.comb_ml[(cw * H + 2 * q + 1) * 2 + 1] = lB;
    }
    named_bar(1, CON_T);  // comb_ml complete
    float* wsc = sm.comb_ml + NCW * H * 2;  // [NCW][H] weights exp2(m_w - M), then [H] M and [H] L
    if (ctid < H) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NCW; ++w) M = fmaxf(M, sm.comb_ml[(w * H + ctid) * 2]);
      float Ls = 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w) {
        const float mw = sm.comb_ml[(w * H + ctid) * 2];
        const float sc = mw == -INFINITY ? 0.f : exp2f(mw - M);
        wsc[w * H + ctid] = sc;
        Ls += sc * sm.comb_ml[(w * H + ctid) * 2 + 1];
      }
      wsc[NCW * H + ctid] = M;
      wsc[NCW * H + H + ctid] = Ls;
    }
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
      // heads 4 pass .. 4 pass + 3 belong to the lanes with q >> 1 == pass
      if ((q >> 1) == pass) {
        const int hl = 2 * q - kCombHeads * pass;  // local head of O[.][0]
#pragma unroll
        for (int mb = 0; mb < 16; ++mb) {
          float* oA = sm.comb_o + (cw * kCombHeads + hl) * OSTR + 16 * mb + g;
          float* oB = oA + OSTR;
          oA[0] = O[mb][0];
          oB[0] = O[mb][1];
          oA[8] = O[mb][2];
          oB[8] = O[mb][3];
        }
      }
      named_bar(1, CON_T);
#pragma unroll
      for (int hl = 0; hl < kCombHeads; ++hl) {
        const int h = kCombHeads * pass + hl;
        const float M = wsc[NCW * H + h], Ls = wsc[NCW * H + H + h];
        float o0 = 0.f, o1 = 0.f;
#pragma unroll
        for (int w = 0; w < NCW; ++w) {
          const float sc = wsc[w * H + h];
          const float2 ov = *reinterpret_cast<const float2*>(sm.comb_o + (w * kCombHeads + hl) * OSTR + 2 * ctid);
          o0 += sc * ov.x;
          o1 += sc * ov.y;
        }
        if (whole) {
          const float inv = 1.f / Ls;
          *reinterpret_cast<float2*>(p.o.out + ((size_t)b * H + h) * R + 2 * ctid) = make_float2(o0 * inv, o1 * inv);
          if (p.o.lse && ctid == 0) p.o.lse[(size_t)b * H + h] = (M + log2f(Ls)) * 0.69314718055994531f;
        } else {
          *reinterpret_cast<float2*>(p.ws_o + ((size_t)part * H + h) * R + 2 * ctid) = make_float2(o0, o1);
          if (ctid == 0) reinterpret_cast<float2*>(p.ws_ml)[(size_t)part * H + h] = make_float2(M, Ls);
        }
      }
      named_bar(1, CON_T);  // the buffer is rewritten by the next pass / segment
    }
    ++seg;
  }
  if (!ok && ctid == 0) set_err(p.a.dev_err, MTLA_DEVERR_TIMEOUT);
}

// Combine of every split sequence's parts and the length bookkeeping.  One
// block of 256 threads per (sequence, head), thread = latent channel;
// launched right after the decode kernel with programmatic dependent launch
// (its blocks wait for the decode grid to complete).  The parts of sequence b
// are those of blocks cf..cl (slot 2c, or first_slot for block cf).  Per
// group of up to kGroup parts: their (max, sum) pairs go to shared memory
// while the first kChunk outputs are already in flight; warp 0 turns the
// pairs into weights e^{m_i - M}; every thread then sums its channel.  Groups
// merge online: out = sum_i e^{m_i - M} o_i / sum_i e^{m_i - M} l_i,
// lse = M + ln(sum).  Block (b, 0) also advances t_processed and cache_len
// and resets b's gate counter for the next call.
constexpr int kGroup = 256, kChunk = 40;
__global__ void __launch_bounds__(256) decode_combine_kernel(const Params p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float wts[kGroup];  // maxima, then weights
  __shared__ float lsum[kGroup];
  __shared__ float red[2];
  const int b = blockIdx.x / H, h = blockIdx.x % H, c = threadIdx.x;
  const int4 info = __ldcg(p.seq_info + b);  // rows, merged, first part's slot, parts
  if (h == 0 && c == 0) {
    if (info.y) p.a.t_processed[b] = p.a.t_processed[b] + 1;
    if (p.a.cache_len) p.a.cache_len[b] = info.x;
    p.gate_cnt[b] = 0u;
  }
  float* out = p.o.out + ((size_t)b * H + h) * R;
  if (info.x == 0) {
    if (h == 0 && c == 0) set_err(p.a.dev_err, MTLA_DEVERR_EMPTY);
    out[c] = 0.f;
    if (p.o.lse && c == 0) p.o.lse[(size_t)b * H + h] = -INFINITY;
    return;
  }
  if (info.w <= 1) return;  // one block held the whole sequence and wrote it
  const int nparts = info.w;
  const int cf = info.z >> 1;
  auto part_of = [&](int i) { return i == 0 ? info.z : 2 * (cf + i); };
  float M = -INFINITY, S = 0.f, acc = 0.f;
  for (int g0 = 0; g0 < nparts; g0 += kGroup) {
    const int ng = nparts - g0 < kGroup ? nparts - g0 : kGroup;
    float v[kChunk];
#pragma unroll
    for (int u = 0; u < kChunk; ++u)
      v[u] = u < ng ? __ldcg(p.ws_o + ((size_t)part_of(g0 + u) * H + h) * R + c) : 0.f;
    for (int i = c; i < ng; i += 256) {
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.ws_ml) + (size_t)part_of(g0 + i) * H + h);
      wts[i] = ml.x;
      lsum[i] = ml.y;
    }
    __syncthreads();
    if (c < 32) {
      float Mg = -INFINITY;
      for (int i = c; i < ng; i += 32) Mg = fmaxf(Mg, wts[i]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) Mg = fmaxf(Mg, __shfl_xor_sync(0xffffffffu, Mg, o));
      float Sg = 0.f;
      for (int i = c; i < ng; i += 32) {
        const float w = wts[i] == -INFINITY ? 0.f : exp2f(wts[i] - Mg);
        wts[i] = w;
        Sg += w * lsum[i];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) Sg += __shfl_xor_sync(0xffffffffu, Sg, o);
      if (c == 0) {
        red[0] = Mg;
        red[1] = Sg;
      }
    }
    __syncthreads();
    float accg = 0.f;
#pragma unroll
    for (int u = 0; u < kChunk; ++u)
      if (u < ng) accg += wts[u] * v[u];
    for (int i0 = kChunk; i0 < ng; i0 += kChunk) {
#pragma unroll
      for (int u = 0; u < kChunk; ++u)
        v[u] = i0 + u < ng ? __ldcg(p.ws_o + ((size_t)part_of(g0 + i0 + u) * H + h) * R + c) : 0.f;
#pragma unroll
      for (int u = 0; u < kChunk; ++u)
        if (i0 + u < ng) accg += wts[i0 + u] * v[u];
    }
    // merge this group into the running result
    const float Mg = red[0], Sg = red[1];
    const float nM = fmaxf(M, Mg);
    const float a = exp2f(M - nM), bg = exp2f(Mg - nM);  // a = 0 while M is -inf
    S = S * a + Sg * bg;
    acc = acc * a + accg * bg;
    M = nM;
    __syncthreads();  // wts / red are rewritten by the next group
  }
  out[c] = acc / S;
  if (p.o.lse && c == 0) p.o.lse[(size_t)b * H + h] = (M + log2f(S)) * 0.69314718055994531f;
}

int grid_size() {
  int dev = 0, sms = 0, occ = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  // two blocks of ~107 KB need the largest shared-memory configuration
  for (const void* fn : {(const void*)decode_tc_kernel<2>, (const void*)decode_tc_kernel<8>}) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes()) != cudaSuccess)
      return 0;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared) !=
        cudaSuccess)
      return 0;
    int o = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, fn, NT, smem_bytes()) != cudaSuccess) return 0;
    occ = occ == 0 ? o : (o < occ ? o : occ);
  }
  if (occ < 1) return 0;
  const int g = sms * (occ < 2 ? occ : 2);
  return g < MAXG ? g : MAXG;
}

}  // namespace dtc

cudaError_t launch_decode_tc(const dtc::Params& p, const CUtensorMap& map64, const CUtensorMap& map8, int grid,
                             cudaStream_t st) {
  const size_t smem = dtc::smem_bytes();
  // the attributes are set once per device (also keeps the call out of stream captures)
  static uint64_t done_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(done_mask & (1ull << dev))) {
    for (const void* fn : {(const void*)dtc::decode_tc_kernel<2>, (const void*)dtc::decode_tc_kernel<8>}) {
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
      if (e != cudaSuccess) return e;
    }
    // the same shared-memory configuration for the combine kernel, so that an
    // SM running its blocks can take the next step's decode blocks at once
    e = cudaFuncSetAttribute(dtc::decode_combine_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    if (dev < 64) done_mask |= 1ull << dev;
  }
  // programmatic dependent launch: the blocks may start (barrier set-up,
  // tensor-map prefetch) while the previous launch on the stream finishes;
  // griddepcontrol.wait holds them before their first read
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(dtc::NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = p.tok_per_unit == 2 ? cudaLaunchKernelEx(&cfg, dtc::decode_tc_kernel<2>, map64, map8, p)
                          : cudaLaunchKernelEx(&cfg, dtc::decode_tc_kernel<8>, map64, map8, p);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg2 = {};
  cfg2.gridDim = dim3((unsigned)(p.B * dtc::H));
  cfg2.blockDim = dim3(256);
  cfg2.stream = st;
  cfg2.attrs = attr;
  cfg2.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg2, dtc::decode_combine_kernel, p);
}

}  // namespace mtla
