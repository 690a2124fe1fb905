// Split-L tensor-core decode step for bf16 caches with H = 8, r = 256, d_R = 32.
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
//    balanced to the row; a merge counts as MERGE_COST rows).
//  * One producer warp streams 64-row tiles HBM -> shared memory with 3-D TMA
//    boxes {32 elements, 64 rows, 9 planes}: the tensor map orders the row's
//    nine 32-element segments as the outer dimension, so a tile lands as nine
//    [64 rows x 64 B] planes with the 64-byte swizzle, whose XOR phase then
//    depends on the row only (every ldmatrix address is a per-lane base plus a
//    constant; this is also the canonical K-major SW64 operand layout).  A
//    ragged last tile uses {32, 8, 1} boxes.  NS stages, mbarrier completion.
//  * Four consumer warps each own 16 rows of a tile.  Scores S^T = rows . Q^T
//    (M = rows, N = the 8 heads, K = 288) and values O^T += C_hat^T . P^T
//    (M = 256 latent channels, N = 8 heads, K = rows) run on the tensor cores
//    with bf16 operands and fp32 accumulators; the score fragment becomes the
//    value-MMA operand with one in-register 8x8 transpose (movmatrix).  Each
//    warp keeps its own online-softmax state, so no block barrier is needed
//    per tile.
//  * The merge of the B new tokens runs in a small kernel launched just before
//    (gate contraction with W_c read as coalesced row segments, gate, gated
//    entry, append / in-place update of the tail row, written to the cache and
//    to a workspace copy).  It releases the decode grid at once (programmatic
//    dependent launch), so the decode blocks set up and stream meanwhile.
//    Every block visits its share's sequences last to first, so a tail row is
//    the last tile of its block; the warp holding it waits for the merge
//    kernel (hardware-tracked) and patches the finished row into the tile.
//  * At the end of each of its sequences a block's four warps combine their
//    online-softmax states through shared memory.  A sequence held by one
//    block is written out; otherwise the block writes one partial (max, sum,
//    unnormalised output per head) to the workspace and moves on: no fence,
//    no atomic, no block ever waits for another.  A second, small kernel chained with
//    programmatic dependent launch (its blocks are resident and waiting
//    before the first kernel ends) combines the split sequences from a
//    per-sequence partition summary that block 0 publishes (one dependent
//    load, then every part's loads at once) and advances t_processed /
//    cache_len.  Every block's share and first sequence are tabulated once in
//    shared memory, so the bookkeeping in the loops needs no division.
#include "kernels.cuh"

namespace mtla {
namespace dtc {

// every region starts on a 128-byte boundary (the tail row is read with
// 16-byte vector loads, the mbarriers need 8)
constexpr size_t kAlign = 128;
__host__ __device__ constexpr size_t rup(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
constexpr int kCombHeads = 4;  // heads per pass of the block combine
constexpr int QSTR = D / 2 + 4;  // words per query row in shared memory (148: conflict-free)
static_assert((size_t)H * QSTR * 4 <= (size_t)NCW * kCombHeads * OSTR * 4, "query buffer must fit the combine buffer");
constexpr size_t kOffComb = rup((size_t)NS * STAGE);
constexpr size_t kOffCombMl = kOffComb + rup((size_t)NCW * kCombHeads * OSTR * 4);
constexpr size_t kOffPrefix = kOffCombMl + rup((size_t)NCW * H * 2 * 4 + (size_t)(NCW + 2) * H * 4);
constexpr size_t kOffMeta = kOffPrefix + rup((size_t)(MAXB + 1) * 8);
constexpr size_t kOffLo = kOffMeta + rup((size_t)MAXB * 4);
constexpr size_t kOffFs = kOffLo + rup((size_t)(MAXG + 1) * 8);
constexpr size_t kOffQx = kOffFs + rup((size_t)MAXG * 4);
constexpr size_t kOffBar = kOffQx + rup((size_t)H * QSTR * 4);
constexpr size_t kOffFlags = kOffBar + rup(2 * NS * 8);
constexpr size_t kSmemUsed = kOffFlags + rup(16);
static_assert(kOffQx % 16 == 0 && kOffBar % 8 == 0, "shared-memory regions must stay aligned");
static_assert(128 * 8 <= (size_t)NCW * kCombHeads * OSTR * 4, "scan scratch must fit the combine buffer");
// two decode blocks plus two merge-kernel blocks (1 KB each) fit one SM's 228 KB
static_assert(2 * (kSmemUsed + 1024 + 1024) + 2 * (1024 + 1024) <= 233472, "shared memory per SM");

size_t smem_bytes() { return kSmemUsed + 1024; }  // + slack to align the base to 1024

WsLayout ws_layout(int B, int grid) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  WsLayout l;
  l.seq_info = 0;                                     // [B] per-sequence partition summary
  l.tails = up(l.seq_info + (size_t)B * 16);          // [B][D] tail rows
  l.ml = up(l.tails + (size_t)B * D * 2);             // parts: (max, sum) per head, two slots per block
  l.o = up(l.ml + (size_t)2 * grid * H * 2 * 4);      // parts: unnormalised outputs
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

constexpr uint32_t kMetaMergeOk = 1u << 30;

struct Smem {
  uint8_t* stages;
  float* comb_o;
  float* comb_ml;
  int64_t* prefix;
  uint32_t* meta;     // rows (bits 0..29) | merge ok (bit 30)
  int64_t* scan;
  int64_t* lo;        // [G + 1] first cost position of each block's share
  int32_t* fs;        // [G] first sequence with rows in each block's share
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
  s.lo = reinterpret_cast<int64_t*>(p + kOffLo);
  s.fs = reinterpret_cast<int32_t*>(p + kOffFs);
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

constexpr int PRO_T = 32 * (NCW + 1);  // threads of the consumer and producer warps

// 16-byte asynchronous global -> shared copies (completion per thread)
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ int64_t rows_of(const uint32_t* meta, int b) {
  return (int64_t)(meta[b] & (kMetaMergeOk - 1));
}

// Block c's share of the C cost positions starts at c C / G.
// floor(c C / G) in double precision: c C < 2^53 is exact, and a quotient
// that is not an integer lies at least 1/G from one, far beyond the rounding
// error (below 2^-3 ulp of 2^40), so truncation gives the integer quotient
// without a 64-bit integer division
__device__ __forceinline__ int64_t share_start(int c, int64_t C, int G) {
  return C > 0 ? (int64_t)(((double)c * (double)C) / (double)G) : 0;
}
// The first sequence with rows in the share [lo, hi), B if the share is empty.
__device__ __forceinline__ int first_seq(const int64_t* prefix, const uint32_t* meta, int B, int64_t lo, int64_t hi) {
  if (lo >= hi) return B;
  int b = upper_bound_i64(prefix, B + 1, lo) - 1;
  if (b < 0) b = 0;
  if (b < B && lo - prefix[b] >= rows_of(meta, b)) ++b;
  return b;
}

// Sequence b after this call: its rows, whether its new token is merged, and
// the device-error bits the checks raise.  The merge kernel (which writes the
// tail row) and the decode kernel (which partitions the rows) decide alike.
struct SeqState {
  int64_t t;        // processed tokens after the call
  int64_t L;        // cache rows after the call
  bool merge_ok;
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
  if (st.L >= (int64_t)kMetaMergeOk) {  // beyond what one call can address
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

__global__ void __launch_bounds__(NT, 2)
decode_tc_kernel(const __grid_constant__ CUtensorMap map64, const __grid_constant__ CUtensorMap map8,
                 const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const Smem sm = carve(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = p.B, s = p.a.s, G = gridDim.x, cta = blockIdx.x;
  const bool with_merge = p.with_merge != 0;
  const int64_t mcost = with_merge ? p.merge_cost : 0;

  // let the next launch on the stream be scheduled as soon as blocks retire.
  // Without a merge, wait for the previous launch before reading anything it
  // may write; with a merge the merge kernel just before has already waited
  // for it, and only the tail rows it writes need it to be complete.
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
  if (!with_merge) asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- 1. rows per sequence and the cost prefix (identical in every block)
  const int per = (B + 127) / 128;
  if (tid < 128) {
    int64_t sum = 0;
    for (int b = tid * per; b < B && b < (tid + 1) * per; ++b) {
      const SeqState st = seq_state(p, b, with_merge);
      if (st.err && cta == 0) set_err(p.a.dev_err, st.err);
      // a merged sequence, or (several tokens per call) any sequence with rows:
      // its last row is patched from the tails buffer
      const bool patched = st.merge_ok || (p.patch && st.L > 0 && st.err == 0);
      sm.meta[b] = (uint32_t)st.L | (patched ? kMetaMergeOk : 0u);
      sum += st.L + mcost;
    }
    sm.scan[tid] = sum;
  }
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
  // this block's share: cost positions [my_lo, my_hi).  While the prefix is
  // written, the threads that own the sequences holding its first and last
  // positions record them: its first sequence with rows (B if none, the rule
  // block 0 tabulates for every block below with first_seq) and the sequence
  // of its last position
  const int64_t my_lo = share_start(cta, C, G), my_hi = share_start(cta + 1, C, G);
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
  // row (whose merge the merge kernel finishes meanwhile) is the block's last
  // tile
  const int b_first = my_lo < my_hi ? sm.flags[0] : B;
  const int b_last = my_lo < my_hi ? sm.flags[1] : -1;
  const __nv_bfloat16* cache = reinterpret_cast<const __nv_bfloat16*>(p.a.cache);

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
  int seg = 0;

  // the partition as the combine kernel needs it, published by block 0 while
  // its first tile is in flight: rows, merge flag, the first part's slot and
  // the number of parts (blocks cf..cl; block c > cf stored its part in slot
  // 2c, block cf in 2cf or 2cf + 1)
  if (cta == 0) {
    for (int c = ctid; c <= G; c += 128) sm.lo[c] = share_start(c, C, G);
    named_bar(1, 128);
    for (int c = ctid; c < G; c += 128) sm.fs[c] = first_seq(sm.prefix, sm.meta, B, sm.lo[c], sm.lo[c + 1]);
    named_bar(1, 128);
    for (int bb = ctid; bb < B; bb += 128) {
      const int64_t Lb = rows_of(sm.meta, bb);
      const int ok_m = (sm.meta[bb] & kMetaMergeOk) ? 1 : 0;
      int first = 0, n = 0;
      if (Lb > 0) {
        const int cf = upper_bound_i64(sm.lo, G + 1, sm.prefix[bb]) - 1;
        const int cl = upper_bound_i64(sm.lo, G + 1, sm.prefix[bb] + Lb - 1) - 1;
        first = 2 * cf + (sm.fs[cf] == bb ? 0 : 1);
        n = cl - cf + 1;
      }
      p.seq_info[bb] = make_int4((int)Lb, ok_m, first, n);
    }
  }

  for (int b = b_last; b >= b_first; --b) {
    const int64_t Lb = rows_of(sm.meta, b);
    const int64_t r_lo = (my_lo > sm.prefix[b] ? my_lo : sm.prefix[b]) - sm.prefix[b];
    const int64_t r_end = sm.prefix[b] + Lb < my_hi ? sm.prefix[b] + Lb : my_hi;
    const int64_t r_hi = r_end - sm.prefix[b];
    if (r_lo >= r_hi) continue;
    const bool merge_here = (sm.meta[b] & kMetaMergeOk) && r_hi == Lb;

    // [q_abs ; q_rope] of the 8 heads into shared memory (rows padded to
    // QSTR words so the B-fragment loads below are free of bank conflicts):
    // the prefetched buffer for the second sequence, else loaded now into the
    // combine buffer, which is only used after the segment's last tile
    const bool pre = (seg == 1 && b == b_second);
    if (pre) {
      cp_async_wait_all();
      named_bar(1, 128);
    } else {
      if (seg > 0) named_bar(1, 128);  // every warp is done with the previous queries
      const uint32_t* qa = reinterpret_cast<const uint32_t*>(
          reinterpret_cast<const __nv_bfloat16*>(p.o.q_abs) + (size_t)b * H * R);
      const uint32_t* qr = reinterpret_cast<const uint32_t*>(
          reinterpret_cast<const __nv_bfloat16*>(p.o.q_rope) + (size_t)b * H * DR);
      uint32_t* qs = reinterpret_cast<uint32_t*>(sm.comb_o);
      for (int i = ctid; i < H * (D / 2); i += 128) {
        const int h = i / (D / 2), w = i % (D / 2);
        qs[h * QSTR + w] = w < R / 2 ? __ldg(qa + h * (R / 2) + w) : __ldg(qr + h * (DR / 2) + (w - R / 2));
      }
      named_bar(1, 128);
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
            // the merge kernel wrote the updated row (the copy the tile holds
            // may predate it); hardware-tracked wait for that kernel, no polling
            asm volatile("griddepcontrol.wait;" ::: "memory");
            const uint4* src = reinterpret_cast<const uint4*>(p.tails + (size_t)b * D);
            for (int ch = lane; ch < 36; ch += 32) {
              const uint4 v = __ldcg(src + ch);
              asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(tile + swz_off(lr, ch)), "r"(v.x),
                           "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
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
    // head) for the combine kernel
    const bool whole = r_lo == 0 && r_hi == Lb;
    const int part = 2 * cta + (b == b_first ? 0 : 1);
    named_bar(1, 128);  // every warp is done with the query buffer
    if (g == 0) {
      sm.comb_ml[(cw * H + 2 * q) * 2 + 0] = mA;
      sm.comb_ml[(cw * H + 2 * q) * 2 + 1] = lA;
      sm.comb_ml[(cw * H + 2 * q + 1) * 2 + 0] = mB;
      sm.comb_ml[(cw * H + 2 * q + 1) * 2 + 1] = lB;
    }
    named_bar(1, 128);  // comb_ml complete
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
      named_bar(1, 128);
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
      named_bar(1, 128);  // the buffer is rewritten by the next pass / segment
    }
    ++seg;
  }
  // a block with an empty share holds no parts; its slot says so to the combine
  if (my_lo >= my_hi && ctid < H)
    reinterpret_cast<float2*>(p.ws_ml)[(size_t)2 * cta * H + ctid] = make_float2(-INFINITY, 0.f);
  if (!ok && ctid == 0) set_err(p.a.dev_err, MTLA_DEVERR_TIMEOUT);
}

// Combine of every sequence's parts and the length bookkeeping.  One block
// of 256 threads per (sequence, head), thread = latent channel; launched right
// after the decode kernel with programmatic dependent launch (its blocks wait
// for the decode grid to complete).  The parts of sequence b are those of
// blocks cf..cl (slot 2c, or 2cf + 1 for block cf when b is not its first
// sequence); a block whose share is empty marks its slot with a zero weight,
// and a part of weight zero is never read.  Per group of up to kGroup parts: their (max, sum)
// pairs go to shared memory while the first kChunk outputs are already in
// flight; warp 0 turns the pairs into weights e^{m_i - M}; every thread then
// sums its channel.  Groups merge online:
// out = sum_i e^{m_i - M} o_i / sum_i e^{m_i - M} l_i, lse = M + ln(sum).
constexpr int kGroup = 256, kChunk = 40;
__global__ void __launch_bounds__(256) decode_combine_kernel(const Params p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float wts[kGroup];  // maxima, then weights
  __shared__ float lsum[kGroup];
  __shared__ float red[2];
  const int b = blockIdx.x / H, h = blockIdx.x % H, c = threadIdx.x;
  const int4 info = __ldcg(p.seq_info + b);  // rows, merge ok, first block's slot, blocks
  if (h == 0 && c == 0) {
    if (p.with_merge && info.y) p.a.t_processed[b] = p.a.t_processed[b] + 1;
    if (p.a.cache_len) p.a.cache_len[b] = info.x;
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
        const float w = wts[i] == -INFINITY ? 0.f : exp2f(wts[i] - Mg);  // a warp without rows weighs 0
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
      if (u < ng && wts[u] != 0.f) accg += wts[u] * v[u];  // a part without rows is never read
    for (int i0 = kChunk; i0 < ng; i0 += kChunk) {
#pragma unroll
      for (int u = 0; u < kChunk; ++u)
        v[u] = i0 + u < ng ? __ldcg(p.ws_o + ((size_t)part_of(g0 + i0 + u) * H + h) * R + c) : 0.f;
#pragma unroll
      for (int u = 0; u < kChunk; ++u)
        if (i0 + u < ng && wts[i0 + u] != 0.f) accg += wts[i0 + u] * v[u];
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

// The merge of every sequence's new token (Linear(c_t) of the merge, the gate,
// the gated entry and the append / in-place update of the tail row), before
// the decode kernel reads the cache.  Block = 32 channels x 2 tokens, 128
// threads: warp w takes input rows 64w .. 64w+63 of the gate contraction (its
// W_c column segments all in flight at once), lanes are channels; the four
// warps' partial sums are added in a fixed order, so the result is
// deterministic.  Small on purpose (1 KB of shared memory, few registers): its
// blocks share SMs with two decode blocks, which start while it runs.  The
// updated row goes to the cache and to the workspace copy that the decode
// kernel patches into its tile.
constexpr int kMergeTok = 2;
__global__ void __launch_bounds__(128) decode_merge_kernel(const Params p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float part[4][kMergeTok][32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = blockIdx.x % (D / 32), bt = blockIdx.x / (D / 32);
  const int k = kt * 32 + lane, b0 = bt * kMergeTok, i0 = w * 64;
  const __nv_bfloat16* cn = reinterpret_cast<const __nv_bfloat16*>(p.m.c_new);
  float acc[kMergeTok];
#pragma unroll
  for (int u = 0; u < kMergeTok; ++u) acc[u] = 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int ib = i0 + 32 * half;
    float wv[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) wv[i] = __ldg(p.m.W_c + (size_t)(ib + i) * D + k);
    float cv[kMergeTok];
#pragma unroll
    for (int u = 0; u < kMergeTok; ++u)
      cv[u] = b0 + u < p.B ? __bfloat162float(cn[(size_t)(b0 + u) * R + ib + lane]) : 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i)
#pragma unroll
      for (int u = 0; u < kMergeTok; ++u) acc[u] = fmaf(__shfl_sync(0xffffffffu, cv[u], i), wv[i], acc[u]);
  }
#pragma unroll
  for (int u = 0; u < kMergeTok; ++u) part[w][u][lane] = acc[u];
  __syncthreads();
  if (w >= kMergeTok) return;
  const int u = w;  // thread -> token b0 + u, channel k
  float g = 0.f;
#pragma unroll
  for (int ww = 0; ww < 4; ++ww) g += part[ww][u][lane];
  const int b = b0 + u;
  if (b >= p.B) return;
  const SeqState st = seq_state(p, b, true);
  if (!st.merge_ok) return;  // the decode kernel reports why
  const int s = p.a.s;
  const int64_t j = group_of(st.t, s);
  const bool opens = opens_row(st.t, s);
  __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(p.a.cache) + (p.a.seq_offset[b] + j - 1) * p.a.row_stride;
  const float gv = g + __ldg(p.m.b_c + k);
  const float wt = sigmoidf_(__fmul_rn(gv, __ldg(p.m.P + (j - 1) * D + k)));
  const __nv_bfloat16* xin = k < R ? reinterpret_cast<const __nv_bfloat16*>(p.m.c_new) + (size_t)b * R + k
                                   : reinterpret_cast<const __nv_bfloat16*>(p.m.kR_new) + (size_t)b * DR + (k - R);
  const float e = __fmul_rn(wt, __bfloat162float(*xin));
  const float v = opens ? e : __fadd_rn(__bfloat162float(row[k]), e);
  const __nv_bfloat16 vb = __float2bfloat16_rn(v);
  row[k] = vb;
  p.tails[(size_t)b * D + k] = vb;
}

int grid_size() {
  int dev = 0, sms = 0, occ = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes()) !=
      cudaSuccess)
    return 0;
  // two blocks of ~110 KB need the largest shared-memory configuration
  if (cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared) != cudaSuccess)
    return 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_tc_kernel, NT, smem_bytes()) != cudaSuccess)
    return 0;
  if (occ < 1) return 0;
  const int g = sms * (occ < 2 ? occ : 2);
  return g < MAXG ? g : MAXG;
}

}  // namespace dtc

cudaError_t launch_decode_tc(const dtc::Params& p, const CUtensorMap& map64, const CUtensorMap& map8, int grid,
                             cudaStream_t st) {
  const size_t smem = dtc::smem_bytes();
  // the attribute is set once per device (also keeps the call out of stream captures)
  static uint64_t done_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(done_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(dtc::decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(dtc::decode_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    // the same shared-memory configuration for the kernels around it, so that
    // an SM running one of their blocks can take decode blocks at once
    // (changing the configuration waits for the SM to drain)
    e = cudaFuncSetAttribute(dtc::decode_merge_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(dtc::decode_combine_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    if (dev < 64) done_mask |= 1ull << dev;
  }
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
  if (p.with_merge) {
    cudaLaunchConfig_t cfg0 = {};
    cfg0.gridDim = dim3((unsigned)((dtc::D / 32) * ((p.B + dtc::kMergeTok - 1) / dtc::kMergeTok)));
    cfg0.blockDim = dim3(128);
    cfg0.stream = st;
    // plain stream order (no early launch): launched early, its blocks would
    // pile onto the SMs the previous step's kernels leave free first and keep
    // decode blocks off them; after the previous step they spread one per SM
    cfg0.numAttrs = 0;
    e = cudaLaunchKernelEx(&cfg0, dtc::decode_merge_kernel, p);
    if (e != cudaSuccess) return e;
  }
  e = cudaLaunchKernelEx(&cfg, dtc::decode_tc_kernel, map64, map8, p);
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
