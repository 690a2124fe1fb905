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
//    boxes {32 elements, 9 chunks, 64 rows} and 64-byte swizzle (a ragged last
//    tile uses 8-row boxes), NS stages deep, completion on mbarriers.
//  * Four consumer warps each own 16 rows of a tile.  Scores S^T = rows . Q^T
//    (M = rows, N = the 8 heads, K = 288) and values O^T += C_hat^T . P^T
//    (M = 256 latent channels, N = 8 heads, K = rows) run on the tensor cores
//    with bf16 operands and fp32 accumulators; the score fragment becomes the
//    value-MMA operand with one in-register 8x8 transpose (movmatrix).  Each
//    warp keeps its own online-softmax state, so no block barrier is needed
//    per tile.
//  * The merge of the new tokens is spread over the whole grid: the gate
//    pre-activations Linear(c_t) = c_t W_c + b_c of all B tokens are cut into
//    channel-major slices, one per block, computed while the block's first
//    tiles are in flight (each block reads about one column of W_c).  The
//    block owning a sequence's tail row waits (bounded) for all slices, then
//    forms the gate, the gated entry and the updated row in fp32, writes it to
//    the cache in bf16 and patches it into the tile before the tile is used.
//  * Launched with programmatic dependent launch: the next call's blocks are
//    scheduled while this call's last blocks finish and wait for it before
//    touching memory.
//  * Partial results of sequences split between blocks go to the workspace;
//    the last block to finish a sequence (atomic ticket) combines them.  No
//    block ever waits for another.  The last block of the grid advances
//    t_processed and resets the counters.  Every block's share and first
//    sequence are tabulated once in shared memory, so the bookkeeping in the
//    loops needs no integer division.
#include "kernels.cuh"

namespace mtla {
namespace dtc {

// every region starts on a 128-byte boundary (the tail row is read with
// 16-byte vector loads, the mbarriers need 8)
constexpr size_t kAlign = 128;
__host__ __device__ constexpr size_t rup(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
constexpr int kCombHeads = 4;  // heads per pass of the block combine
constexpr int QSTR = D / 2 + 4;  // words per query row in shared memory (148: conflict-free)
static_assert(17 * H * 2 <= NCW * kCombHeads * OSTR, "combine scratch must fit the combine buffer");
static_assert((size_t)H * QSTR * 4 <= (size_t)NCW * kCombHeads * OSTR * 4, "query buffer must fit the combine buffer");
constexpr size_t kOffComb = rup((size_t)NS * STAGE);
constexpr size_t kOffCombMl = kOffComb + rup((size_t)NCW * kCombHeads * OSTR * 4);
constexpr size_t kOffPrefix = kOffCombMl + rup((size_t)NCW * H * 2 * 4);
constexpr size_t kOffMeta = kOffPrefix + rup((size_t)(MAXB + 1) * 8);
constexpr size_t kOffScan = kOffMeta + rup((size_t)MAXB * 4);
constexpr size_t kOffLo = kOffScan + rup(128 * 8);
constexpr size_t kOffFs = kOffLo + rup((size_t)(MAXG + 1) * 8);
constexpr size_t kOffSlots = kOffFs + rup((size_t)MAXG * 4);
constexpr size_t kOffC = kOffSlots + rup((size_t)MAXG * 4);
constexpr size_t kOffTail = kOffC + rup((size_t)R * 4);
constexpr size_t kOffBar = kOffTail + rup((size_t)D * 2);
constexpr size_t kOffFlags = kOffBar + rup(2 * NS * 8);
constexpr size_t kSmemUsed = kOffFlags + rup(16);
static_assert(kOffTail % 16 == 0 && kOffBar % 8 == 0, "shared-memory regions must stay aligned");

size_t smem_bytes() { return kSmemUsed + 1024; }  // + slack to align the base to 1024

size_t workspace_bytes(int B, int grid) {
  size_t b = 0;
  b += ((size_t)B + 2) * 4;
  b = (b + 255) & ~(size_t)255;
  b += (size_t)B * D * 4;
  b = (b + 255) & ~(size_t)255;
  b += (size_t)2 * grid * H * 2 * 4;
  b = (b + 255) & ~(size_t)255;
  b += (size_t)2 * grid * H * R * 4;
  return b;
}

// byte offset, inside a swizzled tile, of row `row`, 16-byte chunk `ch` (0..35):
// TMA's 64-byte swizzle XORs chunk bits [4:5] with address bits [7:8]
__host__ __device__ __forceinline__ uint32_t swz_off(int row, int ch) {
  const uint32_t seg = (uint32_t)row * ROWB + (uint32_t)(ch >> 2) * 64u;
  return seg + ((((uint32_t)ch & 3u) ^ ((seg >> 7) & 3u)) << 4);
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
  int32_t* slots;     // [G] workspace slots of the sequence being combined
  float* c_sm;
  __nv_bfloat16* tail_sm;
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
  s.scan = reinterpret_cast<int64_t*>(p + kOffScan);
  s.lo = reinterpret_cast<int64_t*>(p + kOffLo);
  s.fs = reinterpret_cast<int32_t*>(p + kOffFs);
  s.slots = reinterpret_cast<int32_t*>(p + kOffSlots);
  s.c_sm = reinterpret_cast<float*>(p + kOffC);
  s.tail_sm = reinterpret_cast<__nv_bfloat16*>(p + kOffTail);
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

constexpr uint32_t kSpinLimit = 1u << 22;  // x 64 ns sleeps: gives up after ~0.3 s

__device__ __forceinline__ int ld_acquire_gpu(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ int64_t rows_of(const uint32_t* meta, int b) {
  return (int64_t)(meta[b] & (kMetaMergeOk - 1));
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

  // let the next launch on the stream be scheduled as soon as blocks retire;
  // then wait for the previous launch before reading anything it may write
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sm.full_bar[i], 1);
      mbar_init(&sm.empty_bar[i], NCW);
    }
    fence_mbar_init();
  }
  if (warp == NCW && lane == 0) {
    prefetch_tmap(&map64);
    prefetch_tmap(&map8);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- 1. rows per sequence and the cost prefix (identical in every block)
  const int per = (B + 127) / 128;
  if (tid < 128) {
    int64_t sum = 0;
    for (int b = tid * per; b < B && b < (tid + 1) * per; ++b) {
      const int64_t t0 = p.a.t_processed[b];
      const int64_t t = t0 + (with_merge ? 1 : 0);
      const int64_t off = p.a.seq_offset[b], cap = p.a.seq_capacity[b];
      int64_t L = t > 0 ? group_of(t, s) : 0;
      bool ok = with_merge;
      const bool report = (cta == 0);
      if (t0 < 0 || off < 0 || cap < 0 || off > p.a.cache_rows || cap > p.a.cache_rows - off) {
        if (report) set_err(p.a.dev_err, MTLA_DEVERR_CAPACITY);
        L = 0;
        ok = false;
      } else if (L > cap) {
        if (report) set_err(p.a.dev_err, MTLA_DEVERR_CAPACITY);
        L = cap;
        ok = false;
      }
      if (L >= (int64_t)kMetaMergeOk) {  // beyond what one call can address
        if (report) set_err(p.a.dev_err, MTLA_DEVERR_CAPACITY);
        L = 0;
        ok = false;
      }
      if (ok && group_of(t, s) > p.m.J_max) {
        if (report) set_err(p.a.dev_err, MTLA_DEVERR_PE_RANGE);
        ok = false;
      }
      sm.meta[b] = (uint32_t)L | (ok ? kMetaMergeOk : 0u);
      sum += L + mcost;
    }
    sm.scan[tid] = sum;
  }
  __syncthreads();
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
  __syncthreads();
  if (tid < 128) {
    int64_t run = sm.scan[tid];
    for (int b = tid * per; b < B && b < (tid + 1) * per; ++b) {
      sm.prefix[b] = run;
      run += rows_of(sm.meta, b) + mcost;
    }
  }
  const int64_t C = sm.prefix[B];
  // share starts: block c owns cost positions [lo[c], lo[c+1])
  for (int c = tid; c <= G; c += NT) sm.lo[c] = C > 0 ? (int64_t)c * C / G : 0;
  __syncthreads();
  // first sequence with rows in each share (B if none)
  for (int c = tid; c < G; c += NT) {
    const int64_t x = sm.lo[c];
    int b = upper_bound_i64(sm.prefix, B + 1, x) - 1;
    if (b < 0) b = 0;
    if (b < B && x - sm.prefix[b] >= rows_of(sm.meta, b)) ++b;
    sm.fs[c] = (x < sm.lo[c + 1]) ? b : B;
  }
  __syncthreads();

  const int64_t my_lo = sm.lo[cta], my_hi = sm.lo[cta + 1];
  const int b_first = sm.fs[cta];
  const __nv_bfloat16* cache = reinterpret_cast<const __nv_bfloat16*>(p.a.cache);

  // ======================= producer warp =======================
  if (warp == NCW) {
    if (lane == 0 && my_lo < my_hi) {
      uint32_t job = 0;
      bool ok = true;
      for (int b = b_first; b < B && sm.prefix[b] < my_hi && ok; ++b) {
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
            tma_load_3d(dst, &map64, 0, 0, (int32_t)(row0 + u), &sm.full_bar[st]);
          } else {
            const int nsub = (int)((nrows + SUB - 1) / SUB);
            mbar_arrive_expect_tx(&sm.full_bar[st], (uint32_t)(nsub * SUB * ROWB));
            for (int i = 0; i < nsub; ++i)
              tma_load_3d(dst + i * SUB * ROWB, &map8, 0, 0, (int32_t)(row0 + u + i * SUB), &sm.full_bar[st]);
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
  uint32_t job = 0;
  bool ok = true;

  // ---- merge gates: this block's slice of Linear(c_t) = c_t W_c + b_c,
  // channel-major (index k * B + b), while its first tiles are in flight
  if (with_merge) {
    const int N = B * D;
    const int i_lo = (int)((int64_t)cta * N / G), i_hi = (int)((int64_t)(cta + 1) * N / G);
    float* wcol = sm.c_sm;  // one column of W_c
    const uint4* cnew = reinterpret_cast<const uint4*>(p.m.c_new);
    for (int k = i_lo / B; i_lo < i_hi && k <= (i_hi - 1) / B; ++k) {
      const int b_lo = i_lo - k * B > 0 ? i_lo - k * B : 0;
      const int b_hi = i_hi - k * B < B ? i_hi - k * B : B;
      for (int i = ctid; i < R; i += 128) wcol[i] = __ldg(p.m.W_c + (size_t)i * D + k);
      named_bar(1, 128);
      float wv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) wv[e] = wcol[8 * lane + e];
      const float bias = __ldg(p.m.b_c + k);
      // warp cw takes sequences b_lo + cw, + NCW, ...; four at a time so that
      // their loads overlap; lane covers inputs 8 lane .. 8 lane + 7
      for (int b0 = b_lo + cw; b0 < b_hi; b0 += 4 * NCW) {
        uint4 cv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int bb = b0 + u * NCW;
          cv[u] = bb < b_hi ? __ldg(cnew + (size_t)bb * (R / 8) + lane) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&cv[u]);
          float acc = 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h2[e]);
            acc = fmaf(f.x, wv[2 * e], acc);
            acc = fmaf(f.y, wv[2 * e + 1], acc);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          const int bb = b0 + u * NCW;
          if (lane == 0 && bb < b_hi) p.gates[(size_t)bb * D + k] = acc + bias;
        }
      }
      named_bar(1, 128);  // the column buffer is reused for the next channel
    }
    __threadfence();
    named_bar(1, 128);
    if (ctid == 0) atomicAdd(p.gate_done, 1);
  }

  for (int b = b_first; b < B && sm.prefix[b] < my_hi; ++b) {
    const int64_t Lb = rows_of(sm.meta, b);
    const int64_t r_lo = (my_lo > sm.prefix[b] ? my_lo : sm.prefix[b]) - sm.prefix[b];
    const int64_t r_end = sm.prefix[b] + Lb < my_hi ? sm.prefix[b] + Lb : my_hi;
    const int64_t r_hi = r_end - sm.prefix[b];
    if (r_lo >= r_hi) continue;
    const bool merge_here = (sm.meta[b] & kMetaMergeOk) && r_hi == Lb;
    const bool full = (r_lo == 0 && r_hi == Lb);

    // [q_abs ; q_rope] of the 8 heads into shared memory (rows padded to
    // QSTR words so the B-fragment loads below are free of bank conflicts);
    // the buffer shares space with the combine buffer, which is only used
    // after the segment's last tile
    {
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
    const uint32_t qrow = smem_u32(sm.comb_o) + (uint32_t)(g * QSTR + q) * 4u;
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    float O[16][4];
#pragma unroll
    for (int mb = 0; mb < 16; ++mb) O[mb][0] = O[mb][1] = O[mb][2] = O[mb][3] = 0.f;


    for (int64_t u = r_lo; u < r_hi; u += UNIT) {
      const bool is_tail = merge_here && u + UNIT >= r_hi;
      if (is_tail) {
        // every block's slice of the gates must be written (bounded wait)
        if (ctid == 0) {
          uint32_t it = 0;
          while (ld_acquire_gpu(p.gate_done) < G) {
            if (++it > kSpinLimit) {
              set_err(p.a.dev_err, MTLA_DEVERR_TIMEOUT);
              break;
            }
            __nanosleep(64);
          }
        }
        named_bar(1, 128);
        // gate, gated entry and the updated tail row (fp32 math, bf16 storage)
        const int64_t t = (int64_t)p.a.t_processed[b] + 1;
        const int64_t j = group_of(t, s);
        const bool opens = opens_row(t, s);
        __nv_bfloat16* row = const_cast<__nv_bfloat16*>(cache) + (p.a.seq_offset[b] + j - 1) * p.a.row_stride;
        const __nv_bfloat16* cn = reinterpret_cast<const __nv_bfloat16*>(p.m.c_new) + (size_t)b * R;
        const __nv_bfloat16* kR = reinterpret_cast<const __nv_bfloat16*>(p.m.kR_new) + (size_t)b * DR;
        const float* Pj = p.m.P + (j - 1) * D;
#pragma unroll
        for (int ci = 0; ci < 3; ++ci) {
          const int k = ctid + 128 * ci;
          if (k < D) {
            const float gv = __ldcg(p.gates + (size_t)b * D + k);
            const float w = sigmoidf_(__fmul_rn(gv, Pj[k]));
            const float x = __bfloat162float(k < R ? cn[k] : kR[k - R]);
            const float e = __fmul_rn(w, x);
            const float v = opens ? e : __fadd_rn(__bfloat162float(row[k]), e);
            const __nv_bfloat16 vb = __float2bfloat16_rn(v);
            row[k] = vb;
            sm.tail_sm[k] = vb;
          }
        }
        named_bar(1, 128);
      }

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
            const uint4* src = reinterpret_cast<const uint4*>(sm.tail_sm);
            for (int ch = lane; ch < 36; ch += 32) {
              const uint4 v = src[ch];
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
          ldsm_x4(tile + swz_off(arow, 2 * kk + ach), a0, a1, a2, a3);
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
#pragma unroll
        for (int mb = 0; mb < 16; ++mb) {
          O[mb][0] *= aA;
          O[mb][1] *= aB;
          O[mb][2] *= aA;
          O[mb][3] *= aB;
        }
        // P^T fragments (k = rows, n = heads) by an 8x8 transpose of the score fragment
        const uint32_t pb0 = movmatrix_t(pack_bf16x2(pA0, pB0));
        const uint32_t pb1 = movmatrix_t(pack_bf16x2(pA1, pB1));
        // values O^T (256 channels x 8 heads) += C_hat^T . P^T
#pragma unroll
        for (int mb = 0; mb < 16; ++mb) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(tile + swz_off(vrow, 2 * mb + vch), a0, a1, a2, a3);
          mma_bf16(O[mb], a0, a1, a2, a3, pb0, pb1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty_bar[st]);
      ++job;
    }

    // ---- segment end: combine the four warps, then write out or a partial
    named_bar(1, 128);  // every warp is done with the query buffer
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      lA += __shfl_xor_sync(0xffffffffu, lA, o);
      lB += __shfl_xor_sync(0xffffffffu, lB, o);
    }
    if (g == 0) {
      sm.comb_ml[(cw * H + 2 * q) * 2 + 0] = mA;
      sm.comb_ml[(cw * H + 2 * q) * 2 + 1] = lA;
      sm.comb_ml[(cw * H + 2 * q + 1) * 2 + 0] = mB;
      sm.comb_ml[(cw * H + 2 * q + 1) * 2 + 1] = lB;
    }
    const int nslot = full ? -1 : 2 * cta + (b == b_first ? 0 : 1);
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
#pragma unroll 1
      for (int hl = 0; hl < kCombHeads; ++hl) {
        const int h = kCombHeads * pass + hl;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NCW; ++w) M = fmaxf(M, sm.comb_ml[(w * H + h) * 2]);
        float Ls = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll
        for (int w = 0; w < NCW; ++w) {
          const float mw = sm.comb_ml[(w * H + h) * 2];
          const float sc = mw == -INFINITY ? 0.f : exp2f(mw - M);
          Ls += sc * sm.comb_ml[(w * H + h) * 2 + 1];
          const float2 ov = *reinterpret_cast<const float2*>(sm.comb_o + (w * kCombHeads + hl) * OSTR + 2 * ctid);
          o0 += sc * ov.x;
          o1 += sc * ov.y;
        }
        if (full) {
          const float inv = 1.f / Ls;
          *reinterpret_cast<float2*>(p.o.out + ((size_t)b * H + h) * R + 2 * ctid) =
              make_float2(o0 * inv, o1 * inv);
          if (p.o.lse && ctid == 0) p.o.lse[(size_t)b * H + h] = (M + log2f(Ls)) * 0.69314718055994531f;
        } else {
          *reinterpret_cast<float2*>(p.ws_o + ((size_t)nslot * H + h) * R + 2 * ctid) = make_float2(o0, o1);
          if (ctid == 0) {
            p.ws_ml[((size_t)nslot * H + h) * 2 + 0] = M;
            p.ws_ml[((size_t)nslot * H + h) * 2 + 1] = Ls;
          }
        }
      }
      named_bar(1, 128);  // the buffer is rewritten by the next pass / segment
    }
    if (!full) {
      __threadfence();
      named_bar(1, 128);
      if (ctid == 0) {
        // the blocks holding part of sequence b and their workspace slots
        const int64_t first_pos = sm.prefix[b], last_pos = sm.prefix[b] + Lb - 1;
        const int c_first = upper_bound_i64(sm.lo, G + 1, first_pos) - 1;
        const int c_last = upper_bound_i64(sm.lo, G + 1, last_pos) - 1;
        int nparts = 0;
        for (int c = c_first; c <= c_last; ++c)
          if (sm.lo[c] < sm.lo[c + 1]) sm.slots[nparts++] = 2 * c + (sm.fs[c] == b ? 0 : 1);
        const int old = atomicAdd(&p.tickets[b], 1);
        sm.flags[0] = (old == nparts - 1) ? nparts : 0;
        __threadfence();
      }
      named_bar(1, 128);
      const int nparts = sm.flags[0];
      if (nparts) {
        // last block of this sequence: combine every block's partial.  All
        // loads of a phase are independent, so each phase costs about one L2
        // round trip whatever the number of parts.
        // phase 1: per head, running (max, sum) over the parts, 16 groups of 8 threads
        float* red = sm.comb_o;  // [16][H][2], free at this point
        {
          const int h = ctid & 7, grp = ctid >> 3;
          float M = -INFINITY, Ls = 0.f;
          for (int i = grp; i < nparts; i += 16) {
            const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.ws_ml) + (size_t)sm.slots[i] * H + h);
            if (ml.x == -INFINITY) continue;
            const float nM = fmaxf(M, ml.x);
            Ls = Ls * exp2f(M - nM) + ml.y * exp2f(ml.x - nM);
            M = nM;
          }
          red[(grp * H + h) * 2 + 0] = M;
          red[(grp * H + h) * 2 + 1] = Ls;
        }
        named_bar(1, 128);
        if (ctid < H) {
          float M = -INFINITY, Ls = 0.f;
          for (int grp = 0; grp < 16; ++grp) {
            const float m = red[(grp * H + ctid) * 2], l = red[(grp * H + ctid) * 2 + 1];
            if (m == -INFINITY) continue;
            const float nM = fmaxf(M, m);
            Ls = Ls * exp2f(M - nM) + l * exp2f(m - nM);
            M = nM;
          }
          red[(16 * H + ctid) * 2 + 0] = M;
          red[(16 * H + ctid) * 2 + 1] = Ls;
          if (p.o.lse) p.o.lse[(size_t)b * H + ctid] = (M + log2f(Ls)) * 0.69314718055994531f;
        }
        named_bar(1, 128);
        // phase 2: thread -> head ctid >> 4, 16 channels; parts weighted by exp2(m_i - M) / L
        {
          const int h = ctid >> 4, c0 = (ctid & 15) * 16;
          const float M = red[(16 * H + h) * 2], inv = 1.f / red[(16 * H + h) * 2 + 1];
          float4 acc[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
          for (int i = 0; i < nparts; ++i) {
            const int slot = sm.slots[i];
            const float mc = __ldcg(p.ws_ml + ((size_t)slot * H + h) * 2);
            const float4* src = reinterpret_cast<const float4*>(p.ws_o + ((size_t)slot * H + h) * R + c0);
            float4 v[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) v[k] = __ldcg(src + k);
            const float sc = mc == -INFINITY ? 0.f : exp2f(mc - M);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              acc[k].x += sc * v[k].x;
              acc[k].y += sc * v[k].y;
              acc[k].z += sc * v[k].z;
              acc[k].w += sc * v[k].w;
            }
          }
          float4* dst = reinterpret_cast<float4*>(p.o.out + ((size_t)b * H + h) * R + c0);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dst[k] = make_float4(acc[k].x * inv, acc[k].y * inv, acc[k].z * inv, acc[k].w * inv);
        }
        if (ctid == 0) p.tickets[b] = 0;
      }
      named_bar(1, 128);  // slots / flags are reused by the next segment
    }
  }
  if (!ok && ctid == 0) set_err(p.a.dev_err, MTLA_DEVERR_TIMEOUT);

  // ---- grid epilogue: the last block advances the per-sequence state
  named_bar(1, 128);
  if (ctid == 0) {
    __threadfence();
    const int old = atomicAdd(p.done, 1);
    sm.flags[1] = (old == G - 1) ? 1 : 0;
    __threadfence();
  }
  named_bar(1, 128);
  if (sm.flags[1]) {
    for (int b = ctid; b < B; b += 128) {
      const int64_t Lb = rows_of(sm.meta, b);
      if (with_merge && (sm.meta[b] & kMetaMergeOk)) p.a.t_processed[b] = p.a.t_processed[b] + 1;
      if (p.a.cache_len) p.a.cache_len[b] = (int32_t)Lb;
      if (Lb == 0) {
        set_err(p.a.dev_err, MTLA_DEVERR_EMPTY);
        for (int i = 0; i < H * R; ++i) p.o.out[(size_t)b * H * R + i] = 0.f;
        if (p.o.lse)
          for (int h = 0; h < H; ++h) p.o.lse[(size_t)b * H + h] = -INFINITY;
      }
    }
    if (ctid == 0) {
      *p.done = 0;
      *p.gate_done = 0;
    }
  }
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
    if (dev < 64) done_mask |= 1ull << dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(dtc::NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, dtc::decode_tc_kernel, map64, map8, p);
}

}  // namespace mtla
