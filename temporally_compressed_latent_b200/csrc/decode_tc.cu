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
//    into equal shares for a persistent grid of one block per SM (split-L,
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
//  * The merge of a new token is done by the block owning that sequence's
//    tail row: W_c (fp32) streams through the same pipeline (8 stages), the
//    gate and the updated row are computed in fp32, written to the cache in
//    bf16 and patched into the tile before it is used.
//  * Partial results of sequences split between blocks go to the workspace;
//    the last block to finish a sequence (atomic ticket) combines them.  No
//    block ever waits for another.  The last block of the grid advances
//    t_processed and resets the counters.
#include "kernels.cuh"

namespace mtla {
namespace dtc {

size_t smem_bytes() {
  size_t b = 0;
  b += (size_t)NS * STAGE;                 // stages
  b += (size_t)NCW * H * OSTR * 4;         // combine O
  b += (size_t)NCW * H * 2 * 4;            // combine m, l
  b += (size_t)(MAXB + 1) * 8;             // cost prefix (int64)
  b += (size_t)MAXB * 4;                   // rows + flags per sequence
  b += 128 * 8;                            // scan scratch (int64)
  b += (size_t)R * 4;                      // c_new in fp32
  b += (size_t)D * 2;                      // merged tail row (bf16)
  b += 2 * NS * 8;                         // mbarriers
  b += 16;                                 // flags
  return b + 1024;                         // alignment slack
}

size_t workspace_bytes(int B, int grid) {
  size_t b = 0;
  b += ((size_t)B + 1) * 4;
  b = (b + 255) & ~(size_t)255;
  b += (size_t)2 * grid * H * 2 * 4;
  b = (b + 255) & ~(size_t)255;
  b += (size_t)2 * grid * H * R * 4;
  return b;
}

// byte address in a swizzled tile of row `row`, 16-byte chunk `ch` (0..35)
__device__ __forceinline__ uint32_t swz(uint32_t tile, int row, int ch) {
  const uint32_t seg = tile + (uint32_t)row * ROWB + (uint32_t)(ch >> 2) * 64u;
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
  p += NS * STAGE;
  s.comb_o = reinterpret_cast<float*>(p);
  p += NCW * H * OSTR * 4;
  s.comb_ml = reinterpret_cast<float*>(p);
  p += NCW * H * 2 * 4;
  s.prefix = reinterpret_cast<int64_t*>(p);
  p += (MAXB + 1) * 8;
  s.meta = reinterpret_cast<uint32_t*>(p);
  p += MAXB * 4;
  s.scan = reinterpret_cast<int64_t*>(p);
  p += 128 * 8;
  s.c_sm = reinterpret_cast<float*>(p);
  p += R * 4;
  s.tail_sm = reinterpret_cast<__nv_bfloat16*>(p);
  p += D * 2;
  s.full_bar = reinterpret_cast<uint64_t*>(p);
  p += NS * 8;
  s.empty_bar = reinterpret_cast<uint64_t*>(p);
  p += NS * 8;
  s.flags = reinterpret_cast<int32_t*>(p);
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

struct Part {
  const int64_t* prefix;
  const uint32_t* meta;
  int B;
  int G;
  int64_t C;
  __device__ __forceinline__ int64_t lo(int c) const { return (int64_t)c * C / G; }
  __device__ __forceinline__ int64_t rows(int b) const { return (int64_t)(meta[b] & (kMetaMergeOk - 1)); }
  // block whose share holds cost position pos
  __device__ __forceinline__ int owner(int64_t pos) const { return (int)(((pos + 1) * G - 1) / C); }
  // first sequence with rows inside block c's share (B if none)
  __device__ __forceinline__ int first_seq(int c) const {
    const int64_t x = lo(c);
    int b = upper_bound_i64(prefix, B + 1, x) - 1;
    if (b < 0) b = 0;
    if (b < B && x - prefix[b] >= rows(b)) ++b;
    return b;
  }
};

__global__ void __launch_bounds__(NT, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap map64, const __grid_constant__ CUtensorMap map8,
                 const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const Smem sm = carve(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = p.B, s = p.a.s, G = gridDim.x, cta = blockIdx.x;
  const bool with_merge = p.with_merge != 0;

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
      sum += L + (with_merge ? p.merge_cost : 0);
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
  }
  __syncthreads();
  if (tid < 128) {
    int64_t run = sm.scan[tid];
    for (int b = tid * per; b < B && b < (tid + 1) * per; ++b) {
      sm.prefix[b] = run;
      run += (int64_t)(sm.meta[b] & (kMetaMergeOk - 1)) + (with_merge ? p.merge_cost : 0);
    }
  }
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sm.full_bar[i], 1);
      mbar_init(&sm.empty_bar[i], NCW);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    // total = prefix of the last sequence + its cost
    const int64_t last = B > 0 ? sm.prefix[B - 1] + (int64_t)(sm.meta[B - 1] & (kMetaMergeOk - 1)) +
                                     (with_merge ? p.merge_cost : 0)
                               : 0;
    sm.prefix[B] = last;
  }
  __syncthreads();

  Part part;
  part.prefix = sm.prefix;
  part.meta = sm.meta;
  part.B = B;
  part.G = G;
  part.C = sm.prefix[B];
  const int64_t my_lo = part.C > 0 ? part.lo(cta) : 0;
  const int64_t my_hi = part.C > 0 ? part.lo(cta + 1) : 0;
  const int b_first = part.C > 0 ? part.first_seq(cta) : B;

  const __nv_bfloat16* cache = reinterpret_cast<const __nv_bfloat16*>(p.a.cache);

  // ======================= producer warp =======================
  if (warp == NCW) {
    if (lane == 0 && my_lo < my_hi) {
      prefetch_tmap(&map64);
      prefetch_tmap(&map8);
      uint32_t job = 0;
      bool ok = true;
      for (int b = b_first; b < B && sm.prefix[b] < my_hi && ok; ++b) {
        const int64_t Lb = part.rows(b);
        const int64_t r_lo = (my_lo > sm.prefix[b] ? my_lo : sm.prefix[b]) - sm.prefix[b];
        const int64_t r_end = sm.prefix[b] + Lb < my_hi ? sm.prefix[b] + Lb : my_hi;
        const int64_t r_hi = r_end - sm.prefix[b];
        if (r_lo >= r_hi) continue;
        const bool merge_here = (sm.meta[b] & kMetaMergeOk) && r_hi == Lb;
        const int64_t row0 = p.a.seq_offset[b];
        for (int64_t u = r_lo; u < r_hi && ok; u += UNIT) {
          const bool is_tail = merge_here && u + UNIT >= r_hi;
          if (is_tail) {
            for (int w = 0; w < N_WC && ok; ++w, ++job) {
              const int st = job % NS;
              if (job >= NS && !mbar_wait(&sm.empty_bar[st], ((job / NS) & 1) ^ 1)) { ok = false; break; }
              mbar_arrive_expect_tx(&sm.full_bar[st], STAGE);
              bulk_load(sm.stages + st * STAGE, p.m.W_c + (size_t)w * WC_ROWS * D, STAGE, &sm.full_bar[st]);
            }
            if (!ok) break;
          }
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
  uint32_t job = 0;
  bool ok = true;

  for (int b = b_first; b < B && sm.prefix[b] < my_hi; ++b) {
    const int64_t Lb = part.rows(b);
    const int64_t r_lo = (my_lo > sm.prefix[b] ? my_lo : sm.prefix[b]) - sm.prefix[b];
    const int64_t r_end = sm.prefix[b] + Lb < my_hi ? sm.prefix[b] + Lb : my_hi;
    const int64_t r_hi = r_end - sm.prefix[b];
    if (r_lo >= r_hi) continue;
    const bool merge_here = (sm.meta[b] & kMetaMergeOk) && r_hi == Lb;
    const bool full = (r_lo == 0 && r_hi == Lb);

    // B operand of the score MMA: [q_abs ; q_rope] of head g, k = 16kk + 2q (+1, +8, +9)
    uint32_t bq[18][2];
    {
      const uint32_t* qa = reinterpret_cast<const uint32_t*>(
          reinterpret_cast<const __nv_bfloat16*>(p.o.q_abs) + ((size_t)b * H + g) * R);
      const uint32_t* qr = reinterpret_cast<const uint32_t*>(
          reinterpret_cast<const __nv_bfloat16*>(p.o.q_rope) + ((size_t)b * H + g) * DR);
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        bq[kk][0] = __ldg(qa + kk * 8 + q);
        bq[kk][1] = __ldg(qa + kk * 8 + q + 4);
      }
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        bq[16 + kk][0] = __ldg(qr + kk * 8 + q);
        bq[16 + kk][1] = __ldg(qr + kk * 8 + q + 4);
      }
    }
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    float O[16][4];
#pragma unroll
    for (int mb = 0; mb < 16; ++mb) O[mb][0] = O[mb][1] = O[mb][2] = O[mb][3] = 0.f;

    float gacc[3] = {0.f, 0.f, 0.f};
    if (merge_here) {
      const __nv_bfloat16* c = reinterpret_cast<const __nv_bfloat16*>(p.m.c_new) + (size_t)b * R;
      for (int i = ctid; i < R; i += 128) sm.c_sm[i] = __bfloat162float(c[i]);
      named_bar(1, 128);
    }

    for (int64_t u = r_lo; u < r_hi; u += UNIT) {
      const bool is_tail = merge_here && u + UNIT >= r_hi;
      if (is_tail) {
        for (int w = 0; w < N_WC; ++w, ++job) {
          const int st = job % NS;
          if (ok && !mbar_wait(&sm.full_bar[st], (job / NS) & 1)) ok = false;
          const float* Wsm = reinterpret_cast<const float*>(sm.stages + st * STAGE);
#pragma unroll
          for (int ci = 0; ci < 3; ++ci) {
            const int k = ctid + 128 * ci;
            if (k < D) {
              float a = gacc[ci];
#pragma unroll 8
              for (int i = 0; i < WC_ROWS; ++i) a = fmaf(sm.c_sm[w * WC_ROWS + i], Wsm[i * D + k], a);
              gacc[ci] = a;
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.empty_bar[st]);
        }
        // gate, gated entry and the updated tail row (fp32 math, bf16 storage)
        const int64_t t = (int64_t)p.a.t_processed[b] + 1;
        const int64_t j = group_of(t, s);
        const bool opens = opens_row(t, s);
        __nv_bfloat16* row = const_cast<__nv_bfloat16*>(cache) + (p.a.seq_offset[b] + j - 1) * p.a.row_stride;
        const __nv_bfloat16* kR = reinterpret_cast<const __nv_bfloat16*>(p.m.kR_new) + (size_t)b * DR;
        const float* Pj = p.m.P + (j - 1) * D;
#pragma unroll
        for (int ci = 0; ci < 3; ++ci) {
          const int k = ctid + 128 * ci;
          if (k < D) {
            const float gv = __fadd_rn(gacc[ci], p.m.b_c[k]);
            const float w = sigmoidf_(__fmul_rn(gv, Pj[k]));
            const float x = k < R ? sm.c_sm[k] : __bfloat162float(kR[k - R]);
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
      const uint32_t tile = smem_u32(sm.stages + st * STAGE);
      const int rows = (int)(r_hi - u < UNIT ? r_hi - u : UNIT);
      const int w_lo = 16 * cw;
      if (w_lo < rows) {
        bool wrote = false;
        if (w_lo + 16 > rows) {
          // rows past the segment's end: zero them (they may hold anything)
          for (int i = lane; i < (w_lo + 16 - rows) * 36; i += 32) {
            const int rr = rows + i / 36, ch = i % 36;
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(swz(tile, rr, ch)), "r"(0u) : "memory");
          }
          wrote = true;
        }
        if (is_tail) {
          const int lr = (int)(Lb - 1 - u);
          if (lr >= w_lo && lr < w_lo + 16) {
            const uint4* src = reinterpret_cast<const uint4*>(sm.tail_sm);
            for (int ch = lane; ch < 36; ch += 32) {
              const uint4 v = src[ch];
              asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(swz(tile, lr, ch)), "r"(v.x), "r"(v.y),
                           "r"(v.z), "r"(v.w) : "memory");
            }
            wrote = true;
          }
        }
        if (wrote) fence_proxy_async_smem();
        __syncwarp();

        // scores S^T (16 rows x 8 heads) = rows . [q_abs ; q_rope]^T
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
        const int arow = w_lo + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int kk = 0; kk < 18; kk += 2) {
          uint32_t a0, a1, a2, a3, c0, c1, c2, c3;
          ldsm_x4(swz(tile, arow, 2 * kk + (lane >> 4)), a0, a1, a2, a3);
          ldsm_x4(swz(tile, arow, 2 * kk + 2 + (lane >> 4)), c0, c1, c2, c3);
          mma_bf16(sa, a0, a1, a2, a3, bq[kk][0], bq[kk][1]);
          mma_bf16(sb, c0, c1, c2, c3, bq[kk + 1][0], bq[kk + 1][1]);
        }
        const bool v0 = (w_lo + g) < rows, v1 = (w_lo + g + 8) < rows;
        const float xA0 = v0 ? (sa[0] + sb[0]) * sl2 : -INFINITY;
        const float xB0 = v0 ? (sa[1] + sb[1]) * sl2 : -INFINITY;
        const float xA1 = v1 ? (sa[2] + sb[2]) * sl2 : -INFINITY;
        const float xB1 = v1 ? (sa[3] + sb[3]) * sl2 : -INFINITY;
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
        const int vrow = w_lo + (lane & 7) + (lane >> 4) * 8;
        const int vch = (lane >> 3) & 1;
#pragma unroll
        for (int mb = 0; mb < 16; ++mb) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(swz(tile, vrow, 2 * mb + vch), a0, a1, a2, a3);
          mma_bf16(O[mb], a0, a1, a2, a3, pb0, pb1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty_bar[st]);
      ++job;
    }

    // ---- segment end: combine the four warps, then write out or a partial
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
#pragma unroll
    for (int mb = 0; mb < 16; ++mb) {
      float* oA = sm.comb_o + (cw * H + 2 * q) * OSTR + 16 * mb + g;
      float* oB = sm.comb_o + (cw * H + 2 * q + 1) * OSTR + 16 * mb + g;
      oA[0] = O[mb][0];
      oB[0] = O[mb][1];
      oA[8] = O[mb][2];
      oB[8] = O[mb][3];
    }
    named_bar(1, 128);

    const int nslot = full ? -1 : 2 * cta + (b == b_first ? 0 : 1);
#pragma unroll 1
    for (int h = 0; h < H; ++h) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NCW; ++w) M = fmaxf(M, sm.comb_ml[(w * H + h) * 2]);
      float Ls = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w) {
        const float mw = sm.comb_ml[(w * H + h) * 2];
        const float sc = mw == -INFINITY ? 0.f : exp2f(mw - M);
        Ls += sc * sm.comb_ml[(w * H + h) * 2 + 1];
        const float2 ov = *reinterpret_cast<const float2*>(sm.comb_o + (w * H + h) * OSTR + 2 * ctid);
        o0 += sc * ov.x;
        o1 += sc * ov.y;
      }
      if (full) {
        const float inv = 1.f / Ls;
        *reinterpret_cast<float2*>(p.o.out + ((size_t)b * H + h) * R + 2 * ctid) = make_float2(o0 * inv, o1 * inv);
        if (p.o.lse && ctid == 0) p.o.lse[(size_t)b * H + h] = (M + log2f(Ls)) * 0.69314718055994531f;
      } else {
        *reinterpret_cast<float2*>(p.ws_o + ((size_t)nslot * H + h) * R + 2 * ctid) = make_float2(o0, o1);
        if (ctid == 0) {
          p.ws_ml[((size_t)nslot * H + h) * 2 + 0] = M;
          p.ws_ml[((size_t)nslot * H + h) * 2 + 1] = Ls;
        }
      }
    }
    if (!full) {
      __threadfence();
      named_bar(1, 128);
      const int c_first = part.owner(sm.prefix[b]);
      const int c_last = part.owner(sm.prefix[b] + Lb - 1);
      if (ctid == 0) {
        int nparts = 0;
        for (int c = c_first; c <= c_last; ++c) nparts += part.lo(c) < part.lo(c + 1) ? 1 : 0;
        const int old = atomicAdd(&p.tickets[b], 1);
        sm.flags[0] = (old == nparts - 1) ? 1 : 0;
        __threadfence();
      }
      named_bar(1, 128);
      if (sm.flags[0]) {
        // last block of this sequence: combine every block's partial
#pragma unroll 1
        for (int h = 0; h < H; ++h) {
          float M = -INFINITY;
          for (int c = c_first; c <= c_last; ++c) {
            if (part.lo(c) >= part.lo(c + 1)) continue;
            const int slot = 2 * c + (part.first_seq(c) == b ? 0 : 1);
            M = fmaxf(M, __ldcg(p.ws_ml + ((size_t)slot * H + h) * 2));
          }
          float Ls = 0.f, o0 = 0.f, o1 = 0.f;
          for (int c = c_first; c <= c_last; ++c) {
            if (part.lo(c) >= part.lo(c + 1)) continue;
            const int slot = 2 * c + (part.first_seq(c) == b ? 0 : 1);
            const float mc = __ldcg(p.ws_ml + ((size_t)slot * H + h) * 2);
            const float sc = mc == -INFINITY ? 0.f : exp2f(mc - M);
            Ls += sc * __ldcg(p.ws_ml + ((size_t)slot * H + h) * 2 + 1);
            const float2 ov = __ldcg(reinterpret_cast<const float2*>(p.ws_o + ((size_t)slot * H + h) * R + 2 * ctid));
            o0 += sc * ov.x;
            o1 += sc * ov.y;
          }
          const float inv = 1.f / Ls;
          *reinterpret_cast<float2*>(p.o.out + ((size_t)b * H + h) * R + 2 * ctid) = make_float2(o0 * inv, o1 * inv);
          if (p.o.lse && ctid == 0) p.o.lse[(size_t)b * H + h] = (M + log2f(Ls)) * 0.69314718055994531f;
        }
        if (ctid == 0) p.tickets[b] = 0;
      }
    }
    named_bar(1, 128);  // combine buffers are reused by the next segment
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
      const int64_t Lb = part.rows(b);
      if (with_merge && (sm.meta[b] & kMetaMergeOk)) p.a.t_processed[b] = p.a.t_processed[b] + 1;
      if (p.a.cache_len) p.a.cache_len[b] = (int32_t)Lb;
      if (Lb == 0) {
        set_err(p.a.dev_err, MTLA_DEVERR_EMPTY);
        for (int i = 0; i < H * R; ++i) p.o.out[(size_t)b * H * R + i] = 0.f;
        if (p.o.lse)
          for (int h = 0; h < H; ++h) p.o.lse[(size_t)b * H + h] = -INFINITY;
      }
    }
    if (ctid == 0) *p.done = 0;
  }
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
    if (dev < 64) done_mask |= 1ull << dev;
  }
  dtc::decode_tc_kernel<<<grid, dtc::NT, smem, st>>>(map64, map8, p);
  return cudaGetLastError();
}

}  // namespace mtla
