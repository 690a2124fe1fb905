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
//  * The gate pre-activations are a dense contraction (tokens x 256 x 288), so
//    they run as tcgen05.mma with fp32 accumulators in TMEM.  W_c stays
//    near-fp32: each CTA splits its half of W_c (144 output channels) into
//    bf16 hi + lo parts once, keeps both resident in shared memory (K-major,
//    128-byte swizzle) and issues two MMAs per K step; the latents are bf16
//    already, so the products are exact and only the lo part's rounding
//    (2^-17 relative) remains.  The two channel halves of a token tile run in
//    neighbouring CTAs, so the second read of the latent tile hits L2.
//  * An MMA tile is 128 rows = 4 warp blocks of 32.  A warp block holds
//    floor(32 / s) * s consecutive tokens that start on a group boundary, so
//    no group crosses a warp: the running merge inside a group is a
//    Hillis-Steele scan over lanes of ceil(log2 s) shuffle steps, with no
//    carry between warps or tiles.  TMA loads the four 32-row boxes of a K
//    block (64 latents, 128 B per row) into one pipeline stage.
//  * Roles: one TMA warp, one MMA warp (one elected lane issues), twelve
//    epilogue warps (three per TMEM lane quarter, 48 of the 144 channels
//    each: the epilogue is latency-bound, so more warps overlap more of it).
//    The accumulator is
//    double-buffered in TMEM so a tile's epilogue overlaps the next tile's
//    MMAs.  The epilogue reads each token's P row, b_c and its own latent /
//    RoPE key (just loaded, so L2-resident), forms the gate and the gated
//    entry in fp32 with non-contracted multiplies, scans, and stores bf16.
#include "kernels.cuh"

namespace mtla {
namespace mtc {

constexpr int R = 256, DR = 32, D = R + DR;
constexpr int NH = D / 2;            // output channels per CTA (one half): 144
constexpr int KB = R / 64;           // K blocks of 64 latents (128-byte rows): 4
constexpr int ROWS = 128;            // MMA rows: 4 warp blocks of 32
constexpr int WROWS = 32;            // rows of one warp block / one TMA box
constexpr int ABLK = ROWS * 128;     // one K block of the latent tile: 16384 B
constexpr int KS = 4;                // latent-tile stages
constexpr int WKB = NH * 128;        // one K block of a W part: 18432 B
constexpr int WBYTES = KB * WKB;     // one W part (hi or lo): 73728 B
constexpr int NEPI = 12;             // epilogue warps: three per TMEM lane quarter, three chunks each
constexpr int TMA_WARP = NEPI, MMA_WARP = NEPI + 1, NT = 32 * (NEPI + 2);
constexpr int NCH = NH / 16;         // 16-column chunks per half: 9
constexpr uint32_t TMEM_COLS = 512, ACC_STRIDE = 256;
constexpr uint32_t IDESC = umma_idesc_bf16(ROWS, NH, false, false);

constexpr size_t OFF_WHI = 0;
constexpr size_t OFF_WLO = OFF_WHI + WBYTES;
constexpr size_t OFF_A = OFF_WLO + WBYTES;
constexpr size_t OFF_BAR = OFF_A + (size_t)KS * ABLK;
constexpr int NBAR = 2 * KS + 2 + 2 + 1;
constexpr size_t OFF_TMEM = OFF_BAR + NBAR * 8;
constexpr size_t OFF_BC = OFF_TMEM + 16;             // this CTA's half of b_c (fp32)
constexpr size_t SMEM_USED = OFF_BC + NH * 4;
static_assert(OFF_WLO % 1024 == 0 && OFF_A % 1024 == 0 && WKB % 1024 == 0, "swizzle atoms must be 1024-aligned");
static_assert(NH % 16 == 0 && NH <= 256, "N of one MMA");

size_t smem_bytes() { return SMEM_USED + 1024; }

struct Params {
  int B, s, tpw, tiles_per_seq, n_tiles;
  int64_t T, n_groups;
  const __nv_bfloat16* c;
  const __nv_bfloat16* kR;
  const float* W_c;
  const float* b_c;
  const float* P;
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

// The gate's sigmoid with the hardware exponential and divide: a few fp32 ulp
// (relative error near 1e-6), far below the bf16 rounding of what it scales;
// the fp32 paths of the library keep the correctly rounded form.
__device__ __forceinline__ float gate_sigmoid(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}

__global__ void __launch_bounds__(NT, 1) merge_tc_kernel(const __grid_constant__ CUtensorMap cmap, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* const k_full = bar;                // [KS]
  uint64_t* const k_empty = bar + KS;          // [KS]
  uint64_t* const acc_full = bar + 2 * KS;     // [2]
  uint64_t* const acc_empty = bar + 2 * KS + 2;  // [2]
  uint64_t* const mma_done = bar + 2 * KS + 4;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = blockIdx.x & 1;
  const int G2 = gridDim.x >> 1;
  const int first = blockIdx.x >> 1;

  if (tid == 0) {
    for (int i = 0; i < KS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], NEPI);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == TMA_WARP && lane == 0) prefetch_tmap(&cmap);

  // this CTA's half of W_c -> bf16 hi + lo, K-major with the 128-byte swizzle:
  // output channel n, latents k = kb*64 + ch*8 .. +7 form one 16-byte chunk.
  // Each thread first loads all of its chunks (at most 11, 88 values), so the
  // L2 round trips overlap instead of following one another.
  constexpr int NIT = (KB * 8 * NH + NT - 1) / NT;
  float wv[NIT][8];
#pragma unroll
  for (int u = 0; u < NIT; ++u) {
    const int it = tid + u * NT;
    if (it < KB * 8 * NH) {
      const int n = it % NH, kc = it / NH;
      const float* src = p.W_c + (size_t)((kc >> 3) * 64 + (kc & 7) * 8) * D + half * NH + n;
#pragma unroll
      for (int e = 0; e < 8; ++e) wv[u][e] = __ldg(src + (size_t)e * D);
    }
  }
#pragma unroll
  for (int u = 0; u < NIT; ++u) {
    const int it = tid + u * NT;
    if (it >= KB * 8 * NH) break;
    const int n = it % NH, kc = it / NH;
    const int kb = kc >> 3, ch = kc & 7;
    const float* v = wv[u];
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float h0 = __bfloat162float(__float2bfloat16_rn(v[2 * e]));
      const float h1 = __bfloat162float(__float2bfloat16_rn(v[2 * e + 1]));
      hi[e] = pack_bf16x2(h0, h1);
      lo[e] = pack_bf16x2(v[2 * e] - h0, v[2 * e + 1] - h1);
    }
    const uint32_t off = (uint32_t)(kb * WKB + (n >> 3) * 1024 + (n & 7) * 128 + ((ch ^ (n & 7)) << 4));
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(sm + OFF_WHI + off)), "r"(hi[0]),
                 "r"(hi[1]), "r"(hi[2]), "r"(hi[3]) : "memory");
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(sm + OFF_WLO + off)), "r"(lo[0]),
                 "r"(lo[1]), "r"(lo[2]), "r"(lo[3]) : "memory");
  }
  float* const bc_s = reinterpret_cast<float*>(sm + OFF_BC);
  for (int n = tid; n < NH; n += NT) bc_s[n] = __ldg(p.b_c + half * NH + n);
  fence_proxy_async_smem();  // the tensor core reads what the threads wrote
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  bool ok = true;

  if (warp == TMA_WARP) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      uint32_t kc = 0;
      for (int it = first; it < p.n_tiles && ok; it += G2) {
        const int b = it / p.tiles_per_seq, tb = it % p.tiles_per_seq;
        const int64_t row_base = (int64_t)b * p.T;
        for (int kb = 0; kb < KB; ++kb, ++kc) {
          const int st = kc % KS;
          if (kc >= KS && !mbar_wait(&k_empty[st], ((kc / KS) & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[st], ABLK);
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            // a warp block past the prompt's end loads rows it never uses
            const int64_t n0 = ((int64_t)tb * 4 + w) * p.tpw;
            tma_load_2d(sm + OFF_A + st * ABLK + w * (WROWS * 128), &cmap, kb * 64, (int32_t)(row_base + n0),
                        &k_full[st]);
          }
        }
      }
      if (!ok) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
      // drain: no copy may still be writing shared memory when the block exits
      for (uint32_t j = kc > (uint32_t)KS ? kc - KS : 0; j < kc; ++j) mbar_wait(&k_full[j % KS], (j / KS) & 1);
    }
  } else if (warp == MMA_WARP) {
    // ======================= MMA issuer =======================
    // The whole warp runs the loop (warp-uniform operands); one elected lane
    // issues the MMAs and the commits that track them.
    const uint32_t sA = smem_u32(sm + OFF_A), sHi = smem_u32(sm + OFF_WHI), sLo = smem_u32(sm + OFF_WLO);
    uint32_t kc = 0, tc = 0;
    for (int it = first; it < p.n_tiles && ok; it += G2, ++tc) {
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
            const uint64_t ad = umma_desc(sA + st * ABLK + kk * 32, 16, 1024, 2);
            const uint64_t bh = umma_desc(sHi + kb * WKB + kk * 32, 16, 1024, 2);
            const uint64_t bl = umma_desc(sLo + kb * WKB + kk * 32, 16, 1024, 2);
            umma_bf16(dcol, ad, bh, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
            umma_bf16(dcol, ad, bl, IDESC, 1u);
          }
          umma_commit(&k_empty[st]);
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
  } else {
    // ======================= epilogue: gate, gated entry, group scan =======================
    const int q = warp & 3;                            // TMEM lane quarter = warp block
    const int cbeg = (warp >> 2) * (NCH / 3), cend = cbeg + NCH / 3;
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const int s = p.s;
    const int pos = lane % s;                          // position inside the token's group
    uint32_t tc = 0;
    for (int it = first; it < p.n_tiles && ok; it += G2, ++tc) {
      const int ab = tc & 1;
      const int b = it / p.tiles_per_seq, tb = it % p.tiles_per_seq;
      const int64_t n = ((int64_t)tb * 4 + q) * p.tpw + lane;  // 0-based token of sequence b
      const bool valid = lane < p.tpw && n < p.T;
      const int64_t nn = valid ? n : 0;
      const int64_t tok = (int64_t)b * p.T + nn;
      const int64_t grp = nn / s;                       // 0-based group = P row = cache row
      const bool closes = valid && (pos == s - 1 || n == p.T - 1);
      // a chunk's inputs (the token's latent or RoPE key, its group's P row)
      // do not depend on the accumulator: the first chunk's are requested
      // before the wait, every next chunk's while the current one is processed
      uint4 vin_c[2], vin_n[2];
      float4 pr_c[4], pr_n[4];
      auto fetch = [&](int c16, uint4 (&vi)[2], float4 (&pr)[4]) {
        if (!valid || c16 >= cend) return;
        const int ch0 = half * NH + c16 * 16;
        const __nv_bfloat16* vin = ch0 < R ? p.c + tok * R + ch0 : p.kR + tok * DR + (ch0 - R);
        vi[0] = __ldg(reinterpret_cast<const uint4*>(vin));
        vi[1] = __ldg(reinterpret_cast<const uint4*>(vin) + 1);
        const float4* Pr = reinterpret_cast<const float4*>(p.P + grp * D + ch0);
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) pr[e4] = __ldg(Pr + e4);
      };
      fetch(cbeg, vin_c, pr_c);
      if (!warp_wait(&acc_full[ab], (tc >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      for (int c16 = cbeg; c16 < cend; ++c16) {
        fetch(c16 + 1, vin_n, pr_n);
        uint32_t g[16];
        tmem_ld16(lane_base + ab * ACC_STRIDE + c16 * 16, g);
        tmem_wait_ld();
        const int ch0 = half * NH + c16 * 16;
        float x[16];
        if (valid) {
          float v[16];
          unpack8(vin_c[0], v);
          unpack8(vin_c[1], v + 8);
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            const float pe[4] = {pr_c[e4].x, pr_c[e4].y, pr_c[e4].z, pr_c[e4].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int k = 4 * e4 + e;
              const float gate = __fadd_rn(__uint_as_float(g[k]), bc_s[c16 * 16 + k]);
              const float w = gate_sigmoid(__fmul_rn(gate, pe[e]));
              x[k] = __fmul_rn(w, v[k]);
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) x[k] = 0.f;
        }
        vin_c[0] = vin_n[0];
        vin_c[1] = vin_n[1];
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) pr_c[e4] = pr_n[e4];
        // running merge inside the group: groups start at lanes that are multiples of s
        for (int d = 1; d < s; d <<= 1) {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float y = __shfl_up_sync(0xffffffffu, x[k], d);
            if (pos >= d) x[k] = __fadd_rn(x[k], y);
          }
        }
        if (valid) {
          uint4 o[2];
          o[0] = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                            pack_bf16x2(x[6], x[7]));
          o[1] = make_uint4(pack_bf16x2(x[8], x[9]), pack_bf16x2(x[10], x[11]), pack_bf16x2(x[12], x[13]),
                            pack_bf16x2(x[14], x[15]));
          uint4* dst = reinterpret_cast<uint4*>(p.cp + tok * D + ch0);
          dst[0] = o[0];
          dst[1] = o[1];
          if (closes && p.cache) {
            uint4* cdst = reinterpret_cast<uint4*>(p.cache + ((int64_t)b * p.n_groups + grp) * D + ch0);
            cdst[0] = o[0];
            cdst[1] = o[1];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
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

}  // namespace mtc

cudaError_t launch_merge_tc(const PrefillArgs& a, int B, const CUtensorMap& cmap, int sms, cudaStream_t st) {
  mtc::Params p;
  p.B = B;
  p.T = a.T;
  p.s = a.s;
  p.tpw = (mtc::WROWS / a.s) * a.s;
  const int64_t wblocks = cdiv(a.T, p.tpw);
  p.tiles_per_seq = (int)cdiv(wblocks, 4);
  p.n_tiles = B * p.tiles_per_seq;
  p.n_groups = cdiv(a.T, a.s);
  p.c = static_cast<const __nv_bfloat16*>(a.c);
  p.kR = static_cast<const __nv_bfloat16*>(a.kR);
  p.W_c = a.W_c;
  p.b_c = a.b_c;
  p.P = a.P;
  p.cp = static_cast<__nv_bfloat16*>(a.c_partial);
  p.cache = static_cast<__nv_bfloat16*>(a.cache_out);
  p.dev_err = a.dev_err;
  const size_t smem = mtc::smem_bytes();
  static uint64_t done_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(done_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(mtc::merge_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev < 64) done_mask |= 1ull << dev;
  }
  int pairs = sms / 2 > 0 ? sms / 2 : 1;
  if (p.n_tiles < pairs) pairs = p.n_tiles;
  mtc::merge_tc_kernel<<<2 * pairs, mtc::NT, smem, st>>>(cmap, p);
  return cudaGetLastError();
}

}  // namespace mtla
