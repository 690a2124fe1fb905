// The layer's linear maps around the decode attention, with the key and value
// maps absorbed (MTLA paper notes, "Key designs: decoupled RoPE with temporal
// compression": Y = softmax((X W_Q W_K^T C_hat^T + Q^R K_hat^R^T)/sqrt(d_h))
// C_hat (W_V W_O); abstract page, Figure 1: the latent-to-KV maps are
// absorbed into the query and output layers by associativity).
//
//   in:  x_t [d] -> [ q_abs (H r) | q_rope (H d_R) | c_t (r) | k^R_t (d_R) ]
//        = x_t W_in^T, with RoPE at the token's position on the q_rope and
//        k^R parts.  W_in's rows are the per-head products W_Q^h W_K^h^T
//        (a d x r block per head, transposed), W_QR^h, W_down and W_KR.
//   out: y [d] = o_flat W_out^T, o_flat = [o_1 | ... | o_H] (H r), W_out's
//        row n holds (W_V^h W_O^h)[:, n] for every head.
//
// Both are one skinny GEMM D [B x N] = X [B x K] W^T [K x N] per call with a
// small batch B (one token per sequence), so they are bound by streaming W.
// Design (B200): the GEMM runs transposed on the 5th-generation tensor cores,
// D^T tile [128 rows of W x Bp] = W tile [128 x K] . X^T, so W fills the
// 128-lane M dimension and the batch (padded to a multiple of 16) is N.  A CTA
// takes one 128-row tile of W and a range of 64-wide K blocks (split-K, so that
// every SM streams a share of W): TMA loads the W tiles (128-byte swizzle),
// the threads stage X (bf16, or fp32 rounded to bf16) into the same K-major
// swizzled layout, one thread issues the MMAs into a TMEM accumulator, and the
// four warps read their 32 TMEM lanes back and store fp32 partial sums.  A
// second kernel, launched behind it with programmatic dependent launch, adds
// the K splits in a fixed order (deterministic) and writes the outputs: the
// input map also applies RoPE and splits the row into its four parts.
#include <math.h>

#include "kernels.cuh"

namespace mtla {
namespace prj {

constexpr int BM = 128;            // rows of W per tile (MMA M)
constexpr int BK = 64;             // K per block: 128-byte rows
constexpr int MAXKPB = 4;          // K blocks per CTA
constexpr int NT = 128;
constexpr int WTILE = BM * BK * 2;            // 16 KB
// Shared memory of a launch, sized to its K blocks per CTA and padded batch:
// kpb W tiles, kpb X tiles of Bp rows (each a multiple of 1024 bytes, the
// swizzle atom), then the barriers and the TMEM address.
struct Layout {
  size_t x, xtile, bar, tmem, total;
};
__host__ __device__ __forceinline__ Layout layout(int kpb, int Bp) {
  Layout l;
  l.xtile = ((size_t)Bp * BK * 2 + 1023) / 1024 * 1024;
  l.x = (size_t)kpb * WTILE;
  l.bar = l.x + (size_t)kpb * l.xtile;
  l.tmem = l.bar + (MAXKPB + 1) * 8;
  l.total = l.tmem + 16 + 1024;  // + slack to align the base to 1024
  return l;
}
static_assert(WTILE % 1024 == 0, "swizzle atoms must be 1024-aligned");
static_assert(MAXKPB * (WTILE + MAXBP * BK * 2) + 2048 <= 232448, "one block's shared memory (227 KB)");

size_t smem_bytes() { return layout(MAXKPB, MAXBP).total; }

// mbarrier wait by every lane of a warp with a warp-uniform result (the
// tcgen05.ld that follow are warp-collective)
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

template <typename TX>
__global__ void __launch_bounds__(NT, 1) proj_gemm_kernel(const __grid_constant__ CUtensorMap wmap, const GemmArgs p) {
  // blockIdx.x: 128-row tile of W; blockIdx.y: K split
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Layout L = layout(p.kpb, p.Bp);
  uint64_t* w_full = reinterpret_cast<uint64_t*>(sm + L.bar);
  uint64_t* mma_done = w_full + MAXKPB;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + L.tmem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * BM, ks = blockIdx.y;
  const int kb0 = ks * p.kpb;
  const int nkb = (kb0 + p.kpb <= p.nkb ? p.kpb : p.nkb - kb0);  // this split's K blocks (>= 1)
  const uint32_t ncols = p.Bp <= 32 ? 32u : (p.Bp <= 64 ? 64u : (p.Bp <= 128 ? 128u : 256u));

  if (tid == 0) {
    for (int i = 0; i < MAXKPB; ++i) mbar_init(&w_full[i], 1);
    mbar_init(mma_done, 1);
    fence_mbar_init();
    prefetch_tmap(&wmap);
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, ncols);
    tmem_relinquish();
  }
  // the activations (and the partial-sum buffer, which the previous call's
  // finishing kernel may still read) belong to earlier launches on the stream
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (tid == 0) {
    for (int i = 0; i < nkb; ++i) {
      mbar_arrive_expect_tx(&w_full[i], WTILE);
      tma_load_2d(sm + (size_t)i * WTILE, &wmap, (kb0 + i) * BK, m0, &w_full[i]);
    }
  }
  // X: row b of K block i -> eight 16-byte chunks, chunk c at b * 128 +
  // ((c ^ (b % 8)) * 16): the 128-byte swizzle of a K-major operand whose
  // 8-row groups are 1024 bytes apart
  for (int i = 0; i < nkb; ++i) {
    const uint32_t xbase = smem_u32(sm + L.x + (size_t)i * L.xtile);
    const int64_t k0 = (int64_t)(kb0 + i) * BK;
    for (int idx = tid; idx < p.Bp * 8; idx += NT) {
      const int b = idx >> 3, c = idx & 7;
      uint32_t w[4] = {0u, 0u, 0u, 0u};
      if (b < p.B) {
        const TX* src = reinterpret_cast<const TX*>(p.x) + (int64_t)b * p.ldx + k0 + c * 8;
        if constexpr (sizeof(TX) == 2) {
          const uint4 v = *reinterpret_cast<const uint4*>(src);
          w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
        } else {
          const float4 a = *reinterpret_cast<const float4*>(src);
          const float4 b4 = *reinterpret_cast<const float4*>(src + 4);
          w[0] = pack_bf16x2(a.x, a.y);
          w[1] = pack_bf16x2(a.z, a.w);
          w[2] = pack_bf16x2(b4.x, b4.y);
          w[3] = pack_bf16x2(b4.z, b4.w);
        }
      }
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(xbase + (uint32_t)(b * 128 + ((c ^ (b & 7)) << 4))),
                   "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
    }
  }
  fence_proxy_async_smem();  // the tensor core reads what the threads wrote
  __syncthreads();

  bool ok = true;
  if (warp == 0) {
    const uint32_t idesc = umma_idesc_bf16(BM, p.Bp, false, false);
    for (int i = 0; i < nkb && ok; ++i) {
      if (!warp_wait(&w_full[i], 0)) { ok = false; break; }
      tc_fence_after();
      if (elect_one()) {
        const uint32_t sW = smem_u32(sm + (size_t)i * WTILE);
        const uint32_t sX = smem_u32(sm + L.x + (size_t)i * L.xtile);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = umma_desc(sW + kk * 32, 16, 1024, 2);
          const uint64_t bd = umma_desc(sX + kk * 32, 16, 1024, 2);
          umma_bf16(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
      }
      __syncwarp();
    }
    if (elect_one()) umma_commit(mma_done);  // also when a wait gave up: the block must not wait forever
    __syncwarp();
  }
  if (!warp_wait(mma_done, 0)) ok = false;
  tc_fence_after();
  // warp w reads TMEM lanes 32 w .. 32 w + 31 = rows m0 + 32 w + lane of W
  const int m = m0 + 32 * warp + lane;
  float* dst = p.part + (size_t)ks * p.Bp * p.N;
  for (int c0 = 0; c0 < p.Bp; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0, v);
    tmem_wait_ld();
    if (m < p.N) {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (c0 + j < p.B) dst[(size_t)(c0 + j) * p.N + m] = __uint_as_float(v[j]);
    }
  }
  if (!ok && tid == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
  // drain: no copy may still be writing shared memory when the block exits
  if (tid == 0)
    for (int i = 0; i < nkb; ++i) mbar_wait(&w_full[i], 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

// Rotation of the channel pair (2k, 2k+1) of a d_R-wide RoPE vector at
// position pos by pos * 10000^(-2k/d_R) (the angle in double precision).
__device__ __forceinline__ void rope_pair(float& v0, float& v1, int32_t pos, int k, int d_R) {
  const double ang = (double)pos * pow(10000.0, -2.0 * (double)k / (double)d_R);
  double sn, cs;
  sincos(ang, &sn, &cs);
  const float c = (float)cs, s = (float)sn;
  const float a = v0, b = v1;
  v0 = a * c - b * s;
  v1 = a * s + b * c;
}

// Sum of the K splits of the input map for every (token, channel pair), then
// RoPE on the q_rope and k^R parts and the split into the four outputs.
template <typename TO>
__global__ void __launch_bounds__(256) proj_in_finish_kernel(const InFinishArgs p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int N = p.H * (p.r + p.d_R) + p.r + p.d_R;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)p.B * (N / 2)) return;
  const int b = (int)(idx / (N / 2)), n = 2 * (int)(idx % (N / 2));
  float v0 = 0.f, v1 = 0.f;
  for (int s = 0; s < p.KS; ++s) {
    const float* src = p.part + ((size_t)s * p.Bp + b) * N + n;
    v0 += src[0];
    v1 += src[1];
  }
  const int nq = p.H * p.r, nqr = nq + p.H * p.d_R, nc = nqr + p.r;
  TO* out;
  if (n < nq) {
    out = reinterpret_cast<TO*>(p.q_abs) + (size_t)b * nq + n;
  } else if (n < nqr) {
    const int j = n - nq;
    rope_pair(v0, v1, p.pos[b], (j % p.d_R) / 2, p.d_R);
    out = reinterpret_cast<TO*>(p.q_rope) + (size_t)b * (p.H * p.d_R) + j;
  } else if (n < nc) {
    out = reinterpret_cast<TO*>(p.c_new) + (size_t)b * p.r + (n - nqr);
  } else {
    const int j = n - nc;
    rope_pair(v0, v1, p.pos[b], j / 2, p.d_R);
    out = reinterpret_cast<TO*>(p.kR_new) + (size_t)b * p.d_R + j;
  }
  st_elem(out, v0);
  st_elem(out + 1, v1);
}

// Sum of the K splits of the output map: y [B, N] fp32.
__global__ void __launch_bounds__(256) proj_out_finish_kernel(const float* part, int KS, int Bp, int B, int N,
                                                                float* y) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)B * N) return;
  const int b = (int)(idx / N), n = (int)(idx % N);
  float v = 0.f;
  for (int s = 0; s < KS; ++s) v += part[((size_t)s * Bp + b) * N + n];
  y[idx] = v;
}

// fp32 layers (any size): one thread per output, the K products summed in
// order; the same finishing kernels then run with a single split.
__global__ void __launch_bounds__(256) proj_simt_kernel(const float* x, int64_t ldx, const float* W, int B, int K,
                                                          int N, float* part) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)B * N) return;
  const int b = (int)(idx / N), n = (int)(idx % N);
  const float* xr = x + (int64_t)b * ldx;
  const float* wr = W + (int64_t)n * K;
  float acc = 0.f;
  for (int k = 0; k < K; ++k) acc = fmaf(xr[k], wr[k], acc);
  part[(size_t)b * N + n] = acc;
}

}  // namespace prj

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
namespace {
cudaLaunchAttribute pdl_attr() {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}
}  // namespace

size_t proj_smem_bytes() { return prj::smem_bytes(); }

ProjSplit proj_split(int B, int K, int N, int sms) {
  ProjSplit s;
  s.Bp = ((B < MAXBP ? B : MAXBP) + 15) / 16 * 16;
  const int nkb = K / prj::BK;
  const int m_tiles = (N + prj::BM - 1) / prj::BM;
  int KS = (nkb + prj::MAXKPB - 1) / prj::MAXKPB;  // at most MAXKPB blocks per CTA
  while (KS < nkb && (int64_t)m_tiles * KS < sms) ++KS;
  s.kpb = (nkb + KS - 1) / KS;
  s.KS = (nkb + s.kpb - 1) / s.kpb;                 // no split is empty
  s.m_tiles = m_tiles;
  s.nkb = nkb;
  return s;
}

cudaError_t launch_proj_gemm(const GemmArgs& a, const CUtensorMap& wmap, int m_tiles, int KS, bool x_f32,
                             cudaStream_t st) {
  const size_t smem = prj::smem_bytes();
  static uint64_t done_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(done_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(prj::proj_gemm_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(prj::proj_gemm_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev < 64) done_mask |= 1ull << dev;
  }
  cudaLaunchAttribute attr[1] = {pdl_attr()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)m_tiles, (unsigned)KS);
  cfg.blockDim = dim3(prj::NT);
  cfg.dynamicSmemBytes = prj::layout(a.kpb, a.Bp).total;  // several CTAs per SM when the tiles are small
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return x_f32 ? cudaLaunchKernelEx(&cfg, prj::proj_gemm_kernel<float>, wmap, a)
               : cudaLaunchKernelEx(&cfg, prj::proj_gemm_kernel<__nv_bfloat16>, wmap, a);
}

cudaError_t launch_proj_simt(const float* x, int64_t ldx, const float* W, int B, int K, int N, float* part,
                             cudaStream_t st) {
  const int64_t n = (int64_t)B * N;
  prj::proj_simt_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(x, ldx, W, B, K, N, part);
  return cudaGetLastError();
}

cudaError_t launch_proj_in_finish(const InFinishArgs& a, int dtype, cudaStream_t st) {
  const int N = a.H * (a.r + a.d_R) + a.r + a.d_R;
  const int64_t n = (int64_t)a.B * (N / 2);
  cudaLaunchAttribute attr[1] = {pdl_attr()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((n + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return dtype == MTLA_BF16 ? cudaLaunchKernelEx(&cfg, prj::proj_in_finish_kernel<__nv_bfloat16>, a)
                            : cudaLaunchKernelEx(&cfg, prj::proj_in_finish_kernel<float>, a);
}

cudaError_t launch_proj_out_finish(const float* part, int KS, int Bp, int B, int N, float* y, cudaStream_t st) {
  const int64_t n = (int64_t)B * N;
  cudaLaunchAttribute attr[1] = {pdl_attr()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((n + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prj::proj_out_finish_kernel, part, KS, Bp, B, N, y);
}

// ---------------------------------------------------------------------------
// Per-head keys and values of a prompt for the un-absorbed forward:
// [K | V] [R x N] = C [R x Kd] . W^T, C the latent part of C_hat' (row stride
// ldc), W [N x Kd] = the rows of W_K^h^T then W_V^h^T per head.  One CTA per
// 128-row x 256-column tile, K <= 256 (four 64-wide blocks, all resident):
// A = C tile and B = W tile both by TMA (K-major, 128-byte swizzle), D in
// TMEM (256 columns); thread = row, bf16 stores of 32 consecutive columns.
// ---------------------------------------------------------------------------
namespace prj {
constexpr int RG_BN = 256;
constexpr int RG_MAXKB = 4;
constexpr int RG_ATILE = BM * BK * 2;     // 16 KB
constexpr int RG_BTILE = RG_BN * BK * 2;  // 32 KB
constexpr size_t RG_OFF_B = (size_t)RG_MAXKB * RG_ATILE;
constexpr size_t RG_OFF_BAR = RG_OFF_B + (size_t)RG_MAXKB * RG_BTILE;
constexpr size_t RG_OFF_TMEM = RG_OFF_BAR + (RG_MAXKB + 1) * 8;
constexpr size_t RG_SMEM = RG_OFF_TMEM + 16 + 1024;
static_assert(RG_SMEM <= 232448, "one block's shared memory (227 KB)");

__global__ void __launch_bounds__(NT, 1) rows_gemm_kernel(const __grid_constant__ CUtensorMap amap,
                                                          const __grid_constant__ CUtensorMap bmap, const RowsGemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + RG_OFF_BAR);
  uint64_t* mma_done = full + RG_MAXKB;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + RG_OFF_TMEM);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * BM, n0 = blockIdx.y * RG_BN;
  if (tid == 0) {
    for (int i = 0; i < RG_MAXKB; ++i) mbar_init(&full[i], 1);
    mbar_init(mma_done, 1);
    fence_mbar_init();
    prefetch_tmap(&amap);
    prefetch_tmap(&bmap);
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, RG_BN);
    tmem_relinquish();
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // C_hat' comes from the previous launch
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (tid == 0) {
    for (int i = 0; i < p.nkb; ++i) {
      mbar_arrive_expect_tx(&full[i], RG_ATILE + RG_BTILE);
      tma_load_2d(sm + (size_t)i * RG_ATILE, &amap, i * BK, m0, &full[i]);
      tma_load_2d(sm + RG_OFF_B + (size_t)i * RG_BTILE, &bmap, i * BK, n0, &full[i]);
      tma_load_2d(sm + RG_OFF_B + (size_t)i * RG_BTILE + RG_BTILE / 2, &bmap, i * BK, n0 + 128, &full[i]);
    }
  }
  bool ok = true;
  if (warp == 0) {
    constexpr uint32_t idesc = umma_idesc_bf16(BM, RG_BN, false, false);
    for (int i = 0; i < p.nkb && ok; ++i) {
      if (!warp_wait(&full[i], 0)) { ok = false; break; }
      tc_fence_after();
      if (elect_one()) {
        const uint32_t sA = smem_u32(sm + (size_t)i * RG_ATILE);
        const uint32_t sB = smem_u32(sm + RG_OFF_B + (size_t)i * RG_BTILE);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma_bf16(tmem, umma_desc(sA + kk * 32, 16, 1024, 2), umma_desc(sB + kk * 32, 16, 1024, 2), idesc,
                    (i > 0 || kk > 0) ? 1u : 0u);
      }
      __syncwarp();
    }
    if (elect_one()) umma_commit(mma_done);
    __syncwarp();
  }
  if (!warp_wait(mma_done, 0)) ok = false;
  tc_fence_after();
  const int64_t row = m0 + 32 * warp + lane;
  for (int c0 = 0; c0 < RG_BN; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0, v);
    tmem_wait_ld();
    if (row < p.R && n0 + c0 < p.N) {
      uint4 o[4];
      uint32_t* w = reinterpret_cast<uint32_t*>(o);
#pragma unroll
      for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
      // columns n0 + c0 .. + 31 of the row: keys below N / 2, values above
      const int n = n0 + c0;
      __nv_bfloat16* dst = n < p.N / 2 ? p.k + row * (int64_t)(p.N / 2) + n : p.v + row * (int64_t)(p.N / 2) + (n - p.N / 2);
      uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
      for (int j = 0; j < 4; ++j) d4[j] = o[j];
    }
  }
  if (!ok && tid == 0) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
  if (tid == 0)
    for (int i = 0; i < p.nkb; ++i) mbar_wait(&full[i], 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, RG_BN);
  }
}
}  // namespace prj

cudaError_t launch_rows_gemm(const RowsGemmArgs& a, const CUtensorMap& amap, const CUtensorMap& bmap,
                             cudaStream_t st) {
  static uint64_t done_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(done_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(prj::rows_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prj::RG_SMEM);
    if (e != cudaSuccess) return e;
    if (dev < 64) done_mask |= 1ull << dev;
  }
  cudaLaunchAttribute attr[1] = {pdl_attr()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((a.R + prj::BM - 1) / prj::BM), (unsigned)(a.N / prj::RG_BN));
  cfg.blockDim = dim3(prj::NT);
  cfg.dynamicSmemBytes = prj::RG_SMEM;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prj::rows_gemm_kernel, amap, bmap, a);
}

}  // namespace mtla
