// The contractions and the gate arithmetic of the training backward pass
// (MTLA paper notes, "Key designs: hyper-network temporal merging" and
// "decoupled RoPE with temporal compression", training shortcut):
//
// - gemm_bt: C[M, N] = A[M, K] B[N, K]^T on the tensor cores (tcgen05, TMEM
//   accumulator, a four-stage TMA ring of 128 x 64 A and 256 x 64 B tiles),
//   fp32 out, optionally accumulated into C or split over K; each operand
//   K-major or MN-major (as stored, no transposed copies).  It carries
//     dC_hat' = [dk | dv] W_kv (K = 2 H d_h),  G = c W_c (the gate
//     pre-activations, recomputed), dc += dg W_c^T and dW_c = c^T dg;
// - merge_bwd: per group and latent channel, the reverse scan over the
//   group's tokens and the gate's chain rule (de, w, dz, dg, dP, the direct
//   dc = de w), in a fixed order;
// - small helpers: the conversion of W_c to a bf16 operand, slice sums.
#include "kernels.cuh"

namespace mtla {
namespace tgm {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4, NT = 128;
constexpr uint32_t ATILE = BM * BK * 2;  // 16 KB
constexpr uint32_t BTILE = BN * BK * 2;  // 32 KB
constexpr uint32_t STAGE = ATILE + BTILE;
constexpr size_t OFF_BAR = (size_t)STAGES * STAGE;
constexpr size_t SMEM = OFF_BAR + 128 + 1024;  // barriers + TMEM holder, and the 1 KB alignment slack

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

__global__ void __launch_bounds__(NT, 1) gemm_bt_kernel(const __grid_constant__ CUtensorMap amap0,
                                                        const __grid_constant__ CUtensorMap amap1,
                                                        const __grid_constant__ CUtensorMap bmap, const GemmBtArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* done = empty + STAGES;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = (int64_t)blockIdx.x * BM;
  const int n0 = blockIdx.y * BN;
  const int nkb_all = (p.K + BK - 1) / BK;
  const int kb0 = blockIdx.z * p.kb_per_split;
  const int kb1 = kb0 + p.kb_per_split < nkb_all ? kb0 + p.kb_per_split : nkb_all;
  const int nk = kb1 > kb0 ? kb1 - kb0 : 0;
  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
    prefetch_tmap(&amap0);
    prefetch_tmap(&amap1);
    prefetch_tmap(&bmap);
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  bool ok = true;
  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {  // producer: one TMA lane
      for (int i = 0; i < nk; ++i) {
        const int st = i % STAGES;
        if (i >= STAGES && !mbar_wait(&empty[st], ((i / STAGES) - 1) & 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[st], STAGE);
        const int kc = (kb0 + i) * BK;
        uint8_t* a = sm + (size_t)st * STAGE;
        if (p.a_mn) {
          // [64 K rows x 64 M] boxes, two along M
          tma_load_2d(a, &amap0, (int32_t)m0, kc, &full[st]);
          tma_load_2d(a + ATILE / 2, &amap0, (int32_t)m0 + 64, kc, &full[st]);
        } else if (kc < p.ka_split) {
          tma_load_2d(a, &amap0, kc, (int32_t)m0, &full[st]);
        } else {
          tma_load_2d(a, &amap1, kc - p.ka_split, (int32_t)m0, &full[st]);
        }
        if (p.b_mn) {
#pragma unroll
          for (int u = 0; u < 4; ++u) tma_load_2d(a + ATILE + u * (BTILE / 4), &bmap, n0 + 64 * u, kc, &full[st]);
        } else {
          tma_load_2d(a + ATILE, &bmap, kc, n0, &full[st]);
          tma_load_2d(a + ATILE + BTILE / 2, &bmap, kc, n0 + 128, &full[st]);
        }
        issued = i + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {  // MMA issue: one elected lane
    const uint32_t idesc = umma_idesc_bf16(BM, BN, p.a_mn != 0, p.b_mn != 0);
    for (int i = 0; i < nk; ++i) {
      const int st = i % STAGES;
      if (!warp_wait(&full[st], (i / STAGES) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
        const uint32_t sA = smem_u32(sm + (size_t)st * STAGE), sB = sA + ATILE;
        // K-major: a K step of 16 is 32 bytes along each 128-byte row.
        // MN-major (128-byte swizzle): 64-element chunks along M / N are 8 KB
        // apart (one box each), 8-row groups along K 1 KB apart, and a K step
        // of 16 is 16 rows = 2 KB.
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = p.a_mn ? umma_desc(sA + kk * 2048, ATILE / 2, 1024, 2) : umma_desc(sA + kk * 32, 16, 1024, 2);
          const uint64_t bd = p.b_mn ? umma_desc(sB + kk * 2048, BTILE / 4, 1024, 2) : umma_desc(sB + kk * 32, 16, 1024, 2);
          umma_bf16(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&empty[st]);  // the stage is free once these MMAs have read it
      }
      __syncwarp();
    }
    if (elect_one()) umma_commit(done);
    __syncwarp();
  }
  if (nk > 0 && !mbar_wait(done, 0)) ok = false;
  tc_fence_after();
  // epilogue: warp w owns TMEM lanes (rows) 32 w .. 32 w + 31
  const int64_t row = m0 + 32 * warp + lane;
  float* crow = p.C + (int64_t)blockIdx.z * p.split_stride + row * p.ldc + n0;
  for (int c0 = 0; c0 < BN; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0, v);
    tmem_wait_ld();
    if (row < p.M && n0 + c0 < p.N) {
      float4* d4 = reinterpret_cast<float4*>(crow + c0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 x = nk > 0 ? make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                        __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
        if (p.accumulate) {
          const float4 o = d4[j];
          x.x += o.x;
          x.y += o.y;
          x.z += o.z;
          x.w += o.w;
        }
        d4[j] = x;
      }
    }
  }
  if (!ok) set_err(p.dev_err, MTLA_DEVERR_TIMEOUT);
  if (tid == 0)  // no TMA write may land after the block has left
    for (int i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

// out[r * ld_out + c] = sum_z src[z * stride + r * cols + c] for c < cols, zero for cols <= c < ld_out.
// Slice z goes to partial sum z % 8 and the eight are added in a fixed tree,
// so eight loads are in flight per thread and the result does not depend on
// scheduling.
__global__ void __launch_bounds__(256) sum_slices_kernel(const float* src, int64_t rows, int cols, int64_t ld_out,
                                                         int n, int64_t stride, float* out) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * ld_out) return;
  const int64_t r = idx / ld_out;
  const int c = (int)(idx % ld_out);
  float acc = 0.f;
  if (c < cols) {
    const float* q = src + r * cols + c;
    float a[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) a[u] = 0.f;
    int z = 0;
    for (; z + 8 <= n; z += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldg(q + (int64_t)(z + u) * stride);
#pragma unroll
      for (int u = 0; u < 8; ++u) a[u] += v[u];
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (z + u < n) a[u] += __ldg(q + (int64_t)(z + u) * stride);
    acc = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
  }
  out[idx] = acc;
}

__global__ void __launch_bounds__(256) convert_kernel(const float* in, int64_t rows, int cols, int64_t ld_in,
                                                      __nv_bfloat16* out, int64_t ld_out) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * cols) return;
  const int64_t r = idx / cols;
  const int c = (int)(idx % cols);
  out[r * ld_out + c] = __float2bfloat16_rn(in[r * ld_in + c]);
}

// One thread per (group j, channel k) of the J_max x D table dP: the group's
// tokens of every sequence, last to first.  For channels k < r and groups
// that hold tokens:
//   de = running sum of dC over the group's later positions (C_hat'_n sums
//        the gated entries of its group up to n),
//   g = G + b_c, u = P[j], w = Sigmoid(g u),
//   dz = de c w (1 - w), dg = dz u, dP[j] += dz g, dc = de w (direct term).
// Other entries of dP are zero (the RoPE gate channels do not reach the
// latent merge; groups past the sequence hold no token).
__global__ void __launch_bounds__(256) merge_bwd_kernel(const MergeBwdArgs p) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)p.J_max * p.D) return;
  const int j = (int)(idx / p.D), k = (int)(idx % p.D);
  const int J = (p.T + p.s - 1) / p.s;
  if (k >= p.r || j >= J) {
    p.dP[idx] = 0.f;
    return;
  }
  const float u = p.P[idx], bc = p.b_c[k];
  const int i0 = j * p.s, i1 = i0 + p.s < p.T ? i0 + p.s : p.T;  // 0-based tokens i0 .. i1 - 1
  float dP = 0.f, db = 0.f;
  // four sequences at a time: their loads are independent, so they are in
  // flight together; dP and db are summed in a fixed order (blocks of four
  // sequences, tokens last to first, sequences within a block)
  for (int b0 = 0; b0 < p.B; b0 += 4) {
    const int nb = p.B - b0 < 4 ? p.B - b0 : 4;
    float de[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = i1 - 1; i >= i0; --i) {
      float dCv[4], gv[4], cv[4];
#pragma unroll
      for (int u4 = 0; u4 < 4; ++u4) {
        const int64_t e = ((int64_t)(b0 + (u4 < nb ? u4 : 0)) * p.T + i) * p.r + k;
        dCv[u4] = p.dC[e];
        gv[u4] = p.G[e];
        cv[u4] = __bfloat162float(p.c[e]);
      }
#pragma unroll
      for (int u4 = 0; u4 < 4; ++u4) {
        if (u4 >= nb) break;
        const int64_t e = ((int64_t)(b0 + u4) * p.T + i) * p.r + k;
        de[u4] += dCv[u4];
        const float g = gv[u4] + bc;
        const float w = sigmoidf_(g * u);
        const float dz = de[u4] * cv[u4] * w * (1.f - w);
        const float dg = dz * u;
        dP += dz * g;
        db += dg;
        p.dc[e] = de[u4] * w;
        p.dg[e] = __float2bfloat16_rn(dg);
      }
    }
  }
  p.dP[idx] = dP;
  p.db_part[(int64_t)j * p.r + k] = db;
}

// First pass of db[k] = sum_j part[j][k] in a fixed order: block (x, z) sums
// channels 32 x .. 32 x + 31 over groups j = z, z + DB_SLICES, ... (8 lanes of
// j, then the lanes in order) into out[z][k]; the slices are summed after.
constexpr int DB_SLICES = 64;
__global__ void __launch_bounds__(256) db_partial_kernel(const float* part, int J, int r, float* out) {
  __shared__ float red[8][33];
  const int kx = threadIdx.x & 31, jl = threadIdx.x >> 5;
  const int k = blockIdx.x * 32 + kx, z = blockIdx.y;
  float acc = 0.f;
  if (k < r)
    for (int j = z + jl * DB_SLICES; j < J; j += 8 * DB_SLICES) acc += part[(int64_t)j * r + k];
  red[jl][kx] = acc;
  __syncthreads();
  if (jl == 0 && k < r) {
    float t = 0.f;
    for (int i = 0; i < 8; ++i) t += red[i][kx];
    out[(int64_t)z * r + k] = t;
  }
}

}  // namespace tgm

size_t gemm_bt_smem_bytes() { return tgm::SMEM; }

cudaError_t launch_gemm_bt(const GemmBtArgs& a, const CUtensorMap& amap0, const CUtensorMap& amap1,
                           const CUtensorMap& bmap, int splits, cudaStream_t st) {
  static uint64_t done_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(done_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(tgm::gemm_bt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tgm::SMEM);
    if (e != cudaSuccess) return e;
    if (dev < 64) done_mask |= 1ull << dev;
  }
  const dim3 grid((unsigned)((a.M + tgm::BM - 1) / tgm::BM), (unsigned)(a.N / tgm::BN), (unsigned)splits);
  tgm::gemm_bt_kernel<<<grid, tgm::NT, tgm::SMEM, st>>>(amap0, amap1, bmap, a);
  return cudaGetLastError();
}

cudaError_t launch_sum_slices(const float* src, int64_t rows, int cols, int64_t ld_out, int n, int64_t stride,
                              float* out, cudaStream_t st) {
  const int64_t nth = rows * ld_out;
  tgm::sum_slices_kernel<<<(unsigned)((nth + 255) / 256), 256, 0, st>>>(src, rows, cols, ld_out, n, stride, out);
  return cudaGetLastError();
}

cudaError_t launch_convert_bf16(const float* in, int64_t rows, int cols, int64_t ld_in, __nv_bfloat16* out,
                                int64_t ld_out, cudaStream_t st) {
  const int64_t nth = rows * cols;
  tgm::convert_kernel<<<(unsigned)((nth + 255) / 256), 256, 0, st>>>(in, rows, cols, ld_in, out, ld_out);
  return cudaGetLastError();
}

cudaError_t launch_merge_bwd(const MergeBwdArgs& a, cudaStream_t st) {
  const int64_t nth = (int64_t)a.J_max * a.D;
  tgm::merge_bwd_kernel<<<(unsigned)((nth + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_db_reduce(const float* part, int J, int r, int D, float* slices, float* db, cudaStream_t st) {
  tgm::db_partial_kernel<<<dim3((unsigned)((r + 31) / 32), tgm::DB_SLICES), 256, 0, st>>>(part, J, r, slices);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_sum_slices(slices, 1, r, D, tgm::DB_SLICES, r, db, st);
}

}  // namespace mtla
