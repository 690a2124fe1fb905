// Several new tokens per sequence in one decode call (speculative or beam
// decode): tokens t0 + 1 .. t0 + n of a sequence are merged in order, and the
// query of token i attends the cache as it stands after token i -- what n
// consecutive single-token decode steps would see (MTLA paper notes, "Key
// designs: hyper-network temporal merging": token t joins row ceil(t/s),
// opening it when (t-1) mod s == 0; abstract page, Figure 2(a): a query at a
// step that leaves its group open attends the temporary c_hat'_j).
//
// The merge kernel below runs one block per sequence.  It forms every token's
// gate pre-activation Linear(c_t) (W_c read once for all n tokens), then
// scans the tokens in order per channel: gate, gated entry, append or add,
// rounded to the cache dtype after every token exactly as a single-token step
// stores its row.  It writes the final rows to the cache, and for every token
// the tail row as it stood after it (`tails`).  The attention then runs once
// over B n "virtual" sequences (query i of sequence b is virtual sequence
// b n + i: same cache rows, t = t0 + i, its last row taken from tails), so
// the rows a sequence's queries share are streamed by neighbouring blocks of
// the same launch.
#include "kernels.cuh"

namespace mtla {
namespace {

// The four-part order of the tensor-core decode's merge kernel (four 64-row
// partial sums, added in order, then the bias) for (r, D) = (256, 288), so
// that n tokens merged here store exactly what n single-token steps store.
// Block = 2 D threads: thread (k, q2) forms the partial sums of quarters
// 2 q2 and 2 q2 + 1 of channel k for every token.
template <typename T, bool FOUR>
__global__ void __launch_bounds__(FOUR ? 576 : 256) multi_merge_kernel(const MultiMergeArgs p) {
  extern __shared__ float sm[];
  const int r = p.a.r, dR = p.a.d_R, D = r + dR, n = p.n, s = p.a.s;
  float* c_s = sm;              // [n][r] the tokens' latents
  float* part = c_s + n * r;    // [4][n][D] partial sums (four-part order)
  const int b = blockIdx.x, tid = threadIdx.x;
  const int64_t t0 = p.a.t_processed[b], off = p.a.seq_offset[b], cap = p.a.seq_capacity[b];
  const bool rows_ok = !(t0 < 0 || off < 0 || cap < 0 || off > p.a.cache_rows || cap > p.a.cache_rows - off);
  int err = 0;
  if (!rows_ok || group_of(t0 + n, s) > cap) err = MTLA_DEVERR_CAPACITY;
  else if (group_of(t0 + n, s) > p.m.J_max) err = MTLA_DEVERR_PE_RANGE;
  T* rows = reinterpret_cast<T*>(p.a.cache) + (rows_ok ? off : 0) * p.a.row_stride;
  T* tails = reinterpret_cast<T*>(p.tails) + (int64_t)b * n * D;

  if (err) {
    // nothing is merged: every query attends the cache as it stands
    if (tid == 0) {
      set_err(p.a.dev_err, err);
      for (int i = 0; i < n; ++i) {
        p.t_v[(int64_t)b * n + i] = (int32_t)t0;
        p.off_v[(int64_t)b * n + i] = off;
        p.cap_v[(int64_t)b * n + i] = cap;
      }
    }
    int64_t L0 = rows_ok && t0 > 0 ? group_of(t0, s) : 0;
    if (L0 > cap) L0 = cap;
    for (int i = tid; i < n * D; i += blockDim.x)
      st_elem(tails + i, L0 > 0 ? ld_f32(rows + (L0 - 1) * p.a.row_stride + i % D) : 0.f);
    return;
  }

  const T* cn = reinterpret_cast<const T*>(p.m.c_new) + (int64_t)b * n * r;
  for (int i = tid; i < n * r; i += blockDim.x) c_s[i] = ld_f32(cn + i);
  __syncthreads();
  constexpr int MAXN = MTLA_MAX_NEW_TOKENS;
  if constexpr (FOUR) {
    const int k = tid % D, q2 = tid / D;
#pragma unroll 1
    for (int qq = 0; qq < 2; ++qq) {
      const int quarter = 2 * q2 + qq, i0 = quarter * (r / 4);
      float acc[MAXN];
#pragma unroll
      for (int u = 0; u < MAXN; ++u) acc[u] = 0.f;
      for (int i = i0; i < i0 + r / 4; ++i) {
        const float w = __ldg(p.m.W_c + (int64_t)i * D + k);
#pragma unroll
        for (int u = 0; u < MAXN; ++u)
          if (u < n) acc[u] = fmaf(c_s[u * r + i], w, acc[u]);
      }
#pragma unroll
      for (int u = 0; u < MAXN; ++u)
        if (u < n) part[(quarter * n + u) * D + k] = acc[u];
    }
    __syncthreads();
    if (q2 != 0) return;
  }
  // one channel per thread from here: gate, gated entry, running row, in token order
  for (int k = tid; k < D; k += (FOUR ? D : blockDim.x)) {
    float g[MAXN];
    if constexpr (FOUR) {
#pragma unroll
      for (int u = 0; u < MAXN; ++u) {
        if (u >= n) break;
        float v = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) v += part[(q * n + u) * D + k];
        g[u] = v + __ldg(p.m.b_c + k);
      }
    } else {
      // the single-token SIMT merge's order: one chain in input order, then the bias
#pragma unroll
      for (int u = 0; u < MAXN; ++u) g[u] = 0.f;
      for (int i = 0; i < r; ++i) {
        const float w = p.m.W_c[(int64_t)i * D + k];
#pragma unroll
        for (int u = 0; u < MAXN; ++u)
          if (u < n) g[u] = fmaf(c_s[u * r + i], w, g[u]);
      }
#pragma unroll
      for (int u = 0; u < MAXN; ++u)
        if (u < n) g[u] = __fadd_rn(g[u], p.m.b_c[k]);
    }
    const T* kR = reinterpret_cast<const T*>(p.m.kR_new) + (int64_t)b * n * dR;
    // the row the first token joins, as the cache holds it (used only if the
    // token does not open it)
    const int64_t t1 = t0 + 1;
    float state = opens_row(t1, s) ? 0.f : ld_f32(rows + (group_of(t1, s) - 1) * p.a.row_stride + k);
#pragma unroll
    for (int u = 0; u < MAXN; ++u) {
      if (u >= n) break;
      const int64_t t = t0 + 1 + u, j = group_of(t, s);
      const float w = sigmoidf_(__fmul_rn(g[u], p.m.P[(j - 1) * D + k]));
      const float x = k < r ? c_s[u * r + k] : ld_f32(kR + (int64_t)u * dR + (k - r));
      const float e = __fmul_rn(w, x);
      const float v = round_to<T>(opens_row(t, s) ? e : __fadd_rn(state, e));
      state = v;
      st_elem(tails + (int64_t)u * D + k, v);
      if (t % s == 0 || u == n - 1) st_elem(rows + (j - 1) * p.a.row_stride + k, v);  // the row's last state
    }
  }
  if (tid == 0) {
    for (int i = 0; i < n; ++i) {
      p.t_v[(int64_t)b * n + i] = (int32_t)(t0 + 1 + i);
      p.off_v[(int64_t)b * n + i] = off;
      p.cap_v[(int64_t)b * n + i] = cap;
    }
    p.a.t_processed[b] = (int32_t)(t0 + n);
    if (p.a.cache_len) p.a.cache_len[b] = (int32_t)group_of(t0 + n, s);
  }
}

template <typename T, bool FOUR>
cudaError_t launch_multi_merge_t(const MultiMergeArgs& a, int B, cudaStream_t st) {
  const int D = a.a.r + a.a.d_R;
  const size_t smem = ((size_t)a.n * a.a.r + (FOUR ? (size_t)4 * a.n * D : 0)) * sizeof(float);
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(multi_merge_kernel<T, FOUR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  if (FOUR && 2 * D != 576) return cudaErrorInvalidValue;  // the four-part order is for D = 288
  multi_merge_kernel<T, FOUR><<<B, FOUR ? 2 * D : 256, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_multi_merge(const MultiMergeArgs& a, int B, int dtype, cudaStream_t st) {
  if (dtype == MTLA_BF16)
    return a.four_part ? launch_multi_merge_t<__nv_bfloat16, true>(a, B, st)
                       : launch_multi_merge_t<__nv_bfloat16, false>(a, B, st);
  return launch_multi_merge_t<float, false>(a, B, st);
}

}  // namespace mtla
