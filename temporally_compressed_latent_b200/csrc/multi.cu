// Several new tokens per sequence in one decode call (speculative or beam
// decode): tokens t0 + 1 .. t0 + n of a sequence are merged in order, and the
// query of token i attends the cache as it stands after token i -- what n
// consecutive single-token decode steps would see (MTLA paper notes, "Key
// designs: hyper-network temporal merging": token t joins row ceil(t/s),
// opening it when (t-1) mod s == 0; abstract page, Figure 2(a): a query at a
// step that leaves its group open attends the temporary c_hat'_j).
//
// Two kernels merge the tokens: the gate pre-activations Linear(c_t) of all
// B n tokens in parallel, then one block per sequence scans its tokens in
// order per channel: gate, gated entry, append or add, rounded to the cache
// dtype after every token exactly as a single-token step stores its row.  The
// scan writes the final rows to the cache, and for every token the tail row
// as it stood after it (`tails`).  The attention then runs once
// over B n "virtual" sequences (query i of sequence b is virtual sequence
// b n + i: same cache rows, t = t0 + i, its last row taken from tails), so
// the rows a sequence's queries share are streamed by neighbouring blocks of
// the same launch.
#include "kernels.cuh"

namespace mtla {
namespace {

// Gate pre-activations Linear(c_t) = c_t W_c + b_c of all B n tokens, in the
// tensor-core decode step's order (r = 256, D = 288): a block is 32 channels
// x 2 tokens, 128 threads; warp w sums input rows 64 w .. 64 w + 63 in order
// (its W_c segments in flight at once), lanes are channels; the four partial
// sums are added in order, then the bias -- so that n tokens merged here store
// exactly what n single-token steps store.
__global__ void __launch_bounds__(128) multi_gate4_kernel(const MultiMergeArgs p, int ntok) {
  __shared__ float part[4][2][32];
  const int r = p.a.r, D = r + p.a.d_R;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = blockIdx.x % (D / 32), bt = blockIdx.x / (D / 32);
  const int k = kt * 32 + lane, u0 = bt * 2, i0 = w * 64;
  const __nv_bfloat16* cn = reinterpret_cast<const __nv_bfloat16*>(p.m.c_new);
  float acc[2] = {0.f, 0.f};
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int ib = i0 + 32 * half;
    float wv[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) wv[i] = __ldg(p.m.W_c + (size_t)(ib + i) * D + k);
    float cv[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) cv[u] = u0 + u < ntok ? __bfloat162float(cn[(size_t)(u0 + u) * r + ib + lane]) : 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i)
#pragma unroll
      for (int u = 0; u < 2; ++u) acc[u] = fmaf(__shfl_sync(0xffffffffu, cv[u], i), wv[i], acc[u]);
  }
#pragma unroll
  for (int u = 0; u < 2; ++u) part[w][u][lane] = acc[u];
  __syncthreads();
  if (w >= 2 || u0 + w >= ntok) return;
  float g = 0.f;
#pragma unroll
  for (int ww = 0; ww < 4; ++ww) g += part[ww][w][lane];
  p.gates[(size_t)(u0 + w) * D + k] = g + __ldg(p.m.b_c + k);
}

// The same pre-activations for any dims, in the single-token SIMT merge's
// order (one chain over the inputs in order, then the bias): one thread per
// (token, channel).
template <typename T>
__global__ void __launch_bounds__(256) multi_gate_kernel(const MultiMergeArgs p, int ntok) {
  const int r = p.a.r, D = r + p.a.d_R;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)ntok * D) return;
  const int64_t tok = idx / D;
  const int k = (int)(idx % D);
  const T* c = reinterpret_cast<const T*>(p.m.c_new) + tok * r;
  float g = 0.f;
  for (int i = 0; i < r; ++i) g = fmaf(ld_f32(c + i), p.m.W_c[(int64_t)i * D + k], g);
  p.gates[idx] = __fadd_rn(g, p.m.b_c[k]);
}

// One block per sequence, one thread per channel: the n tokens in order --
// gate, gated entry, append or add, rounded to the cache dtype after every
// token as a single-token step stores its row; the tail row after every token
// to `tails`, the rows' final states to the cache, and the per-query arrays.
template <typename T>
__global__ void multi_scan_kernel(const MultiMergeArgs p) {
  const int r = p.a.r, dR = p.a.d_R, D = r + dR, n = p.n, s = p.a.s;
  const int b = blockIdx.x, tid = threadIdx.x;
  const int64_t t0 = p.a.t_processed[b], off = p.a.seq_offset[b], cap = p.a.seq_capacity[b];
  const bool rows_ok = !(t0 < 0 || off < 0 || cap < 0 || off > p.a.cache_rows || cap > p.a.cache_rows - off);
  int err = 0;
  if (!rows_ok || group_of(t0 + n, s) > cap) err = MTLA_DEVERR_CAPACITY;
  else if (group_of(t0 + n, s) > p.m.J_max) err = MTLA_DEVERR_PE_RANGE;
  T* rows = reinterpret_cast<T*>(p.a.cache) + (rows_ok ? off : 0) * p.a.row_stride;
  T* tails = reinterpret_cast<T*>(p.tails) + (int64_t)b * n * D;
  if (tid == 0) {
    if (err) set_err(p.a.dev_err, err);
    for (int i = 0; i < n; ++i) {
      // with an error nothing is merged: every query attends the cache as it stands
      p.t_v[(int64_t)b * n + i] = (int32_t)(err ? t0 : t0 + 1 + i);
      p.off_v[(int64_t)b * n + i] = off;
      p.cap_v[(int64_t)b * n + i] = cap;
    }
    if (!err) {
      p.a.t_processed[b] = (int32_t)(t0 + n);
      if (p.a.cache_len) p.a.cache_len[b] = (int32_t)group_of(t0 + n, s);
    }
  }
  if (err) {
    int64_t L0 = rows_ok && t0 > 0 ? group_of(t0, s) : 0;
    if (L0 > cap) L0 = cap;
    for (int i = tid; i < n * D; i += blockDim.x)
      st_elem(tails + i, L0 > 0 ? ld_f32(rows + (L0 - 1) * p.a.row_stride + i % D) : 0.f);
    return;
  }
  const T* cn = reinterpret_cast<const T*>(p.m.c_new) + (int64_t)b * n * r;
  const T* kR = reinterpret_cast<const T*>(p.m.kR_new) + (int64_t)b * n * dR;
  const float* gates = p.gates + (int64_t)b * n * D;
  for (int k = tid; k < D; k += blockDim.x) {
    // the row the first token joins, as the cache holds it (used only if the
    // token does not open it)
    const int64_t t1 = t0 + 1;
    float state = opens_row(t1, s) ? 0.f : ld_f32(rows + (group_of(t1, s) - 1) * p.a.row_stride + k);
    for (int u = 0; u < n; ++u) {
      const int64_t t = t0 + 1 + u, j = group_of(t, s);
      const float w = sigmoidf_(__fmul_rn(gates[(int64_t)u * D + k], p.m.P[(j - 1) * D + k]));
      const float x = k < r ? ld_f32(cn + (int64_t)u * r + k) : ld_f32(kR + (int64_t)u * dR + (k - r));
      const float e = __fmul_rn(w, x);
      const float v = round_to<T>(opens_row(t, s) ? e : __fadd_rn(state, e));
      state = v;
      st_elem(tails + (int64_t)u * D + k, v);
      if (t % s == 0 || u == n - 1) st_elem(rows + (j - 1) * p.a.row_stride + k, v);  // the row's last state
    }
  }
}

template <typename T>
cudaError_t launch_multi_merge_t(const MultiMergeArgs& a, int B, cudaStream_t st) {
  const int D = a.a.r + a.a.d_R;
  const int ntok = B * a.n;
  if (a.four_part) {
    if (D != 288 || a.a.r != 256) return cudaErrorInvalidValue;  // the four-part order is for (r, D) = (256, 288)
    multi_gate4_kernel<<<(D / 32) * ((ntok + 1) / 2), 128, 0, st>>>(a, ntok);
  } else {
    const int64_t nthr = (int64_t)ntok * D;
    multi_gate_kernel<T><<<(unsigned)((nthr + 255) / 256), 256, 0, st>>>(a, ntok);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  multi_scan_kernel<T><<<B, (D + 31) / 32 * 32, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_multi_merge(const MultiMergeArgs& a, int B, int dtype, cudaStream_t st) {
  return dtype == MTLA_BF16 ? launch_multi_merge_t<__nv_bfloat16>(a, B, st) : launch_multi_merge_t<float>(a, B, st);
}

}  // namespace mtla
