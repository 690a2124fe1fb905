// Generic SIMT kernels of the MTLA library: any supported (H, r, d_R), fp32 or
// bf16 storage, fp32 arithmetic (expf / sigmoid without fast-math).
//
//   merge_append_kernel   one block per sequence: gate GEMV, append / in-place
//                         update of the tail row (MTLA paper notes, "Key
//                         designs: hyper-network temporal merging").
//   decode_simt_kernel    one block per sequence: optional fused merge, then
//                         absorbed attention over the ceil(t/s) rows with an
//                         online softmax ("Key designs: decoupled RoPE with
//                         temporal compression"; Figure 2(a)).
//   partial_merge_kernel  running merge C_hat' of whole groups of tokens
//                         ("Key designs: stride-aware causal mask"; Fig. 2(c)).
//   prefill_simt_kernel   stride-aware masked attention, one warp per head.
#include "kernels.cuh"

namespace mtla {

// ----------------------------------------------------------------------------
// block reductions (blockDim.x multiple of 32, <= 1024)
// ----------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float r = -INFINITY;
  for (int i = 0; i < nw; ++i) r = fmaxf(r, red[i]);
  return r;
}
__device__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float r = 0.f;
  for (int i = 0; i < nw; ++i) r += red[i];
  return r;
}

// ----------------------------------------------------------------------------
// per-sequence bookkeeping shared by the merge and the SIMT decode
// ----------------------------------------------------------------------------
struct SeqState {
  int64_t t;      // tokens processed after this call's merge
  int64_t L;      // rows the attention reads
  int64_t off;    // first row of the sequence in the cache buffer
  bool merge_ok;  // the merge may write its row
};

__device__ SeqState seq_state(const SeqArgs& a, int b, bool with_merge, int32_t J_max, bool report) {
  SeqState st;
  const int64_t t0 = a.t_processed[b];
  const int64_t cap = a.seq_capacity[b];
  st.t = t0 + (with_merge ? 1 : 0);
  st.off = a.seq_offset[b];
  st.merge_ok = with_merge;
  int64_t L = st.t > 0 ? group_of(st.t, a.s) : 0;
  if (t0 < 0 || st.off < 0 || cap < 0 || st.off > a.cache_rows || cap > a.cache_rows - st.off) {
    // the sequence's rows are not inside the buffer: touch nothing
    if (report) set_err(a.dev_err, MTLA_DEVERR_CAPACITY);
    L = 0;
    st.off = 0;
    st.merge_ok = false;
  } else if (L > cap) {
    if (report) set_err(a.dev_err, MTLA_DEVERR_CAPACITY);
    L = cap;
    st.merge_ok = false;
  }
  if (st.merge_ok && group_of(st.t, a.s) > J_max) {
    if (report) set_err(a.dev_err, MTLA_DEVERR_PE_RANGE);
    st.merge_ok = false;
  }
  st.L = L;
  return st;
}

// Gate and row update of one sequence's new token; all threads of the block.
// c_sm holds c_t in fp32 (r values).
template <typename T>
__device__ void merge_row(const SeqArgs& a, const MergeArgsDev& m, int b, const SeqState& st,
                          const float* c_sm) {
  const int r = a.r, D = a.r + a.d_R;
  const int64_t j = group_of(st.t, a.s);
  const bool opens = opens_row(st.t, a.s);
  T* row = reinterpret_cast<T*>(a.cache) + (st.off + j - 1) * a.row_stride;
  const T* kR = reinterpret_cast<const T*>(m.kR_new) + (int64_t)b * a.d_R;
  const float* Pj = m.P + (j - 1) * D;
  for (int k = threadIdx.x; k < D; k += blockDim.x) {
    // Linear(c_t): the products are summed in input order from zero and the
    // bias added last, the same order every kernel of this library uses.
    float g = 0.f;
    for (int i = 0; i < r; ++i) g = fmaf(c_sm[i], m.W_c[(int64_t)i * D + k], g);
    g = __fadd_rn(g, m.b_c[k]);
    const float w = sigmoidf_(__fmul_rn(g, Pj[k]));
    const float x = k < r ? c_sm[k] : ld_f32(kR + (k - r));
    const float e = __fmul_rn(w, x);  // no contraction: every kernel rounds the same way
    const float v = opens ? e : __fadd_rn(ld_f32(row + k), e);
    st_elem(row + k, v);
  }
}

template <typename T>
__global__ void merge_append_kernel(SeqArgs a, MergeArgsDev m) {
  extern __shared__ float sm[];
  float* c_sm = sm;
  const int b = blockIdx.x;
  const SeqState st = seq_state(a, b, true, m.J_max, threadIdx.x == 0);
  const T* c = reinterpret_cast<const T*>(m.c_new) + (int64_t)b * a.r;
  for (int i = threadIdx.x; i < a.r; i += blockDim.x) c_sm[i] = ld_f32(c + i);
  __syncthreads();
  if (st.merge_ok) merge_row<T>(a, m, b, st, c_sm);
  if (threadIdx.x == 0 && st.merge_ok) {
    a.t_processed[b] = (int32_t)st.t;
    if (a.cache_len) a.cache_len[b] = (int32_t)st.L;
  }
}

// ----------------------------------------------------------------------------
// decode: one block per sequence
// ----------------------------------------------------------------------------
constexpr int kSimtThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kSimtThreads) decode_simt_kernel(SeqArgs a, MergeArgsDev m, bool with_merge,
                                                                   DecodeOut o) {
  extern __shared__ float sm[];
  const int H = o.H, r = a.r, D = a.r + a.d_R;
  float* c_sm = sm;               // [r]
  float* q_sm = c_sm + r;         // [H][D]
  float* p_sm = q_sm + H * D;     // [kSimtThreads]
  float* red = p_sm + kSimtThreads;  // [32]
  const int b = blockIdx.x, tid = threadIdx.x;

  const SeqState st = seq_state(a, b, with_merge, with_merge ? m.J_max : 0, tid == 0);
  if (with_merge) {
    const T* c = reinterpret_cast<const T*>(m.c_new) + (int64_t)b * r;
    for (int i = tid; i < r; i += blockDim.x) c_sm[i] = ld_f32(c + i);
    __syncthreads();
    if (st.merge_ok) merge_row<T>(a, m, b, st, c_sm);
    __syncthreads();  // the new row is read below by other threads of the block
  }
  if (tid == 0) {
    if (with_merge && st.merge_ok) a.t_processed[b] = (int32_t)st.t;
    if (a.cache_len) a.cache_len[b] = (int32_t)st.L;
  }
  const T* qa = reinterpret_cast<const T*>(o.q_abs) + (int64_t)b * H * r;
  const T* qr = reinterpret_cast<const T*>(o.q_rope) + (int64_t)b * H * a.d_R;
  for (int i = tid; i < H * D; i += blockDim.x) {
    const int h = i / D, k = i % D;
    q_sm[i] = k < r ? ld_f32(qa + h * r + k) : ld_f32(qr + h * a.d_R + (k - r));
  }
  __syncthreads();

  const int64_t L = st.L;
  const T* rows = reinterpret_cast<const T*>(a.cache) + st.off * a.row_stride;
  // several tokens per call: the last row as it stood after this query's token
  const T* last = o.tails ? reinterpret_cast<const T*>(o.tails) + (int64_t)b * D : rows + (L - 1) * a.row_stride;
  auto row_of = [&](int64_t j) { return j == L - 1 ? last : rows + j * a.row_stride; };
  if (L == 0) {
    if (tid == 0) set_err(a.dev_err, MTLA_DEVERR_EMPTY);
    for (int i = tid; i < H * r; i += blockDim.x) o.out[(int64_t)b * H * r + i] = 0.f;
    if (o.lse && tid < H) o.lse[(int64_t)b * H + tid] = -INFINITY;
    return;
  }
  constexpr int kMaxPer = 2;  // r <= 512
  for (int h = 0; h < H; ++h) {
    float mx = -INFINITY, l = 0.f, acc[kMaxPer] = {0.f, 0.f};
    const float* q = q_sm + h * D;
    for (int64_t base = 0; base < L; base += kSimtThreads) {
      const int64_t j = base + tid;
      float sc = -INFINITY;
      if (j < L) {
        const T* row = row_of(j);
        float dot = 0.f;
        for (int k = 0; k < D; ++k) dot = fmaf(q[k], ld_f32(row + k), dot);
        sc = dot * o.scale;
      }
      const float cmax = block_max(sc, red);
      const float mnew = fmaxf(mx, cmax);
      const float alpha = expf(mx - mnew);
      const float pj = j < L ? expf(sc - mnew) : 0.f;
      p_sm[tid] = pj;
      const float csum = block_sum(pj, red);
      l = l * alpha + csum;
      const int nrows = (int)(L - base < kSimtThreads ? L - base : kSimtThreads);
#pragma unroll
      for (int c = 0; c < kMaxPer; ++c) {
        const int k = tid + c * kSimtThreads;
        if (k < r) {
          float v = acc[c] * alpha;
          for (int jj = 0; jj < nrows; ++jj) v = fmaf(p_sm[jj], ld_f32(row_of(base + jj) + k), v);
          acc[c] = v;
        }
      }
      mx = mnew;
      __syncthreads();
    }
#pragma unroll
    for (int c = 0; c < kMaxPer; ++c) {
      const int k = tid + c * kSimtThreads;
      if (k < r) o.out[((int64_t)b * H + h) * r + k] = acc[c] / l;
    }
    if (o.lse && tid == 0) o.lse[(int64_t)b * H + h] = mx + logf(l);
  }
}

// ----------------------------------------------------------------------------
// prefill step 1: running merge C_hat' over whole groups (gate GEMM + scan)
// ----------------------------------------------------------------------------
// Block = 256 threads as 16 x 16; a chunk of TC = 16*TPT tokens times 16*CPT
// channels is computed per pass with W_c streamed through shared memory in
// slabs of 32 input rows.  The scan then runs over the chunk's tokens in
// order, carrying each group's running merge in fp32 and rounding only the
// values it stores (a decode step, whose tail row lives in the cache, rounds
// the stored row after every token instead).
template <typename T, int TPT, int CPT>
__global__ void __launch_bounds__(256) partial_merge_kernel(PrefillArgs p) {
  constexpr int TC = 16 * TPT;
  constexpr int KS = 32;
  extern __shared__ float sm[];
  const int r = p.r, d_R = p.d_R, D = r + d_R, s = p.s;
  float* w_sm = sm;                    // [KS][D]
  float* c_sm = w_sm + KS * D;         // [TC][KS]
  float* e_sm = c_sm + TC * KS;        // [TC][D]  gated entries w*x of the chunk
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int b = blockIdx.y;
  const int64_t Tn = p.T;
  const int64_t n_groups = cdiv(Tn, s);
  const int64_t gpb = p.groups_per_block;
  const int64_t g0 = (int64_t)blockIdx.x * gpb;
  if (g0 >= n_groups) return;
  const int64_t g1 = g0 + gpb < n_groups ? g0 + gpb : n_groups;
  const int64_t n_begin = g0 * s, n_end = (g1 * s < Tn) ? g1 * s : Tn;  // 0-based token range

  const T* cin = reinterpret_cast<const T*>(p.c) + (int64_t)b * Tn * r;
  const T* kin = reinterpret_cast<const T*>(p.kR) + (int64_t)b * Tn * d_R;
  T* cp = reinterpret_cast<T*>(p.c_partial) + (int64_t)b * Tn * D;
  T* cache = reinterpret_cast<T*>(p.cache_out);
  const int64_t Lc = n_groups;

  constexpr int kPer = 3;  // channels per thread in the scan (D <= 768)
  float run[kPer] = {0.f, 0.f, 0.f};

  for (int64_t n0 = n_begin; n0 < n_end; n0 += TC) {
    const int tc = (int)(n_end - n0 < TC ? n_end - n0 : TC);
    float acc[TPT][CPT];
#pragma unroll
    for (int i = 0; i < TPT; ++i)
#pragma unroll
      for (int c = 0; c < CPT; ++c) acc[i][c] = 0.f;
    for (int k0 = 0; k0 < r; k0 += KS) {
      const int ks = r - k0 < KS ? r - k0 : KS;
      __syncthreads();
      for (int i = tid; i < KS * D; i += 256) {
        const int kk = i / D, ch = i % D;
        w_sm[i] = kk < ks ? p.W_c[(int64_t)(k0 + kk) * D + ch] : 0.f;
      }
      for (int i = tid; i < TC * KS; i += 256) {
        const int tt = i / KS, kk = i % KS;
        c_sm[i] = (tt < tc && kk < ks) ? ld_f32(cin + (n0 + tt) * r + k0 + kk) : 0.f;
      }
      __syncthreads();
      for (int kk = 0; kk < ks; ++kk) {
        float cv[TPT];
#pragma unroll
        for (int i = 0; i < TPT; ++i) cv[i] = c_sm[(ty * TPT + i) * KS + kk];
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
          const int ch = tx + 16 * c;
          const float wv = ch < D ? w_sm[kk * D + ch] : 0.f;
#pragma unroll
          for (int i = 0; i < TPT; ++i) acc[i][c] = fmaf(cv[i], wv, acc[i][c]);
        }
      }
    }
    __syncthreads();
    // gate and gated entry of every (token, channel) of the chunk
#pragma unroll
    for (int i = 0; i < TPT; ++i) {
      const int tt = ty * TPT + i;
      if (tt >= tc) continue;
      const int64_t n1 = n0 + tt + 1;  // 1-based token index
      const float* Pj = p.P + (group_of(n1, s) - 1) * D;
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const int ch = tx + 16 * c;
        if (ch >= D) continue;
        const float g = __fadd_rn(acc[i][c], p.b_c[ch]);
        const float w = sigmoidf_(__fmul_rn(g, Pj[ch]));
        const float x = ch < r ? ld_f32(cin + (n1 - 1) * r + ch) : ld_f32(kin + (n1 - 1) * d_R + (ch - r));
        e_sm[tt * D + ch] = __fmul_rn(w, x);
      }
    }
    __syncthreads();
    // scan over the chunk's tokens in order
#pragma unroll
    for (int c = 0; c < kPer; ++c) {
      const int ch = tid + 256 * c;
      if (ch >= D) continue;
      float v = run[c];
      for (int tt = 0; tt < tc; ++tt) {
        const int64_t n1 = n0 + tt + 1;
        const float e = e_sm[tt * D + ch];
        v = opens_row(n1, s) ? e : __fadd_rn(v, e);
        st_elem(cp + (n1 - 1) * D + ch, v);
        if (cache && (n1 % s == 0 || n1 == Tn)) {
          const int64_t g = group_of(n1, s);
          st_elem(cache + ((int64_t)b * Lc + g - 1) * D + ch, v);
        }
      }
      run[c] = v;
    }
  }
}

// ----------------------------------------------------------------------------
// prefill step 2 (SIMT): masked attention, one block per (b, m), warp per head
// ----------------------------------------------------------------------------
template <typename T>
__global__ void prefill_simt_kernel(PrefillArgs p) {
  const int H = p.H, r = p.r, d_R = p.d_R, D = r + d_R, s = p.s;
  const int lane = threadIdx.x & 31, h = threadIdx.x >> 5;
  const int64_t Tn = p.T;
  const int64_t bm = blockIdx.x;
  const int64_t b = bm / Tn, m = bm % Tn + 1;  // 1-based query
  if (h >= H) return;
  constexpr int kQ = 18;   // D <= 576
  constexpr int kO = 16;   // r <= 512
  const T* qa = reinterpret_cast<const T*>(p.q_abs) + ((b * Tn + (m - 1)) * H + h) * r;
  const T* qr = reinterpret_cast<const T*>(p.q_rope) + ((b * Tn + (m - 1)) * H + h) * d_R;
  float q[kQ];
#pragma unroll
  for (int i = 0; i < kQ; ++i) {
    const int k = lane + 32 * i;
    q[i] = k < r ? ld_f32(qa + k) : (k < D ? ld_f32(qr + (k - r)) : 0.f);
  }
  const T* cp = reinterpret_cast<const T*>(p.c_partial) + b * Tn * D;
  float mx = -INFINITY, l = 0.f, acc[kO];
#pragma unroll
  for (int i = 0; i < kO; ++i) acc[i] = 0.f;
  const int64_t jm = group_of(m, s);
  // visible columns: n = g*s for g = 1..j(m)-1, then n = m itself
  for (int64_t g = 1; g <= jm; ++g) {
    const int64_t n = g < jm ? g * s : m;
    const T* row = cp + (n - 1) * D;
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < kQ; ++i) {
      const int k = lane + 32 * i;
      if (k < D) dot = fmaf(q[i], ld_f32(row + k), dot);
    }
    dot = warp_sum(dot) * p.scale;
    const float mnew = fmaxf(mx, dot);
    const float alpha = expf(mx - mnew);
    const float pv = expf(dot - mnew);
    l = l * alpha + pv;
#pragma unroll
    for (int i = 0; i < kO; ++i) {
      const int k = lane + 32 * i;
      if (k < r) acc[i] = fmaf(pv, ld_f32(row + k), acc[i] * alpha);
    }
    mx = mnew;
  }
  T* out = reinterpret_cast<T*>(p.out) + ((b * Tn + (m - 1)) * H + h) * r;
#pragma unroll
  for (int i = 0; i < kO; ++i) {
    const int k = lane + 32 * i;
    if (k < r) st_elem(out + k, acc[i] / l);
  }
}

// ----------------------------------------------------------------------------
// launchers
// ----------------------------------------------------------------------------
template <typename T>
cudaError_t launch_merge_append_t(const SeqArgs& a, const MergeArgsDev& m, int B, cudaStream_t st) {
  const size_t smem = (size_t)a.r * sizeof(float);
  merge_append_kernel<T><<<B, 256, smem, st>>>(a, m);
  return cudaGetLastError();
}
cudaError_t launch_merge_append(const SeqArgs& a, const MergeArgsDev& m, int B, int dtype, cudaStream_t st) {
  return dtype == MTLA_BF16 ? launch_merge_append_t<__nv_bfloat16>(a, m, B, st)
                            : launch_merge_append_t<float>(a, m, B, st);
}

template <typename T>
cudaError_t launch_decode_simt_t(const SeqArgs& a, const MergeArgsDev& m, bool with_merge, const DecodeOut& o,
                                 int B, cudaStream_t st) {
  const size_t smem = ((size_t)a.r + (size_t)o.H * (a.r + a.d_R) + kSimtThreads + 32) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  decode_simt_kernel<T><<<B, kSimtThreads, smem, st>>>(a, m, with_merge, o);
  return cudaGetLastError();
}
cudaError_t launch_decode_simt(const SeqArgs& a, const MergeArgsDev& m, bool with_merge, const DecodeOut& o,
                               int B, int dtype, cudaStream_t st) {
  return dtype == MTLA_BF16 ? launch_decode_simt_t<__nv_bfloat16>(a, m, with_merge, o, B, st)
                            : launch_decode_simt_t<float>(a, m, with_merge, o, B, st);
}

template <typename T, int TPT, int CPT>
cudaError_t launch_partial_merge_tc(PrefillArgs p, int B, cudaStream_t st) {
  constexpr int TC = 16 * TPT;
  const int D = p.r + p.d_R;
  const int64_t n_groups = cdiv(p.T, p.s);
  // whole groups per block: as many as fit one chunk, at least one
  int64_t gpb = TC / p.s;
  if (gpb < 1) gpb = 1;
  p.groups_per_block = gpb;
  const size_t smem = ((size_t)32 * D + (size_t)TC * 32 + (size_t)TC * D) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(partial_merge_kernel<T, TPT, CPT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)cdiv(n_groups, gpb), (unsigned)B);
  partial_merge_kernel<T, TPT, CPT><<<grid, 256, smem, st>>>(p);
  return cudaGetLastError();
}
template <typename T>
cudaError_t launch_partial_merge_t(const PrefillArgs& p, int B, cudaStream_t st) {
  const int D = p.r + p.d_R;
  if (D <= 16 * 6) return launch_partial_merge_tc<T, 4, 6>(p, B, st);
  if (D <= 16 * 18) return launch_partial_merge_tc<T, 4, 18>(p, B, st);
  return launch_partial_merge_tc<T, 2, 36>(p, B, st);
}
cudaError_t launch_partial_merge(const PrefillArgs& p, int B, int dtype, cudaStream_t st) {
  return dtype == MTLA_BF16 ? launch_partial_merge_t<__nv_bfloat16>(p, B, st)
                            : launch_partial_merge_t<float>(p, B, st);
}

cudaError_t launch_prefill_simt(const PrefillArgs& p, int B, int dtype, cudaStream_t st) {
  const unsigned blocks = (unsigned)((int64_t)B * p.T);
  if (dtype == MTLA_BF16)
    prefill_simt_kernel<__nv_bfloat16><<<blocks, 32 * p.H, 0, st>>>(p);
  else
    prefill_simt_kernel<float><<<blocks, 32 * p.H, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace mtla
