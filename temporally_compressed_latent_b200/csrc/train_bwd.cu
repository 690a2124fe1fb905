// The two small kernels around the tensor-core gradient kernels of the
// training shortcut's backward pass (MTLA paper notes, "Key designs:
// decoupled RoPE with temporal compression" and "stride-aware causal mask"):
// - prep: Delta_m = dO_m . O_m and the forward's lse in log2 units of the
//   scaled score, per (sequence, head, query), in rows of Tp (T rounded up
//   to 64) so that a 64-query tile of them is one aligned bulk copy;
// - dk^R summed over heads in a fixed order (every head reads the same K^R).
#include "kernels.cuh"

namespace mtla {
namespace tbw {

constexpr int DH = 64, DR = 32;
__device__ __forceinline__ float2 bf2(uint32_t u) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
}
__device__ __forceinline__ float dot2(uint32_t a, uint32_t b) {
  const float2 x = bf2(a), y = bf2(b);
  return x.x * y.x + x.y * y.y;
}
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdArgs p) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // (b, t, h)
  if (idx >= (int64_t)p.B * p.T * p.H) return;
  const int h = (int)(idx % p.H);
  const int64_t bt = idx / p.H;
  const int64_t b = bt / p.T, t = bt % p.T;
  const uint4* o4 = reinterpret_cast<const uint4*>(p.o + idx * DH);
  const uint4* d4 = reinterpret_cast<const uint4*>(p.dout + idx * DH);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < DH / 8; ++i) {
    const uint4 a = o4[i], c = d4[i];
    acc += dot2(a.x, c.x) + dot2(a.y, c.y) + dot2(a.z, c.z) + dot2(a.w, c.w);
  }
  const int64_t o = (b * p.H + h) * p.Tp + t;
  p.ws_delta[o] = acc;
  p.ws_lse2[o] = p.lse[idx] * 1.4426950408889634f;
}

// dk^R [b, t, :] = sum over heads of the per-head RoPE key gradients (fixed order)
__global__ void __launch_bounds__(256) dkr_reduce_kernel(const float* dkrh, float* dkr, int64_t rows, int H) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * DR) return;
  const int64_t row = idx / DR;
  const int c = (int)(idx % DR);
  float acc = 0.f;
  for (int h = 0; h < H; ++h) acc += dkrh[(row * H + h) * DR + c];
  dkr[idx] = acc;
}

}  // namespace tbw

cudaError_t launch_bwd_prep(const BwdArgs& a, cudaStream_t st) {
  const int64_t nth = (int64_t)a.B * a.T * a.H;
  tbw::bwd_prep_kernel<<<(unsigned)((nth + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dkr_reduce(const BwdArgs& a, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * a.T;
  tbw::dkr_reduce_kernel<<<(unsigned)((rows * tbw::DR + 255) / 256), 256, 0, st>>>(a.ws_dkrh, a.dkr, rows, a.H);
  return cudaGetLastError();
}

}  // namespace mtla
