// mtla_decode_attn_static: the decode step with its scratch in a static device
// array instead of a caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory around a decode
// step.  Examples are an engine that has handed all free memory to its cache
// page pool and has nothing left to carve a workspace from, and plain C host
// code that holds no device allocator and would otherwise have to manage a
// workspace's lifetime.  Nothing here calls cudaMalloc, cudaFree or any
// allocating library routine.  The scratch is one array of
// MTLA_DECODE_STATIC_SCRATCH_BYTES per device.  The driver reserves it when
// it loads this library's device code into a context.
//
// Set-up: the first call on a device, with that device current, looks up the
// array's device address (cudaGetSymbolAddress) and clears it on the caller's
// stream.  The decode reads only what the same call wrote, so the clearing is
// not needed for correctness; it only keeps the scratch's first contents
// defined.  Make the first call on each device before any stream capture.
// The driver reserves the array when it loads this library's device code
// into a context; under lazy module loading (the CUDA default) that happens
// at this first call.  The address is kept for the life of the process, so
// the entry point must not be used on a device after cudaDeviceReset (which
// unloads the array).
//
// Sharing: every call on a device uses the same scratch, so calls that can
// overlap (different streams, or threads without ordering between them) race
// on it.  Issue them one after another on one stream.
#include <mutex>

#include "kernels.cuh"

namespace mtla {
namespace {

// file-scope scratch; 24 MiB covers the split-L kernel's workspace for every
// B it accepts (B <= 1024) on a 148-SM B200 (about 5.5 MB at B = 1024)
__device__ __align__(256) unsigned char g_decode_scratch[MTLA_DECODE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// device address of this device's scratch; the first call per device clears
// it on `stream`
mtla_status static_scratch(cudaStream_t stream, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MTLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MTLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) return MTLA_ERR_CUDA;
    if (cudaMemsetAsync(ptr, 0, MTLA_DECODE_STATIC_SCRATCH_BYTES, stream) != cudaSuccess) return MTLA_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return MTLA_OK;
}

}  // namespace
}  // namespace mtla

extern "C" {

mtla_status mtla_decode_attn_static(const mtla_dims* dims, int32_t B, const void* q_abs, const void* q_rope,
                                    const mtla_merge_args* merge, void* cache, int64_t cache_rows,
                                    int64_t row_stride, const int64_t* seq_offset, const int64_t* seq_capacity,
                                    int32_t* t_processed, int32_t* cache_len, float* out, float* lse,
                                    int32_t* dev_err, void* stream) {
  // the scratch this call would need from a workspace; beyond the array's
  // size the call is refused before anything runs
  if (mtla_workspace_bytes(dims, B, MTLA_WS_DECODE) > (size_t)MTLA_DECODE_STATIC_SCRATCH_BYTES)
    return MTLA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const mtla_status st = mtla::static_scratch(static_cast<cudaStream_t>(stream), &scratch);
  if (st != MTLA_OK) return st;
  return mtla_decode_attn(dims, B, q_abs, q_rope, merge, cache, cache_rows, row_stride, seq_offset, seq_capacity,
                          t_processed, cache_len, out, lse, scratch, MTLA_DECODE_STATIC_SCRATCH_BYTES, dev_err,
                          stream);
}

}  // extern "C"
