// C ABI of the MTLA library: argument checks, kernel selection, launches.
// See include/mtla.h for the contract of every entry point.
#include <math.h>
#include <string.h>

#include <mutex>

#include "kernels.cuh"

namespace {

using namespace mtla;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_size(int dtype) { return dtype == MTLA_BF16 ? 2 : 4; }

mtla_status check_dims(const mtla_dims* d) {
  if (!d) return MTLA_ERR_INVALID_ARG;
  if (d->H < 1 || d->d_h < 1 || d->r < 1 || d->d_R < 0 || d->s < 1) return MTLA_ERR_INVALID_ARG;
  if (d->dtype != MTLA_F32 && d->dtype != MTLA_BF16) return MTLA_ERR_INVALID_ARG;
  // limits of the generic kernels (register tiles sized for these)
  if (d->H > 16 || d->r > 512 || d->r + d->d_R > 576) return MTLA_ERR_UNSUPPORTED;
  if (d->dtype == MTLA_BF16 && ((d->r % 8) || (d->d_R % 8))) return MTLA_ERR_UNSUPPORTED;
  if (d->dtype == MTLA_F32 && ((d->r % 4) || (d->d_R % 4))) return MTLA_ERR_UNSUPPORTED;
  return MTLA_OK;
}

bool tc_decode_dims(const mtla_dims* d, int B) {
  return d->dtype == MTLA_BF16 && d->H == dtc::H && d->r == dtc::R && d->d_R == dtc::DR && B <= dtc::MAXB;
}

// persistent grid of the tensor-core decode on the current device, cached per device
int decode_grid() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  const int g = dtc::grid_size();
  if (dev < 64 && g > 0) cached[dev] = g;
  return g;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library needs no link-time dependency on libcuda.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D view of a bf16 cache: {32 elements, cache_rows rows, 9 segments of 32};
// with the segment as the outermost dimension a box lands in shared memory as
// one [rows x 64 B] plane per segment.
bool encode_cache_map(CUtensorMap* map, void* cache, int64_t cache_rows, int64_t row_stride, uint32_t box_rows,
                      uint32_t box_planes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {32, (cuuint64_t)cache_rows, (cuuint64_t)(dtc::D / 32)};
  const cuuint64_t strides[2] = {(cuuint64_t)row_stride * 2, 64};
  const cuuint32_t box[3] = {32, box_rows, box_planes};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, cache, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Generic tiled map of a bf16 tensor with the 64-byte swizzle (dims innermost first).
bool encode_map(CUtensorMap* map, CUtensorMapDataType type, const void* base, int rank, const cuuint64_t* dims,
                const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(map, type, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool encode_bf16_map(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                     const cuuint32_t* box, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_64B) {
  return encode_map(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides, box, swizzle);
}

// the running merge on the tensor cores: bf16, r = 256, d_R = 32, s <= 32
bool tc_merge_dims(const mtla_dims* d, int B, int T) {
  return d->dtype == MTLA_BF16 && d->r == 256 && d->d_R == 32 && d->s <= 32 &&
         (int64_t)B * T + 256 < (int64_t(1) << 31);
}

bool tc_prefill_dims(const mtla_dims* d, int B, int T) {
  return d->dtype == MTLA_BF16 && d->H == 8 && d->r == 256 && d->d_R == 32 && T >= 1 &&
         (int64_t)B * T * 8 < (int64_t(1) << 31);
}

struct CacheMaps {
  void* ptr = nullptr;
  int64_t rows = -1, stride = -1;
  CUtensorMap m64, m8;
};

// The tensor maps of the last few cache buffers a thread used (a caller
// that rotates several caches finds each of them encoded), replaced in
// round-robin order.  Returns nullptr if encoding fails.
const CacheMaps* cache_maps(void* cache, int64_t cache_rows, int64_t row_stride) {
  constexpr int kSlots = 32;
  thread_local CacheMaps slot[kSlots];
  thread_local int next = 0;
  for (int i = 0; i < kSlots; ++i)
    if (slot[i].ptr == cache && slot[i].rows == cache_rows && slot[i].stride == row_stride) return &slot[i];
  CacheMaps& m = slot[next];
  next = (next + 1) % kSlots;
  if (!encode_cache_map(&m.m64, cache, cache_rows, row_stride, dtc::UNIT, dtc::D / 32) ||
      !encode_cache_map(&m.m8, cache, cache_rows, row_stride, dtc::SUB, 1)) {
    m.ptr = nullptr;
    return nullptr;
  }
  m.ptr = cache;
  m.rows = cache_rows;
  m.stride = row_stride;
  return &m;
}

mtla_status seq_args(const mtla_dims* d, void* cache, int64_t cache_rows, int64_t row_stride,
                     const int64_t* seq_offset, const int64_t* seq_capacity, int32_t* t_processed,
                     int32_t* cache_len, int32_t* dev_err, SeqArgs* a) {
  if (!cache || !seq_offset || !seq_capacity || !t_processed || !dev_err) return MTLA_ERR_INVALID_ARG;
  if (!aligned16(cache) || !aligned16(seq_offset) || !aligned16(seq_capacity)) return MTLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(t_processed) & 3) || (cache_len && (reinterpret_cast<uintptr_t>(cache_len) & 3)) ||
      (reinterpret_cast<uintptr_t>(dev_err) & 3))
    return MTLA_ERR_INVALID_ARG;
  const int D = d->r + d->d_R;
  if (cache_rows < 0 || cache_rows >= (int64_t(1) << 31) || row_stride < D) return MTLA_ERR_INVALID_ARG;
  if ((row_stride * (int64_t)elem_size(d->dtype)) % 16) return MTLA_ERR_INVALID_ARG;
  a->cache = cache;
  a->cache_rows = cache_rows;
  a->row_stride = row_stride;
  a->seq_offset = seq_offset;
  a->seq_capacity = seq_capacity;
  a->t_processed = t_processed;
  a->cache_len = cache_len;
  a->dev_err = dev_err;
  a->r = d->r;
  a->d_R = d->d_R;
  a->s = d->s;
  return MTLA_OK;
}

mtla_status merge_args(const mtla_merge_args* m, MergeArgsDev* md) {
  if (!m || !m->c_new || !m->kR_new || !m->W_c || !m->b_c || !m->P || m->J_max < 1) return MTLA_ERR_INVALID_ARG;
  if (!aligned16(m->c_new) || !aligned16(m->kR_new) || !aligned16(m->W_c) || !aligned16(m->b_c) ||
      !aligned16(m->P))
    return MTLA_ERR_INVALID_ARG;
  md->c_new = m->c_new;
  md->kR_new = m->kR_new;
  md->W_c = m->W_c;
  md->b_c = m->b_c;
  md->P = m->P;
  md->J_max = m->J_max;
  return MTLA_OK;
}

mtla_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MTLA_OK : MTLA_ERR_CUDA; }

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return sms;
}

// rows of the input map: H r absorbed-query rows, H d_R RoPE-query rows, r
// latent rows, d_R RoPE-key rows
int64_t proj_in_rows(const mtla_dims* d) { return (int64_t)d->H * (d->r + d->d_R) + d->r + d->d_R; }

// workspace of one projection call: the fp32 partial sums of one launch
size_t proj_ws(const mtla_dims* dims, int32_t B, int32_t d, int32_t which) {
  if (check_dims(dims) != MTLA_OK || B < 1 || d < 1) return 0;
  const int64_t N = which == MTLA_PROJ_IN ? proj_in_rows(dims) : d;
  const int64_t K = which == MTLA_PROJ_IN ? d : (int64_t)dims->H * dims->r;
  if (dims->dtype != MTLA_BF16) return (size_t)B * N * 4;
  const int sms = device_sms();
  if (sms <= 0) return 0;
  const ProjSplit sp = proj_split(B, (int)K, (int)N, sms);
  return (size_t)sp.KS * sp.Bp * N * 4;
}

// 2-D map of a row-major bf16 weight [N rows, K] in boxes of 64 x 128 with the 128-byte swizzle
bool encode_weight_map(CUtensorMap* map, const void* W, int64_t N, int64_t K) {
  const cuuint64_t dims2[2] = {(cuuint64_t)K, (cuuint64_t)N}, str[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {64, 128};
  return encode_bf16_map(map, W, 2, dims2, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

extern "C" {

const char* mtla_status_string(mtla_status st) {
  switch (st) {
    case MTLA_OK: return "ok";
    case MTLA_ERR_INVALID_ARG: return "invalid argument";
    case MTLA_ERR_UNSUPPORTED: return "unsupported dimensions or dtype";
    case MTLA_ERR_WORKSPACE: return "workspace missing or too small";
    case MTLA_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

int64_t mtla_cache_length(int64_t t, int32_t s) {
  if (t <= 0 || s < 1) return 0;
  return group_of(t, s);
}

mtla_status mtla_debug_stride_mask(int32_t s, int32_t T, uint8_t* host_out) {
  if (s < 1 || T < 0 || (T > 0 && !host_out)) return MTLA_ERR_INVALID_ARG;
  for (int64_t m = 1; m <= T; ++m)
    for (int64_t n = 1; n <= T; ++n) host_out[(m - 1) * T + (n - 1)] = stride_visible(m, n, s) ? 1 : 0;
  return MTLA_OK;
}

size_t mtla_workspace_bytes(const mtla_dims* dims, int32_t B, int32_t which) {
  if (check_dims(dims) != MTLA_OK || B < 0) return 0;
  if (which == MTLA_WS_DECODE && tc_decode_dims(dims, B)) {
    const int g = decode_grid();
    return g > 0 ? dtc::workspace_bytes(B, g) : 0;
  }
  return 0;
}

mtla_status mtla_merge_append(const mtla_dims* dims, int32_t B, const mtla_merge_args* merge, void* cache,
                              int64_t cache_rows, int64_t row_stride, const int64_t* seq_offset,
                              const int64_t* seq_capacity, int32_t* t_processed, int32_t* cache_len,
                              int32_t* dev_err, void* stream) {
  mtla_status st = check_dims(dims);
  if (st != MTLA_OK) return st;
  if (B < 0) return MTLA_ERR_INVALID_ARG;
  SeqArgs a;
  MergeArgsDev m;
  if ((st = seq_args(dims, cache, cache_rows, row_stride, seq_offset, seq_capacity, t_processed, cache_len, dev_err,
                     &a)) != MTLA_OK)
    return st;
  if ((st = merge_args(merge, &m)) != MTLA_OK) return st;
  if (B == 0) return MTLA_OK;
  return from_cuda(launch_merge_append(a, m, B, dims->dtype, static_cast<cudaStream_t>(stream)));
}

mtla_status mtla_decode_attn(const mtla_dims* dims, int32_t B, const void* q_abs, const void* q_rope,
                             const mtla_merge_args* merge, void* cache, int64_t cache_rows, int64_t row_stride,
                             const int64_t* seq_offset, const int64_t* seq_capacity, int32_t* t_processed,
                             int32_t* cache_len, float* out, float* lse, void* workspace, size_t workspace_bytes,
                             int32_t* dev_err, void* stream) {
  mtla_status st = check_dims(dims);
  if (st != MTLA_OK) return st;
  if (B < 0) return MTLA_ERR_INVALID_ARG;
  SeqArgs a;
  MergeArgsDev m = {};
  if ((st = seq_args(dims, cache, cache_rows, row_stride, seq_offset, seq_capacity, t_processed, cache_len, dev_err,
                     &a)) != MTLA_OK)
    return st;
  if (merge && (st = merge_args(merge, &m)) != MTLA_OK) return st;
  if (!q_abs || !q_rope || !out || !aligned16(q_abs) || !aligned16(q_rope) || !aligned16(out) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
    return MTLA_ERR_INVALID_ARG;
  if (B == 0) return MTLA_OK;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  DecodeOut o;
  o.q_abs = q_abs;
  o.q_rope = q_rope;
  o.out = out;
  o.lse = lse;
  o.scale = (float)(1.0 / sqrt((double)dims->d_h));
  o.H = dims->H;
  o.tails = nullptr;

  if (!tc_decode_dims(dims, B))
    return from_cuda(launch_decode_simt(a, m, merge != nullptr, o, B, dims->dtype, cs));

  const int grid = decode_grid();
  if (grid <= 0) return MTLA_ERR_CUDA;
  const size_t need = dtc::workspace_bytes(B, grid);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return MTLA_ERR_WORKSPACE;

  const CacheMaps* maps = cache_maps(cache, cache_rows, row_stride);
  if (!maps) return MTLA_ERR_CUDA;
  dtc::Params p;
  p.a = a;
  p.m = m;
  p.o = o;
  p.with_merge = merge != nullptr;
  p.patch = 0;
  p.B = B;
  p.merge_cost = dtc::MERGE_COST;
  p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)dims->d_h));
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const dtc::WsLayout wl = dtc::ws_layout(B, grid);
  p.seq_info = reinterpret_cast<int4*>(ws + wl.seq_info);
  p.tails = reinterpret_cast<__nv_bfloat16*>(ws + wl.tails);
  p.ws_ml = reinterpret_cast<float*>(ws + wl.ml);
  p.ws_o = reinterpret_cast<float*>(ws + wl.o);
  return from_cuda(launch_decode_tc(p, maps->m64, maps->m8, grid, cs));
}

mtla_status mtla_prefill_masked_attn(const mtla_dims* dims, int32_t B, int32_t T, const void* q_abs,
                                     const void* q_rope, const void* c, const void* kR, const float* W_c,
                                     const float* b_c, const float* P, int32_t J_max, void* c_partial,
                                     void* cache_out, void* out, int32_t* dev_err, void* stream) {
  mtla_status st = check_dims(dims);
  if (st != MTLA_OK) return st;
  if (B < 0 || T < 0) return MTLA_ERR_INVALID_ARG;
  if (!c || !kR || !W_c || !b_c || !P || !c_partial || !dev_err) return MTLA_ERR_INVALID_ARG;
  if (out && (!q_abs || !q_rope)) return MTLA_ERR_INVALID_ARG;
  const void* ptrs[] = {c, kR, W_c, b_c, P, c_partial};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return MTLA_ERR_INVALID_ARG;
  if (out && (!aligned16(out) || !aligned16(q_abs) || !aligned16(q_rope))) return MTLA_ERR_INVALID_ARG;
  if (cache_out && !aligned16(cache_out)) return MTLA_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return MTLA_OK;
  if ((int64_t)J_max < cdiv(T, dims->s)) return MTLA_ERR_INVALID_ARG;
  if ((int64_t)B * T >= (int64_t(1) << 31)) return MTLA_ERR_UNSUPPORTED;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  PrefillArgs p;
  p.q_abs = q_abs;
  p.q_rope = q_rope;
  p.c = c;
  p.kR = kR;
  p.W_c = W_c;
  p.b_c = b_c;
  p.P = P;
  p.c_partial = c_partial;
  p.cache_out = cache_out;
  p.out = out;
  p.dev_err = dev_err;
  p.T = T;
  p.groups_per_block = 1;
  p.H = dims->H;
  p.r = dims->r;
  p.d_R = dims->d_R;
  p.s = dims->s;
  p.scale = (float)(1.0 / sqrt((double)dims->d_h));
  p.J_max = J_max;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MTLA_ERR_CUDA;
  cudaError_t e;
  if (tc_merge_dims(dims, B, T)) {  // every pointer is 16-byte aligned (checked above)
    // latents as [B*T rows, 256], boxes of 64 latents x 128 rows, 128-byte
    // swizzle; RoPE keys [B*T rows, 32], boxes of 128 rows; P [J rows, 288]
    // fp32, boxes of one channel tile (96) x one tile's groups; C_hat' as
    // [B][T][288] and the cache rows as [B][groups][288], boxes of one
    // warp's 32 channels x a quarter of a 128-token tile (or its groups)
    const int s = dims->s, tt = (128 / s) * s;
    const int64_t ng = cdiv(T, s);
    MergeMaps mm;
    const CUtensorMapSwizzle none = CU_TENSOR_MAP_SWIZZLE_NONE;
    {
      const cuuint64_t dims2[2] = {256, (cuuint64_t)B * T}, str[1] = {512};
      const cuuint32_t box[2] = {64, 128};
      if (!encode_bf16_map(&mm.c, c, 2, dims2, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MTLA_ERR_CUDA;
    }
    {
      const cuuint64_t dims2[2] = {32, (cuuint64_t)B * T}, str[1] = {64};
      const cuuint32_t box[2] = {32, 128};
      if (!encode_bf16_map(&mm.kr, kR, 2, dims2, str, box, none)) return MTLA_ERR_CUDA;
    }
    {
      const cuuint64_t dims2[2] = {288, (cuuint64_t)J_max}, str[1] = {288 * 4};
      const cuuint32_t box[2] = {96, (cuuint32_t)(tt / s)};
      if (!encode_map(&mm.p, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, P, 2, dims2, str, box, none)) return MTLA_ERR_CUDA;
    }
    {
      const cuuint64_t dims3[3] = {288, (cuuint64_t)T, (cuuint64_t)B}, str[2] = {576, (cuuint64_t)T * 576};
      const cuuint32_t box[3] = {32, 32, 1};  // one warp's channels x a quarter of a 128-token tile
      if (!encode_bf16_map(&mm.out, c_partial, 3, dims3, str, box, none)) return MTLA_ERR_CUDA;
    }
    mm.cache = mm.out;
    if (cache_out) {
      const cuuint64_t dims3[3] = {288, (cuuint64_t)ng, (cuuint64_t)B}, str[2] = {576, (cuuint64_t)ng * 576};
      const cuuint32_t box[3] = {32, (cuuint32_t)(s <= 32 ? 32 / s : 1), 1};  // the groups of a quarter
      if (!encode_bf16_map(&mm.cache, cache_out, 3, dims3, str, box, none)) return MTLA_ERR_CUDA;
    }
    e = launch_merge_tc(p, B, mm, sms, cs);
  } else {
    e = launch_partial_merge(p, B, dims->dtype, cs);
  }
  if (e != cudaSuccess) return MTLA_ERR_CUDA;
  if (!out) return MTLA_OK;
  if (!tc_prefill_dims(dims, B, T)) return from_cuda(launch_prefill_simt(p, B, dims->dtype, cs));

  // tensor-core path: queries as 9 planes of 32, own rows, and the completed
  // groups C_hat'_{g s} read through a map whose row stride is s rows
  const int s = dims->s;
  const cuuint64_t rows_q = (cuuint64_t)B * T * 8, rows_c = (cuuint64_t)B * T;
  CUtensorMap qmap, rmap, smap, kmap;
  {
    const cuuint64_t dims3[3] = {32, rows_q, 8}, str[2] = {512, 64};
    const cuuint32_t box[3] = {32, 128, 8};
    if (!encode_bf16_map(&qmap, q_abs, 3, dims3, str, box)) return MTLA_ERR_CUDA;
  }
  {
    const cuuint64_t dims2[2] = {32, rows_q}, str[1] = {64};
    const cuuint32_t box[2] = {32, 128};
    if (!encode_bf16_map(&rmap, q_rope, 2, dims2, str, box)) return MTLA_ERR_CUDA;
  }
  {
    const cuuint64_t dims3[3] = {32, rows_c, 9}, str[2] = {576, 64};
    const cuuint32_t box[3] = {32, 16, 9};
    if (!encode_bf16_map(&smap, c_partial, 3, dims3, str, box)) return MTLA_ERR_CUDA;
  }
  {
    const int64_t groups = T / s;
    const cuuint64_t dims4[4] = {32, (cuuint64_t)(groups > 0 ? groups : 1), 9, (cuuint64_t)B};
    const cuuint64_t str[3] = {(cuuint64_t)s * 576, 64, (cuuint64_t)T * 576};
    const cuuint32_t box[4] = {32, 64, 9, 1};
    const __nv_bfloat16* base = reinterpret_cast<const __nv_bfloat16*>(c_partial) + (s - 1) * 288;
    if (!encode_bf16_map(&kmap, base, 4, dims4, str, box)) return MTLA_ERR_CUDA;
  }
  PrefillTcLaunch a;
  a.B = B;
  a.T = T;
  a.s = s;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)dims->d_h));
  a.out = out;
  a.dev_err = dev_err;
  const int tiles = B * ((T + 15) / 16);
  return from_cuda(launch_prefill_tc_args(a, qmap, rmap, smap, kmap, tiles < sms ? tiles : sms, cs));
}

// Workspace of a call with n new tokens per sequence: the B n virtual
// sequences' arrays, their tail rows, then the split-L workspace for B n.
struct MultiLayout {
  size_t t_v, off_v, cap_v, tails, gates, dec, total;
};
static MultiLayout multi_layout(const mtla_dims* dims, int32_t B, int32_t n, size_t dec_bytes) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t Bv = (size_t)B * n;
  MultiLayout l;
  l.t_v = 0;
  l.off_v = up(Bv * 4);
  l.cap_v = l.off_v + up(Bv * 8);
  l.tails = l.cap_v + up(Bv * 8);
  l.gates = l.tails + up(Bv * (dims->r + dims->d_R) * elem_size(dims->dtype));
  l.dec = l.gates + up(Bv * (dims->r + dims->d_R) * 4);
  l.total = l.dec + dec_bytes;
  return l;
}

size_t mtla_decode_multi_workspace_bytes(const mtla_dims* dims, int32_t B, int32_t n) {
  if (check_dims(dims) != MTLA_OK || B < 0 || n < 1 || n > MTLA_MAX_NEW_TOKENS) return 0;
  return multi_layout(dims, B, n, mtla_workspace_bytes(dims, B * n, MTLA_WS_DECODE)).total;
}

mtla_status mtla_decode_attn_multi(const mtla_dims* dims, int32_t B, int32_t n, const void* q_abs, const void* q_rope,
                                   const mtla_merge_args* merge, void* cache, int64_t cache_rows, int64_t row_stride,
                                   const int64_t* seq_offset, const int64_t* seq_capacity, int32_t* t_processed,
                                   int32_t* cache_len, float* out, float* lse, void* workspace,
                                   size_t workspace_bytes, int32_t* dev_err, void* stream) {
  mtla_status st = check_dims(dims);
  if (st != MTLA_OK) return st;
  if (B < 0 || n < 1 || n > MTLA_MAX_NEW_TOKENS || (int64_t)B * n > (int64_t(1) << 24)) return MTLA_ERR_INVALID_ARG;
  SeqArgs a;
  MergeArgsDev m = {};
  if ((st = seq_args(dims, cache, cache_rows, row_stride, seq_offset, seq_capacity, t_processed, cache_len, dev_err,
                     &a)) != MTLA_OK)
    return st;
  if ((st = merge_args(merge, &m)) != MTLA_OK) return st;
  if (!q_abs || !q_rope || !out || !aligned16(q_abs) || !aligned16(q_rope) || !aligned16(out) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
    return MTLA_ERR_INVALID_ARG;
  if (B == 0) return MTLA_OK;
  const int Bv = B * n;
  const bool tc = tc_decode_dims(dims, Bv);
  const int grid = tc ? decode_grid() : 0;
  if (tc && grid <= 0) return MTLA_ERR_CUDA;
  const size_t dec_bytes = tc ? dtc::workspace_bytes(Bv, grid) : 0;
  const MultiLayout ml = multi_layout(dims, B, n, dec_bytes);
  if (!workspace || !aligned16(workspace) || workspace_bytes < ml.total) return MTLA_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  // 1. the n tokens of every sequence, merged in order
  MultiMergeArgs mm;
  mm.a = a;
  mm.m = m;
  mm.n = n;
  mm.four_part = tc && dims->r == dtc::R && dims->d_R == dtc::DR;  // the tensor-core step's gate order
  mm.tails = ws + ml.tails;
  mm.gates = reinterpret_cast<float*>(ws + ml.gates);
  mm.t_v = reinterpret_cast<int32_t*>(ws + ml.t_v);
  mm.off_v = reinterpret_cast<int64_t*>(ws + ml.off_v);
  mm.cap_v = reinterpret_cast<int64_t*>(ws + ml.cap_v);
  if (launch_multi_merge(mm, B, dims->dtype, cs) != cudaSuccess) return MTLA_ERR_CUDA;

  // 2. the attention of the B n queries: virtual sequence b n + i reads b's
  // rows up to ceil((t0 + i + 1) / s) with its last row from the tails
  SeqArgs av = a;
  av.t_processed = mm.t_v;
  av.seq_offset = mm.off_v;
  av.seq_capacity = mm.cap_v;
  av.cache_len = nullptr;
  DecodeOut o;
  o.q_abs = q_abs;
  o.q_rope = q_rope;
  o.out = out;
  o.lse = lse;
  o.scale = (float)(1.0 / sqrt((double)dims->d_h));
  o.H = dims->H;
  o.tails = mm.tails;
  if (!tc) return from_cuda(launch_decode_simt(av, m, false, o, Bv, dims->dtype, cs));

  const CacheMaps* maps = cache_maps(cache, cache_rows, row_stride);
  if (!maps) return MTLA_ERR_CUDA;
  dtc::Params p;
  p.a = av;
  p.m = m;
  p.o = o;
  p.with_merge = 0;
  p.patch = 1;
  p.B = Bv;
  p.merge_cost = 0;
  p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)dims->d_h));
  const dtc::WsLayout wl = dtc::ws_layout(Bv, grid);
  uint8_t* dws = ws + ml.dec;
  p.seq_info = reinterpret_cast<int4*>(dws + wl.seq_info);
  p.tails = reinterpret_cast<__nv_bfloat16*>(mm.tails);
  p.ws_ml = reinterpret_cast<float*>(dws + wl.ml);
  p.ws_o = reinterpret_cast<float*>(dws + wl.o);
  return from_cuda(launch_decode_tc(p, maps->m64, maps->m8, grid, cs));
}

static bool unabs_dims(const mtla_dims* d) {
  return d->dtype == MTLA_BF16 && d->d_h == 64 && d->d_R == 32 && d->r % 64 == 0 && d->r <= 256 && d->H % 2 == 0;
}

// Tensor maps of the un-absorbed attention's bf16 operands, 64-byte swizzle,
// boxes 32 elements wide: a 64-wide row lands as two [rows x 64 B] planes.
// Rows of a [B T, H, 64] tensor for one head: 4-D {32, H, B T, 2 planes}.
static bool map_head_rows(CUtensorMap* m, const void* base, int H, int64_t BT, uint32_t rows) {
  const cuuint64_t d[4] = {32, (cuuint64_t)H, (cuuint64_t)BT, 2}, st[3] = {128, (cuuint64_t)H * 128, 64};
  const cuuint32_t box[4] = {32, 1, rows, 2};
  return encode_bf16_map(m, base, 4, d, st, box);
}
// Rows of a [B T, H, 32] tensor (q^R) for one head: 3-D {32, H, B T}.
static bool map_head_rope(CUtensorMap* m, const void* base, int H, int64_t BT, uint32_t rows) {
  const cuuint64_t d[3] = {32, (cuuint64_t)H, (cuuint64_t)BT}, st[2] = {64, (cuuint64_t)H * 64};
  const cuuint32_t box[3] = {32, 1, rows};
  return encode_bf16_map(m, base, 3, d, st, box);
}
// Rows of the RoPE keys (row n at kr + n kr_stride): 2-D {32, B T}.
static bool map_key_rope(CUtensorMap* m, const void* kr, int64_t kr_stride, int64_t BT, uint32_t rows) {
  const cuuint64_t d[2] = {32, (cuuint64_t)BT}, st[1] = {(cuuint64_t)kr_stride * 2};
  const cuuint32_t box[2] = {32, rows};
  return encode_bf16_map(m, kr, 2, d, st, box);
}
// The group columns n = g s (0-based rows s - 1, 2 s - 1, ...) of each
// sequence; G = T / s of them (a sequence with none still gets a valid map,
// never read).  [B T, H, 64] tensors: 5-D {32, H, G, B, 2 planes}.
static bool map_group_rows(CUtensorMap* m, const void* base, int H, int s, int T, int B, uint32_t groups) {
  const int64_t G = T / s, Gm = G > 0 ? G : 1, off = G > 0 ? s - 1 : 0;
  const cuuint64_t d[5] = {32, (cuuint64_t)H, (cuuint64_t)Gm, (cuuint64_t)B, 2};
  const cuuint64_t st[4] = {128, (cuuint64_t)s * H * 128, (cuuint64_t)T * H * 128, 64};
  const cuuint32_t box[5] = {32, 1, groups, 1, 2};
  return encode_bf16_map(m, static_cast<const __nv_bfloat16*>(base) + off * H * 64, 5, d, st, box);
}
// [B T, H, 32] tensors (q^R) at the group columns: 4-D {32, H, G, B}.
static bool map_group_rope(CUtensorMap* m, const void* base, int H, int s, int T, int B, uint32_t groups) {
  const int64_t G = T / s, Gm = G > 0 ? G : 1, off = G > 0 ? s - 1 : 0;
  const cuuint64_t d[4] = {32, (cuuint64_t)H, (cuuint64_t)Gm, (cuuint64_t)B};
  const cuuint64_t st[3] = {64, (cuuint64_t)s * H * 64, (cuuint64_t)T * H * 64};
  const cuuint32_t box[4] = {32, 1, groups, 1};
  return encode_bf16_map(m, static_cast<const __nv_bfloat16*>(base) + off * H * 32, 4, d, st, box);
}
// The RoPE keys at the group columns: 3-D {32, G, B}.
static bool map_group_key_rope(CUtensorMap* m, const void* kr, int64_t kr_stride, int s, int T, int B,
                               uint32_t groups) {
  const int64_t G = T / s, Gm = G > 0 ? G : 1, off = G > 0 ? s - 1 : 0;
  const cuuint64_t d[3] = {32, (cuuint64_t)Gm, (cuuint64_t)B};
  const cuuint64_t st[2] = {(cuuint64_t)s * kr_stride * 2, (cuuint64_t)T * kr_stride * 2};
  const cuuint32_t box[3] = {32, groups, 1};
  return encode_bf16_map(m, static_cast<const __nv_bfloat16*>(kr) + off * kr_stride, 3, d, st, box);
}

// The un-absorbed attention on the tensor cores: the tensor maps of q, q^R,
// k, v and the RoPE keys (row n at kr + n kr_stride), then a persistent grid.
static mtla_status launch_unabs_attn(const mtla_dims* dims, int32_t B, int32_t T, const void* q, const void* q_rope,
                                     const void* k, const void* v, const void* kr, int64_t kr_stride, void* out,
                                     float* lse, int32_t* dev_err, void* stream) {
  const int H = dims->H, s = dims->s;
  const int64_t BT = (int64_t)B * T;
  UnabsTcLaunch a;
  if (!map_head_rows(&a.q, q, H, BT, 128) || !map_head_rows(&a.k_own, k, H, BT, 128) ||
      !map_head_rows(&a.v_own, v, H, BT, 128) || !map_head_rope(&a.qr, q_rope, H, BT, 128) ||
      !map_key_rope(&a.kr_own, kr, kr_stride, BT, 128) || !map_group_rows(&a.k_grp, k, H, s, T, B, 64) ||
      !map_group_rows(&a.v_grp, v, H, s, T, B, 64) || !map_group_key_rope(&a.kr_grp, kr, kr_stride, s, T, B, 64))
    return MTLA_ERR_CUDA;
  a.B = B;
  a.T = T;
  a.H = H;
  a.s = s;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)dims->d_h));
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.dev_err = dev_err;
  const int64_t tiles = (int64_t)B * H * ((T + 127) / 128);
  const int sms = device_sms();
  if (sms <= 0) return MTLA_ERR_CUDA;
  const int grid = (int)(tiles < sms ? tiles : sms);
  return from_cuda(launch_prefill_unabs_tc(a, grid, static_cast<cudaStream_t>(stream)));
}

mtla_status mtla_prefill_kv(const mtla_dims* dims, int32_t B, int32_t T, const void* c_partial, const void* W_kv,
                            void* k, void* v, int32_t* dev_err, void* stream) {
  mtla_status st = check_dims(dims);
  if (st != MTLA_OK) return st;
  if (!unabs_dims(dims)) return MTLA_ERR_UNSUPPORTED;
  if (B < 0 || T < 0) return MTLA_ERR_INVALID_ARG;
  const void* ptrs[] = {c_partial, W_kv, k, v};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return MTLA_ERR_INVALID_ARG;
  if (!dev_err) return MTLA_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return MTLA_OK;
  const int64_t R = (int64_t)B * T, D = dims->r + dims->d_R;
  if (R >= (int64_t(1) << 31)) return MTLA_ERR_UNSUPPORTED;
  const int N = 2 * dims->H * dims->d_h;
  CUtensorMap amap, bmap;
  {
    const cuuint64_t d2[2] = {(cuuint64_t)dims->r, (cuuint64_t)R}, str[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, 128};
    if (!encode_bf16_map(&amap, c_partial, 2, d2, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MTLA_ERR_CUDA;
  }
  if (!encode_weight_map(&bmap, W_kv, N, dims->r)) return MTLA_ERR_CUDA;
  RowsGemmArgs a;
  a.R = R;
  a.N = N;
  a.nkb = dims->r / 64;
  a.k = static_cast<__nv_bfloat16*>(k);
  a.v = static_cast<__nv_bfloat16*>(v);
  a.dev_err = dev_err;
  return from_cuda(launch_rows_gemm(a, amap, bmap, static_cast<cudaStream_t>(stream)));
}

mtla_status mtla_prefill_unabsorbed_attn(const mtla_dims* dims, int32_t B, int32_t T, const void* q,
                                         const void* q_rope, const void* k, const void* v, const void* c_partial,
                                         void* out, int32_t* dev_err, void* stream) {
  mtla_status st = check_dims(dims);
  if (st != MTLA_OK) return st;
  if (!unabs_dims(dims)) return MTLA_ERR_UNSUPPORTED;
  if (B < 0 || T < 0) return MTLA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, q_rope, k, v, c_partial, out};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return MTLA_ERR_INVALID_ARG;
  if (!dev_err) return MTLA_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return MTLA_OK;
  if ((int64_t)B * T * dims->H >= (int64_t(1) << 31)) return MTLA_ERR_UNSUPPORTED;
  return launch_unabs_attn(dims, B, T, q, q_rope, k, v, static_cast<const __nv_bfloat16*>(c_partial) + dims->r,
                           dims->r + dims->d_R, out, nullptr, dev_err, stream);
}

size_t mtla_project_workspace_bytes(const mtla_dims* dims, int32_t B, int32_t d, int32_t which) {
  if (which != MTLA_PROJ_IN && which != MTLA_PROJ_OUT) return 0;
  return proj_ws(dims, B < MAXBP || (dims && dims->dtype != MTLA_BF16) ? B : MAXBP, d, which);
}

mtla_status mtla_project_in(const mtla_dims* dims, int32_t B, int32_t d, const void* x, const void* W_in,
                            const int32_t* pos, void* q_abs, void* q_rope, void* c_new, void* kR_new,
                            void* workspace, size_t workspace_bytes, int32_t* dev_err, void* stream) {
  mtla_status st = check_dims(dims);
  if (st != MTLA_OK) return st;
  if (B < 0 || d < 1) return MTLA_ERR_INVALID_ARG;
  const void* ptrs[] = {x, W_in, q_abs, q_rope, c_new, kR_new};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return MTLA_ERR_INVALID_ARG;
  if (!pos || (reinterpret_cast<uintptr_t>(pos) & 3) || !dev_err) return MTLA_ERR_INVALID_ARG;
  const bool bf = dims->dtype == MTLA_BF16;
  if (bf ? (d % 64) : (d % 4)) return MTLA_ERR_UNSUPPORTED;
  if (B == 0) return MTLA_OK;
  const int64_t N = proj_in_rows(dims);
  const int sms = device_sms();
  if (sms <= 0) return MTLA_ERR_CUDA;
  if (!workspace || !aligned16(workspace) || workspace_bytes < mtla_project_workspace_bytes(dims, B, d, MTLA_PROJ_IN))
    return MTLA_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const size_t es = elem_size(dims->dtype);
  float* part = static_cast<float*>(workspace);
  CUtensorMap wmap;
  if (bf && !encode_weight_map(&wmap, W_in, N, d)) return MTLA_ERR_CUDA;
  const int chunk = bf ? MAXBP : B;
  for (int b0 = 0; b0 < B; b0 += chunk) {
    const int nb = B - b0 < chunk ? B - b0 : chunk;
    InFinishArgs f;
    f.part = part;
    f.B = nb;
    f.H = dims->H;
    f.r = dims->r;
    f.d_R = dims->d_R;
    f.pos = pos + b0;
    f.q_abs = static_cast<uint8_t*>(q_abs) + (size_t)b0 * dims->H * dims->r * es;
    f.q_rope = static_cast<uint8_t*>(q_rope) + (size_t)b0 * dims->H * dims->d_R * es;
    f.c_new = static_cast<uint8_t*>(c_new) + (size_t)b0 * dims->r * es;
    f.kR_new = static_cast<uint8_t*>(kR_new) + (size_t)b0 * dims->d_R * es;
    cudaError_t e;
    if (bf) {
      const ProjSplit sp = proj_split(nb, d, (int)N, sms);
      GemmArgs g;
      g.x = static_cast<const uint8_t*>(x) + (size_t)b0 * d * es;
      g.ldx = d;
      g.B = nb;
      g.Bp = sp.Bp;
      g.N = (int)N;
      g.nkb = sp.nkb;
      g.kpb = sp.kpb;
      g.part = part;
      g.dev_err = dev_err;
      e = launch_proj_gemm(g, wmap, sp.m_tiles, sp.KS, false, cs);
      f.KS = sp.KS;
      f.Bp = sp.Bp;
    } else {
      e = launch_proj_simt(static_cast<const float*>(x) + (size_t)b0 * d, d, static_cast<const float*>(W_in), nb, d,
                           (int)N, part, cs);
      f.KS = 1;
      f.Bp = nb;
    }
    if (e != cudaSuccess) return MTLA_ERR_CUDA;
    if ((e = launch_proj_in_finish(f, dims->dtype, cs)) != cudaSuccess) return MTLA_ERR_CUDA;
  }
  return MTLA_OK;
}

mtla_status mtla_project_out(const mtla_dims* dims, int32_t B, int32_t d, const float* o, const void* W_out,
                             float* y, void* workspace, size_t workspace_bytes, int32_t* dev_err, void* stream) {
  mtla_status st = check_dims(dims);
  if (st != MTLA_OK) return st;
  if (B < 0 || d < 1) return MTLA_ERR_INVALID_ARG;
  const void* ptrs[] = {o, W_out, y};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return MTLA_ERR_INVALID_ARG;
  if (!dev_err) return MTLA_ERR_INVALID_ARG;
  const bool bf = dims->dtype == MTLA_BF16;
  const int64_t K = (int64_t)dims->H * dims->r;
  if (bf ? (K % 64) : (K % 4)) return MTLA_ERR_UNSUPPORTED;
  if (B == 0) return MTLA_OK;
  const int sms = device_sms();
  if (sms <= 0) return MTLA_ERR_CUDA;
  if (!workspace || !aligned16(workspace) || workspace_bytes < mtla_project_workspace_bytes(dims, B, d, MTLA_PROJ_OUT))
    return MTLA_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  float* part = static_cast<float*>(workspace);
  CUtensorMap wmap;
  if (bf && !encode_weight_map(&wmap, W_out, d, K)) return MTLA_ERR_CUDA;
  const int chunk = bf ? MAXBP : B;
  for (int b0 = 0; b0 < B; b0 += chunk) {
    const int nb = B - b0 < chunk ? B - b0 : chunk;
    cudaError_t e;
    int KS = 1, Bp = nb;
    if (bf) {
      const ProjSplit sp = proj_split(nb, (int)K, d, sms);
      GemmArgs g;
      g.x = o + (size_t)b0 * K;
      g.ldx = K;
      g.B = nb;
      g.Bp = sp.Bp;
      g.N = d;
      g.nkb = sp.nkb;
      g.kpb = sp.kpb;
      g.part = part;
      g.dev_err = dev_err;
      e = launch_proj_gemm(g, wmap, sp.m_tiles, sp.KS, true, cs);
      KS = sp.KS;
      Bp = sp.Bp;
    } else {
      e = launch_proj_simt(o + (size_t)b0 * K, K, static_cast<const float*>(W_out), nb, (int)K, d, part, cs);
    }
    if (e != cudaSuccess) return MTLA_ERR_CUDA;
    if ((e = launch_proj_out_finish(part, KS, Bp, nb, d, y + (size_t)b0 * d, cs)) != cudaSuccess)
      return MTLA_ERR_CUDA;
  }
  return MTLA_OK;
}


// ---------------------------------------------------------------------------
// training path: the uncompressed-RoPE-key shortcut and its backward pass

static bool train_dims(const mtla_dims* d) {
  return d->dtype == MTLA_BF16 && d->d_h == 64 && d->d_R == 32 && d->r == 256;
}

static size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

struct MergeBwdLayout {
  int64_t BT;
  int J, splits, kb_per;
  size_t wc, G, dg, dbp, dbs, dwp, total;
};

static MergeBwdLayout merge_bwd_layout(const mtla_dims* d, int32_t B, int32_t T) {
  MergeBwdLayout L = {};
  const int64_t r = d->r;
  L.BT = (int64_t)B * T;
  L.J = (int)((T + d->s - 1) / d->s);
  const int64_t nkb = (L.BT + 63) / 64;  // K blocks of the dW_c GEMM (K = the tokens)
  int sms = device_sms();
  if (sms < 2) sms = 2;
  const int64_t want = sms / 2;  // two 128-row tiles of dW_c per K slice: one wave
  L.kb_per = (int)((nkb + (want < nkb ? want : nkb) - 1) / (want < nkb ? want : nkb));
  L.splits = (int)((nkb + L.kb_per - 1) / L.kb_per);
  size_t o = 0;
  L.wc = o;  o = up256(o + (size_t)r * r * 2);
  L.G = o;   o = up256(o + (size_t)L.BT * r * 4);
  L.dg = o;  o = up256(o + (size_t)L.BT * r * 2);
  L.dbp = o; o = up256(o + (size_t)L.J * r * 4);
  L.dbs = o; o = up256(o + (size_t)DB_SLICE_COUNT * r * 4);
  L.dwp = o; o = up256(o + (size_t)L.splits * r * r * 4);
  L.total = o;
  return L;
}

// lse2 and Delta [B, H, Tp] (Tp = T rounded up to 64), then the per-head RoPE
// key gradients [B, T, H, d_R]
static size_t attn_bwd_bytes(const mtla_dims* d, int32_t B, int32_t T, size_t* off_delta, size_t* off_dkrh) {
  const size_t Tp = ((size_t)T + 63) / 64 * 64;
  const size_t a = up256((size_t)B * d->H * Tp * 4);
  if (off_delta) *off_delta = a;
  if (off_dkrh) *off_dkrh = 2 * a;
  return 2 * a + up256((size_t)B * T * d->H * 32 * 4);
}

size_t mtla_train_workspace_bytes(const mtla_dims* dims, int32_t B, int32_t T, int32_t which) {
  if (check_dims(dims) != MTLA_OK || !train_dims(dims) || B < 1 || T < 1) return 0;
  if (which == MTLA_TRAIN_ATTN_BWD) return attn_bwd_bytes(dims, B, T, nullptr, nullptr);
  if (which == MTLA_TRAIN_KV_BWD) return 0;  // no workspace: W_kv is read as stored
  if (which == MTLA_TRAIN_MERGE_BWD) return merge_bwd_layout(dims, B, T).total;
  return 0;
}

mtla_status mtla_train_attn_fwd(const mtla_dims* dims, int32_t B, int32_t T, const void* q, const void* q_rope,
                                const void* k, const void* v, const void* kR, void* out, float* lse,
                                int32_t* dev_err, void* stream) {
  mtla_status st = check_dims(dims);
  if (st != MTLA_OK) return st;
  if (!unabs_dims(dims)) return MTLA_ERR_UNSUPPORTED;
  if (B < 0 || T < 0) return MTLA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, q_rope, k, v, kR, out, lse};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return MTLA_ERR_INVALID_ARG;
  if (!dev_err) return MTLA_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return MTLA_OK;
  if ((int64_t)B * T * dims->H >= (int64_t(1) << 31)) return MTLA_ERR_UNSUPPORTED;
  return launch_unabs_attn(dims, B, T, q, q_rope, k, v, kR, dims->d_R, out, lse, dev_err, stream);
}

mtla_status mtla_train_attn_bwd(const mtla_dims* dims, int32_t B, int32_t T, const void* q, const void* q_rope,
                                const void* k, const void* v, const void* kR, const void* out, const float* lse,
                                const void* d_out, void* dq, void* dq_rope, void* dk, void* dv, float* dkR,
                                void* workspace, size_t workspace_bytes, int32_t* dev_err, void* stream) {
  mtla_status st = check_dims(dims);
  if (st != MTLA_OK) return st;
  if (!train_dims(dims)) return MTLA_ERR_UNSUPPORTED;
  if (B < 0 || T < 0) return MTLA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, q_rope, k, v, kR, out, lse, d_out, dq, dq_rope, dk, dv, dkR};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return MTLA_ERR_INVALID_ARG;
  if (!dev_err) return MTLA_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return MTLA_OK;
  if ((int64_t)B * T * dims->H * 32 >= (int64_t(1) << 31)) return MTLA_ERR_UNSUPPORTED;
  size_t off_delta = 0, off_dkrh = 0;
  const size_t need = attn_bwd_bytes(dims, B, T, &off_delta, &off_dkrh);
  if (!workspace || !aligned16(workspace) || workspace_bytes < need) return MTLA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  BwdArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.qr = static_cast<const __nv_bfloat16*>(q_rope);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.kr = static_cast<const __nv_bfloat16*>(kR);
  a.o = static_cast<const __nv_bfloat16*>(out);
  a.dout = static_cast<const __nv_bfloat16*>(d_out);
  a.lse = lse;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dqr = static_cast<__nv_bfloat16*>(dq_rope);
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.dkr = dkR;
  a.ws_lse2 = reinterpret_cast<float*>(ws);
  a.ws_delta = reinterpret_cast<float*>(ws + off_delta);
  a.ws_dkrh = reinterpret_cast<float*>(ws + off_dkrh);
  a.B = B;
  a.T = T;
  a.H = dims->H;
  a.s = dims->s;
  a.Tp = (T + 63) / 64 * 64;
  a.scale = (float)(1.0 / sqrt((double)dims->d_h));
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)dims->d_h));
  const int H = dims->H, s = dims->s;
  const int64_t BT = (int64_t)B * T;
  TrainBwdMaps mq;
  TrainBwdKvMaps mk;
  if (!map_head_rows(&mq.q128, q, H, BT, 128) || !map_head_rope(&mq.qr128, q_rope, H, BT, 128) ||
      !map_head_rows(&mq.do128, d_out, H, BT, 128) || !map_head_rows(&mq.k128, k, H, BT, 128) ||
      !map_key_rope(&mq.kr128, kR, dims->d_R, BT, 128) || !map_head_rows(&mq.v128, v, H, BT, 128) ||
      !map_group_rows(&mq.k_g64, k, H, s, T, B, 64) || !map_group_key_rope(&mq.kr_g64, kR, dims->d_R, s, T, B, 64) ||
      !map_group_rows(&mq.v_g64, v, H, s, T, B, 64))
    return MTLA_ERR_CUDA;
  if (!map_group_rows(&mk.k_g, k, H, s, T, B, 128) || !map_group_key_rope(&mk.kr_g, kR, dims->d_R, s, T, B, 128) ||
      !map_group_rows(&mk.v_g, v, H, s, T, B, 128) || !map_group_rows(&mk.q_g, q, H, s, T, B, 128) ||
      !map_group_rope(&mk.qr_g, q_rope, H, s, T, B, 128) || !map_group_rows(&mk.do_g, d_out, H, s, T, B, 128) ||
      !map_head_rows(&mk.q64, q, H, BT, 64) || !map_head_rope(&mk.qr64, q_rope, H, BT, 64) ||
      !map_head_rows(&mk.do64, d_out, H, BT, 64))
    return MTLA_ERR_CUDA;
  TrainBwdTc t;
  t.B = B;
  t.T = T;
  t.H = H;
  t.s = s;
  t.Tp = a.Tp;
  t.scale = a.scale;
  t.scale_log2 = a.scale_log2;
  t.lse2 = a.ws_lse2;
  t.delta = a.ws_delta;
  t.dq = a.dq;
  t.dqr = a.dqr;
  t.dk = a.dk;
  t.dv = a.dv;
  t.dkrh = a.ws_dkrh;
  t.dev_err = dev_err;
  const int sms = device_sms();
  if (sms <= 0) return MTLA_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (launch_bwd_prep(a, cs) != cudaSuccess) return MTLA_ERR_CUDA;
  const int64_t q_tiles = (int64_t)B * H * ((T + 127) / 128);
  if (launch_bwd_dq_tc(mq, t, (int)(q_tiles < sms ? q_tiles : sms), cs) != cudaSuccess) return MTLA_ERR_CUDA;
  const int64_t items = (int64_t)B * H * ((T / s + 127) / 128);
  if (items > 0 && launch_bwd_dkv_tc(mk, t, (int)(items < sms ? items : sms), cs) != cudaSuccess) return MTLA_ERR_CUDA;
  return from_cuda(launch_dkr_reduce(a, cs));
}

// 2-D map of a row-major bf16 matrix [rows, cols] (row stride ld elements) in
// boxes of 64 columns x 128 rows with the 128-byte swizzle: a K-major GEMM operand
static bool encode_operand_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld) {
  const cuuint64_t d2[2] = {(cuuint64_t)cols, (cuuint64_t)rows}, str[1] = {(cuuint64_t)ld * 2};
  const cuuint32_t box[2] = {64, 128};
  return encode_bf16_map(map, base, 2, d2, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}
// The same matrix as an MN-major operand whose K runs along the rows: boxes of
// 64 columns x 64 rows with the 128-byte swizzle
static bool encode_mn_operand_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld) {
  const cuuint64_t d2[2] = {(cuuint64_t)cols, (cuuint64_t)rows}, str[1] = {(cuuint64_t)ld * 2};
  const cuuint32_t box[2] = {64, 64};
  return encode_bf16_map(map, base, 2, d2, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

mtla_status mtla_train_kv_bwd(const mtla_dims* dims, int32_t B, int32_t T, const void* dk, const void* dv,
                              const void* W_kv, float* dC, void* workspace, size_t workspace_bytes,
                              int32_t* dev_err, void* stream) {
  mtla_status st = check_dims(dims);
  if (st != MTLA_OK) return st;
  if (!train_dims(dims)) return MTLA_ERR_UNSUPPORTED;
  if (B < 0 || T < 0) return MTLA_ERR_INVALID_ARG;
  const void* ptrs[] = {dk, dv, W_kv, dC};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return MTLA_ERR_INVALID_ARG;
  if (!dev_err) return MTLA_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return MTLA_OK;
  const int64_t BT = (int64_t)B * T;
  if (BT >= (int64_t(1) << 31)) return MTLA_ERR_UNSUPPORTED;
  const int r = dims->r, Hd = dims->H * dims->d_h;
  (void)workspace;
  (void)workspace_bytes;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // W_kv [2 H d_h, r] as stored is the MN-major B of dC = [dk | dv] W_kv
  CUtensorMap a0, a1, bm;
  if (!encode_operand_map(&a0, dk, BT, Hd, Hd) || !encode_operand_map(&a1, dv, BT, Hd, Hd) ||
      !encode_mn_operand_map(&bm, W_kv, 2 * Hd, r, r))
    return MTLA_ERR_CUDA;
  GemmBtArgs g;
  g.M = BT;
  g.N = r;
  g.K = 2 * Hd;
  g.ka_split = Hd;
  g.kb_per_split = (2 * Hd + 63) / 64;
  g.C = dC;
  g.ldc = r;
  g.split_stride = 0;
  g.accumulate = 0;
  g.a_mn = 0;
  g.b_mn = 1;
  g.dev_err = dev_err;
  return from_cuda(launch_gemm_bt(g, a0, a1, bm, 1, cs));
}

mtla_status mtla_train_merge_bwd(const mtla_dims* dims, int32_t B, int32_t T, const void* c, const float* W_c,
                                 const float* b_c, const float* P, int32_t J_max, const float* dC, float* dc,
                                 float* dW_c, float* db_c, float* dP, void* workspace, size_t workspace_bytes,
                                 int32_t* dev_err, void* stream) {
  mtla_status st = check_dims(dims);
  if (st != MTLA_OK) return st;
  if (!train_dims(dims)) return MTLA_ERR_UNSUPPORTED;
  if (B < 0 || T < 0 || J_max < 0) return MTLA_ERR_INVALID_ARG;
  const void* ptrs[] = {c, W_c, b_c, P, dC, dc, dW_c, db_c, dP};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return MTLA_ERR_INVALID_ARG;
  if (!dev_err) return MTLA_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return MTLA_OK;
  const int r = dims->r, D = dims->r + dims->d_R;
  if ((int64_t)J_max < (T + (int64_t)dims->s - 1) / dims->s) return MTLA_ERR_INVALID_ARG;
  if ((int64_t)B * T * r >= (int64_t(1) << 31) || (int64_t)J_max * D >= (int64_t(1) << 31))
    return MTLA_ERR_UNSUPPORTED;
  const MergeBwdLayout L = merge_bwd_layout(dims, B, T);
  if (!workspace || !aligned16(workspace) || workspace_bytes < L.total) return MTLA_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  __nv_bfloat16* wc = reinterpret_cast<__nv_bfloat16*>(ws + L.wc);    // [i][k] = W_c[i][k], k < r
  float* G = reinterpret_cast<float*>(ws + L.G);
  __nv_bfloat16* dg = reinterpret_cast<__nv_bfloat16*>(ws + L.dg);
  float* dbp = reinterpret_cast<float*>(ws + L.dbp);
  float* dwp = reinterpret_cast<float*>(ws + L.dwp);
  const __nv_bfloat16* cb = static_cast<const __nv_bfloat16*>(c);
  cudaError_t e;
  if ((e = launch_convert_bf16(W_c, r, r, D, wc, r, cs)) != cudaSuccess) return MTLA_ERR_CUDA;
  // wc [i][k] is K-major for dc += dg W_c^T (K = k) and MN-major for G = c W_c (K = i)
  CUtensorMap mc, mwcm, mwc, mdg, mcm, mdgm;
  if (!encode_operand_map(&mc, cb, L.BT, r, r) || !encode_mn_operand_map(&mwcm, wc, r, r, r) ||
      !encode_operand_map(&mwc, wc, r, r, r) || !encode_operand_map(&mdg, dg, L.BT, r, r) ||
      !encode_mn_operand_map(&mcm, cb, L.BT, r, r) || !encode_mn_operand_map(&mdgm, dg, L.BT, r, r))
    return MTLA_ERR_CUDA;
  GemmBtArgs g;
  g.N = r;
  g.dev_err = dev_err;
  g.split_stride = 0;
  g.a_mn = 0;
  g.b_mn = 0;
  // G = c W_c[:, :r]: the gate pre-activations without the bias
  g.M = L.BT;
  g.K = r;
  g.ka_split = r;
  g.kb_per_split = r / 64;
  g.C = G;
  g.ldc = r;
  g.accumulate = 0;
  g.b_mn = 1;
  if ((e = launch_gemm_bt(g, mc, mc, mwcm, 1, cs)) != cudaSuccess) return MTLA_ERR_CUDA;
  g.b_mn = 0;
  MergeBwdArgs m;
  m.c = cb;
  m.G = G;
  m.b_c = b_c;
  m.P = P;
  m.dC = dC;
  m.dc = dc;
  m.dg = dg;
  m.dP = dP;
  m.db_part = dbp;
  m.B = B;
  m.T = T;
  m.r = r;
  m.D = D;
  m.s = dims->s;
  m.J_max = J_max;
  if ((e = launch_merge_bwd(m, cs)) != cudaSuccess) return MTLA_ERR_CUDA;
  // dc += dg W_c[:, :r]^T
  g.C = dc;
  g.accumulate = 1;
  if ((e = launch_gemm_bt(g, mdg, mdg, mwc, 1, cs)) != cudaSuccess) return MTLA_ERR_CUDA;
  // dW_c[:, :r] = c^T dg: a contraction over the tokens, the rows of both
  // c and dg (MN-major operands, no transposed copies), split over the
  // tokens, then the slices summed
  g.M = r;
  g.K = (int)L.BT;
  g.ka_split = (int)L.BT;
  g.kb_per_split = L.kb_per;
  g.C = dwp;
  g.ldc = r;
  g.split_stride = (int64_t)r * r;
  g.accumulate = 0;
  g.a_mn = 1;
  g.b_mn = 1;
  if ((e = launch_gemm_bt(g, mcm, mcm, mdgm, L.splits, cs)) != cudaSuccess) return MTLA_ERR_CUDA;
  if ((e = launch_sum_slices(dwp, r, r, D, L.splits, (int64_t)r * r, dW_c, cs)) != cudaSuccess) return MTLA_ERR_CUDA;
  return from_cuda(launch_db_reduce(dbp, L.J, r, D, reinterpret_cast<float*>(ws + L.dbs), db_c, cs));
}

}  // extern "C"
