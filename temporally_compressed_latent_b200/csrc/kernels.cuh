// Argument blocks and launchers shared by the MTLA kernels and the C ABI.
#pragma once

#include "mtla_common.cuh"

namespace mtla {

// Cache and per-sequence state (device pointers).
struct SeqArgs {
  void* cache;
  int64_t cache_rows;
  int64_t row_stride;  // elements
  const int64_t* seq_offset;
  const int64_t* seq_capacity;
  int32_t* t_processed;
  int32_t* cache_len;
  int32_t* dev_err;
  int r, d_R, s;
};

// Hyper-network merge inputs of one new token per sequence.
struct MergeArgsDev {
  const void* c_new;
  const void* kR_new;
  const float* W_c;
  const float* b_c;
  const float* P;
  int32_t J_max;
};

struct DecodeOut {
  const void* q_abs;
  const void* q_rope;
  float* out;
  float* lse;
  float scale;  // 1/sqrt(d_h)
  int H;
  const void* tails;  // nullable [B][D]: replaces every sequence's last row (several tokens per call)
};

struct PrefillArgs {
  const void* q_abs;
  const void* q_rope;
  const void* c;
  const void* kR;
  const float* W_c;
  const float* b_c;
  const float* P;
  void* c_partial;
  void* cache_out;
  void* out;
  int32_t* dev_err;
  int64_t T;
  int64_t groups_per_block;
  int H, r, d_R, s;
  float scale;
  int32_t J_max;
};

// Split-L tensor-core decode (bf16, H = 8, r = 256, d_R = 32).
namespace dtc {
constexpr int H = 8, R = 256, DR = 32, D = R + DR;
constexpr int UNIT = 64;                 // rows per full TMA box
constexpr int SUB = 8;                   // rows per box of a ragged last unit
constexpr int ROWB = D * 2;              // bytes per cache row (576)
constexpr int STAGE = UNIT * ROWB;       // 36864 bytes per pipeline stage
constexpr int NS = 2;                    // pipeline depth per block (two blocks per SM)
constexpr int NCW = 4;                   // consumer warps
constexpr int PRODUCER_WARP = NCW;       // streams the tiles
constexpr int NT = 32 * (NCW + 1);
constexpr int SEGB = UNIT * 64;          // bytes of one 32-element plane of a tile (4096)
constexpr int MAXB = 1024;               // sequences per call
constexpr int MAXG = 320;                // blocks per launch
constexpr int OSTR = 260;                // head stride of the combine buffer (floats)
constexpr int MERGE_COST = 128;          // partition weight of one merged sequence, in rows: its tail owner's extra work (merge wait, tail patch, segment ends); 128 measured best of 32-256

struct Params {
  SeqArgs a;
  MergeArgsDev m;
  DecodeOut o;
  int with_merge;
  int patch;            // 1: every sequence's last row is taken from tails (several tokens per call)
  int B;
  int merge_cost;
  float scale_log2;     // log2(e) / sqrt(d_h)
  int4* seq_info;       // [B] {rows, merge ok, first part slot, part count} for the combine
  __nv_bfloat16* tails; // [B][D] updated tail row of every merged sequence (merge kernel)
  float* ws_ml;         // [2 * grid][H][2]
  float* ws_o;          // [2 * grid][H][R]
};

size_t smem_bytes();
// Byte offsets of the workspace regions (each on a 256-byte boundary) and its
// size: one layout for the size query and for the pointers a call carves.
struct WsLayout {
  size_t seq_info, tails, ml, o, total;
};
WsLayout ws_layout(int B, int grid);
size_t workspace_bytes(int B, int grid);
int grid_size();  // blocks of the persistent grid on the current device (0 on error)
}  // namespace dtc

cudaError_t launch_merge_append(const SeqArgs& a, const MergeArgsDev& m, int B, int dtype, cudaStream_t st);
cudaError_t launch_decode_simt(const SeqArgs& a, const MergeArgsDev& m, bool with_merge, const DecodeOut& o,
                               int B, int dtype, cudaStream_t st);
cudaError_t launch_decode_tc(const dtc::Params& p, const CUtensorMap& map64, const CUtensorMap& map8, int grid,
                             cudaStream_t st);
cudaError_t launch_partial_merge(const PrefillArgs& p, int B, int dtype, cudaStream_t st);

// Running merge on tcgen05 (merge_tc.cu): the tensor maps it reads and writes
// (latents, RoPE keys, P rows; C_hat' and the cache rows).
struct MergeMaps {
  CUtensorMap c, kr, p, out, cache;
};
cudaError_t launch_merge_tc(const PrefillArgs& a, int B, const MergeMaps& m, int sms, cudaStream_t st);

// Masked prefill on tcgen05 (bf16, H = 8, r = 256, d_R = 32, any T >= 1).
namespace ptc {
struct Params;
size_t smem_bytes();
}
struct PrefillTcLaunch {
  int B, T, s;
  float scale_log2;
  void* out;
  int32_t* dev_err;
};
cudaError_t launch_prefill_tc_args(const PrefillTcLaunch& a, const CUtensorMap& qmap, const CUtensorMap& rmap,
                                   const CUtensorMap& smap, const CUtensorMap& kmap, int grid, cudaStream_t st);
cudaError_t launch_prefill_simt(const PrefillArgs& p, int B, int dtype, cudaStream_t st);

// Several new tokens per sequence in one decode call (multi.cu): the merge of
// the n tokens in order, the tail row as it stands after each token, and the
// per-query ("virtual") sequence arrays the attention kernels read.
struct MultiMergeArgs {
  SeqArgs a;          // the real sequences (B of them)
  MergeArgsDev m;     // c_new [B, n, r], kR_new [B, n, d_R]
  int n;
  int four_part;      // gate sums in four 64-row parts (the tensor-core decode's merge order)
  void* tails;        // [B n][D] cache dtype: the tail row after token i of sequence b
  float* gates;       // [B n][D] fp32: the tokens' gate pre-activations c_t W_c + b_c
  int32_t* t_v;       // [B n] tokens processed after query i's token
  int64_t* off_v;     // [B n]
  int64_t* cap_v;     // [B n]
};
cudaError_t launch_multi_merge(const MultiMergeArgs& a, int B, int dtype, cudaStream_t st);

// The layer's input and output maps with the key / value maps absorbed (proj.cu).
constexpr int MAXBP = 256;  // tokens per projection launch (MMA N)
struct GemmArgs {
  const void* x;   // [B, K] activations (bf16, or fp32 rounded to bf16 when staged)
  int64_t ldx;     // elements between rows of x
  int B, Bp, N, nkb, kpb;
  float* part;     // [KS][Bp][N] fp32 partial sums
  int32_t* dev_err;
};
struct InFinishArgs {
  const float* part;
  int KS, Bp, B, H, r, d_R;
  const int32_t* pos;  // [B] 0-based token positions (RoPE)
  void* q_abs;
  void* q_rope;
  void* c_new;
  void* kR_new;
};
struct ProjSplit {
  int Bp, KS, kpb, m_tiles, nkb;
};
ProjSplit proj_split(int B, int K, int N, int sms);
size_t proj_smem_bytes();
cudaError_t launch_proj_gemm(const GemmArgs& a, const CUtensorMap& wmap, int m_tiles, int KS, bool x_f32,
                             cudaStream_t st);
cudaError_t launch_proj_simt(const float* x, int64_t ldx, const float* W, int B, int K, int N, float* part,
                             cudaStream_t st);
cudaError_t launch_proj_in_finish(const InFinishArgs& a, int dtype, cudaStream_t st);
cudaError_t launch_proj_out_finish(const float* part, int KS, int Bp, int B, int N, float* y, cudaStream_t st);

// Per-head keys and values of a prompt for the un-absorbed forward (proj.cu):
// [k | v] [R x N] = C [R x Kd] W^T, R = B T rows, N = 2 H d_h (a multiple of
// 256), Kd = r <= 256 (a multiple of 64).
struct RowsGemmArgs {
  int64_t R;
  int N, nkb;
  __nv_bfloat16* k;  // [R, N / 2]
  __nv_bfloat16* v;  // [R, N / 2]
  int32_t* dev_err;
};
cudaError_t launch_rows_gemm(const RowsGemmArgs& a, const CUtensorMap& amap, const CUtensorMap& bmap,
                             cudaStream_t st);

// Masked attention with explicit per-head keys and values (the un-absorbed
// prefill, and the training shortcut's forward) on the tensor cores (tcgen05
// + TMEM): tensor maps of the inputs (bf16, 64-byte swizzle, 32-element
// boxes) and the sizes.  The RoPE keys are the last d_R channels of C_hat'
// (row stride D) or the uncompressed K^R (row stride d_R).
struct UnabsTcLaunch {
  CUtensorMap q, qr;          // q: 4-D {32, H, B T, 2 planes}, box {32, 1, 128, 2}; q^R: 3-D {32, H, B T}, box {32, 1, 128}
  CUtensorMap k_own, v_own;   // like q, on k and v
  CUtensorMap kr_own;         // 2-D {32, B T}, box {32, 128}
  CUtensorMap k_grp, v_grp;   // 5-D {32, H, T / s groups, B, 2 planes} from row s - 1, box {32, 1, 64, 1, 2}
  CUtensorMap kr_grp;         // 3-D {32, T / s groups, B} from row s - 1, box {32, 64, 1}
  int B, T, H, s;
  float scale_log2;
  __nv_bfloat16* out;
  float* lse;
  int32_t* dev_err;
};
size_t prefill_unabs_tc_smem();
cudaError_t launch_prefill_unabs_tc(const UnabsTcLaunch& a, int grid, cudaStream_t st);

// Backward of the masked attention with explicit keys and values and the
// uncompressed RoPE keys (training shortcut): bf16, d_h = 64, d_R = 32.
struct BwdArgs {
  const __nv_bfloat16 *q, *qr, *k, *v, *kr;  // [B,T,H,64], [B,T,H,32], [B,T,H,64] x 2, [B,T,32]
  const __nv_bfloat16 *o, *dout;             // [B,T,H,64]
  const float* lse;                          // [B,T,H] natural log
  __nv_bfloat16 *dq, *dqr, *dk, *dv;         // like q, qr, k, v
  float* dkr;                                // [B,T,32], summed over heads
  float* ws_lse2;                            // [B,H,Tp] lse in log2 units of the scaled score
  float* ws_delta;                           // [B,H,Tp] rowsum(dO * O)
  float* ws_dkrh;                            // [B,T,H,32] per-head RoPE key gradients
  int B, T, H, s, Tp;                        // Tp: T rounded up to 64
  float scale, scale_log2;
};
// Delta and lse2 per (sequence, head, query), then (after the gradient
// kernels) dk^R summed over heads.
cudaError_t launch_bwd_prep(const BwdArgs& a, cudaStream_t st);
cudaError_t launch_dkr_reduce(const BwdArgs& a, cudaStream_t st);

// The gradient kernels on the tensor cores (train_bwd_tc.cu).
struct TrainBwdTc {
  int B, T, H, s, Tp;
  float scale, scale_log2;
  const float *lse2, *delta;           // [B, H, Tp]
  __nv_bfloat16 *dq, *dqr, *dk, *dv;   // [B, T, H, 64] (dqr: 32)
  float* dkrh;                         // [B, T, H, 32]
  int32_t* dev_err;
};
// dq kernel: 128-query tiles and 64-column key tiles (bf16, 64-byte swizzle)
struct TrainBwdMaps {
  CUtensorMap q128, qr128, do128;   // q, dO: 4-D {32, H, B T, 2 planes} box {32, 1, 128, 2}; q^R 3-D box {32, 1, 128}
  CUtensorMap k128, kr128, v128;    // the tile's own rows: k, v like q; k^R 2-D {32, B T} box {32, 128}
  CUtensorMap k_g64, kr_g64, v_g64; // group columns: k, v 5-D {32, H, T / s, B, 2} box {32, 1, 64, 1, 2}; k^R 3-D
};
// dk / dv kernel: 128 group columns per item and 64-query tiles
struct TrainBwdKvMaps {
  CUtensorMap k_g, kr_g, v_g;       // group columns, boxes of 128
  CUtensorMap q_g, qr_g, do_g;      // the query rows at the group columns' positions (q^R: 4-D {32, H, T / s, B})
  CUtensorMap q64, qr64, do64;      // query tiles, boxes of 64 rows
};
size_t bwd_dq_tc_smem();
size_t bwd_dkv_tc_smem();
cudaError_t launch_bwd_dq_tc(const TrainBwdMaps& mp, const TrainBwdTc& p, int grid, cudaStream_t st);
cudaError_t launch_bwd_dkv_tc(const TrainBwdKvMaps& mp, const TrainBwdTc& p, int grid, cudaStream_t st);

// C[M, N] (fp32) = A[M, K] B[N, K]^T, A and B bf16 K-major through TMA
// (boxes of 64 x 128, 128-byte swizzle); A from amap0 for k < ka_split, from
// amap1 beyond; N a multiple of 256.  grid.z > 1 splits K into slices of
// kb_per_split blocks, slice z written to C + z * split_stride.
struct GemmBtArgs {
  int64_t M;
  int N, K, ka_split, kb_per_split;
  float* C;
  int64_t ldc, split_stride;
  int accumulate;  // C += A B^T (one slice only)
  // MN-major operands: A stored [K, M] (maps {M, K}, boxes of 64 x 64) and B
  // stored [K, N], so that C = A^T-as-stored B-as-stored: a contraction over
  // the rows of both (K-major: boxes of 64 K x 128 rows)
  int a_mn, b_mn;
  int32_t* dev_err;
};
cudaError_t launch_gemm_bt(const GemmBtArgs& a, const CUtensorMap& amap0, const CUtensorMap& amap1,
                           const CUtensorMap& bmap, int splits, cudaStream_t st);
size_t gemm_bt_smem_bytes();

// out[r * ld_out + c] = sum over the n slices z of src[z * stride + r * cols + c]
// (c < cols; columns cols .. ld_out - 1 written as zeros)
cudaError_t launch_sum_slices(const float* src, int64_t rows, int cols, int64_t ld_out, int n, int64_t stride,
                              float* out, cudaStream_t st);

// out[r][c] = bf16(in[r][c]), r < rows, c < cols (row strides ld_in, ld_out)
cudaError_t launch_convert_bf16(const float* in, int64_t rows, int cols, int64_t ld_in, __nv_bfloat16* out,
                                int64_t ld_out, cudaStream_t st);

// The gate part of the merge backward (latent channels, training shortcut).
struct MergeBwdArgs {
  const __nv_bfloat16* c;  // [B, T, r]
  const float* G;          // [B, T, r] c W_c[:, :r] (bias not included)
  const float *b_c, *P;    // [D], [J_max, D]
  const float* dC;         // [B, T, r]
  float* dc;               // [B, T, r] out: the direct term de * w
  __nv_bfloat16* dg;       // [B, T, r] out: gate pre-activation gradient (bf16, for the GEMMs)
  float* dP;               // [J_max, D] out (all rows and channels written)
  float* db_part;          // [ceil(T/s), r] per-group partial sums of dg
  int B, T, r, D, s, J_max;
};
cudaError_t launch_merge_bwd(const MergeBwdArgs& a, cudaStream_t st);
// db[k] = sum_j part[j][k] for k < r, zero for r <= k < D, through 64 partial
// slices [64, r] in `slices` (fixed order)
constexpr int DB_SLICE_COUNT = 64;
cudaError_t launch_db_reduce(const float* part, int J, int r, int D, float* slices, float* db, cudaStream_t st);

}  // namespace mtla
