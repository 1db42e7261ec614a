// kernels.h - internal launchers shared by the C ABI (mla_abi.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace mla {

// Keys are walked in tiles of this many rows by every attention kernel; the rotated-key
// workspace pads the ring part and the chunk part to a multiple of it.
constexpr int kKeyTile = 128;

// Strided batched GEMM  C[z](m, n) = sum_k A[z](m, k) B[z](n, k)  (element strides).
struct GemmArgs {
  const void* A;
  const void* B;
  void* C;
  int M, N, K, batch;
  int64_t a_sm, a_sk, a_batch;
  int64_t b_sn, b_sk, b_batch;
  int64_t c_sm, c_batch;
  // Optional fused 3D-RoPE of the query path: in every D-wide block of output columns, the
  // pairs of columns d_c.. D-1 are rotated (fp32, before the one rounding) at the position of
  // row m (chunk token m mod rope_n_q).  Needs even d_c.
  int rope_epi;
  int rope_D, rope_dc, rope_n_q, rope_first_frame;
  RopeGeom rope;
};

struct AttnArgs {
  const void* q;          // [B, n_q, H, D]
  const void* chunk_lat;  // [B, n_q, D]
  const void* cache;      // [B, W*tpf, D]
  const void* ws;         // rotated keys [B, rows, d_rope]
  const void* w_uv;       // [H, d_head, d_c] or null
  void* out;              // [B, n_q, H*d_head] or [B, n_q, H, d_c]
  float* lse;             // [B, H, n_q] or null
  int32_t* dev_status;    // or null
};

struct KeyWorkspace {
  int nc;       // ring keys attended (n_valid * tpf)
  int nc_pad;   // nc rounded up to kKeyTile: row of the first chunk key
  int rows;     // rows per sample
  size_t bytes; // whole workspace
};

KeyWorkspace key_workspace_layout(const Dims& d, int n_valid);

// Backward of the attention call (attention_bwd.cu).
struct BwdArgs {
  const void* q;           // [B, n_q, H, D]
  const void* chunk_lat;   // [B, n_q, D]
  const void* cache;       // [B, W*tpf, D]
  const int32_t* slot_frame;
  const void* o_lat;       // [B, n_q, H, d_c]
  const float* lse;        // [B, H, n_q]
  const void* d_o_lat;     // [B, n_q, H, d_c]
  void* d_q;               // [B, n_q, H, D]
  void* d_chunk_lat;       // [B, n_q, D]
  void* d_cache;           // [B, W*tpf, D]
};

struct BwdWorkspace {
  size_t delta_bytes;      // Delta = G . O_lat per (sample, head, row), fp32, then
  KeyWorkspace keys;       // the rotated positional keys, as in the forward, then
  int groups;              // (tensor-core path) the keys as the MMAs read them,
  size_t keys_tc_bytes;    //   [B, keys.rows, 256] bf16 (latent, rotated key, zeros), then per
  size_t partial_bytes;    //   head group the keys' fp32 partial latent gradients
  size_t bytes;            //   [groups, B, keys.rows, D]
};

BwdWorkspace bwd_workspace_layout(const Dims& d, int n_valid);
mla_status attention_bwd(const Dims& d, const BwdArgs& a, int n_valid, int first_frame,
                         void* workspace, int32_t* dev_status, cudaStream_t s);
// tensor-core backward (attention_bwd_sm100.cu)
bool tc_bwd_supported(const Dims& d);
int bwd_tc_head_groups(const Dims& d, int n_valid);
constexpr int kBwdKeyWidth = 256;   // row width of the tensor-core path's key copy
mla_status attention_bwd_tc(const Dims& d, const BwdArgs& a, int n_valid, int first_frame,
                            const float* delta, const void* ws_rope, void* keys_tc,
                            float* partial, int groups, int32_t* dev_status, cudaStream_t s);

// CUDA-core kernels (simt.cu)
mla_status gemm_simt(const GemmArgs& g, int dtype, cudaStream_t s);
mla_status rope3d_inplace(const Dims& d, void* data, int n_samples, int rows, int row_width,
                          int col_offset, int n_vec, int vec_stride, const int32_t* frame_table,
                          int frame_table_stride, int first_frame, cudaStream_t s);
mla_status ring_append(const Dims& d, const void* chunk_lat, void* cache, int32_t* slot_frame,
                       int first_frame, cudaStream_t s);
mla_status key_positions(const Dims& d, const int32_t* slot_frame, int n_valid, int first_frame,
                         int32_t* out, cudaStream_t s);
// Which rows of the rotated-key workspace build_rope_keys writes: all, the ring part (rows
// [0, nc_pad)) or the chunk part (rows [nc_pad, rows)); kRopeKeysNone tells the attention entry
// points that the workspace is complete already (written by the x-projection's epilogue).
enum RopeKeysPart : int { kRopeKeysAll = 0, kRopeKeysRing = 1, kRopeKeysChunk = 2, kRopeKeysNone = 3 };
// dev_status (optional): with MLA_DEBUG builds the kernel checks that every attended ring slot
// holds a frame (t >= 0) and, with check_window, one of the chunk's window
// (first_frame - W <= t < first_frame), writing MLA_ERR_DEVICE_CHECK there otherwise.
mla_status build_rope_keys(const Dims& d, const void* cache, const void* chunk_lat,
                           const int32_t* slot_frame, int n_valid, int first_frame, void* ws,
                           cudaStream_t s, int part = kRopeKeysAll, int32_t* dev_status = nullptr,
                           int check_window = 0);
mla_status attention_simt(const Dims& d, const AttnArgs& a, int n_valid, cudaStream_t s);
mla_status copy_rows(int dtype, const void* src, int64_t src_stride, void* dst,
                     int64_t dst_stride, int rows, int cols, int64_t src_batch,
                     int64_t dst_batch, int batch, cudaStream_t s);

// Tensor-core kernels (gemm_sm100.cu, attention_sm100.cu)

// Epilogues of the tcgen05 GEMM.
enum GemmEpilogue : int {
  kEpiStore = 0,     // C[m, n] = acc (bf16)
  kEpiRopeQ = 1,     // as kEpiStore, and 3D-RoPE on the last rope_dr columns of every
                     // rope_D-wide head block of the output row (query path)
};

struct TcGemmArgs {
  // A: [batch][M, K] rows with element stride a_sm, batch stride a_batch; K contiguous.
  const void* A;
  int64_t a_sm, a_batch;
  // B: [batch][N, K], K contiguous.
  const void* B;
  int64_t b_sn, b_batch;
  // C: [batch][M, N] bf16, row stride c_sm, batch stride c_batch; N contiguous.
  void* C;
  int64_t c_sm, c_batch;
  // Optional second output: when n_split > 0 (a multiple of 32, < N), columns n >= n_split go
  // to C2 at column n - n_split (row stride c2_sm, batch stride c2_batch) instead of C.
  void* C2;
  int64_t c2_sm, c2_batch;
  int n_split;
  int M, N, K, batch;
  int epilogue;
  // kEpiRopeQ: rows are chunk tokens of samples of n_q rows; head blocks of width rope_D whose
  // last rope_dr columns are rotated.
  int rope_D, rope_dr, rope_n_q, rope_first_frame;
  RopeGeom rope;
  // Optional ring append from the epilogue (batch 1, n_split 0): row m = chunk token
  // (sample m / ring_n_q, frame j, token i) is also stored to ring row
  // ((ring_first + j) mod ring_W) * ring_tpf + i of its sample (row width N), and slot_frame of
  // every appended frame is set.
  void* ring;
  int32_t* slot_frame;
  int ring_W, ring_tpf, ring_n_q, ring_first, ring_B;
  // Optional rotated positional keys for the attention's key workspace (batch 1; rk_col a
  // multiple of 32; rk_dr 16, 32 or 64; M = rk_B * rk_n_q; geometry from `rope`): row m = chunk
  // token j = m mod rk_n_q of sample b = m / rk_n_q at frame rk_first + j / tpf.  The epilogue
  // stores RoPE3D of output columns [rk_col, rk_col + rk_dr) of row m, taken as rounded to bf16,
  // to workspace row rk_nc_pad + j of sample b; the epilogue warps also write the zero rows after
  // the chunk and, with rk_ring, the ring part (rows [0, rk_nc_pad): the rotated k_R of ring
  // slots from rk_cache / rk_slot_frame, zeros from rk_nc on) before the first accumulator is
  // ready.  Rows are laid out as key_workspace_layout() gives them (rk_rows per sample).
  void* rk;
  const void* rk_cache;
  const int32_t* rk_slot_frame;
  int32_t* rk_dev_status;
  int rk_col, rk_dr, rk_D, rk_dc, rk_n_q, rk_B, rk_W, rk_nc, rk_nc_pad, rk_rows, rk_first, rk_ring;
};

bool tc_gemm_supported(int M, int N, int K, int64_t a_sm, int64_t b_sn);
mla_status gemm_tc(const TcGemmArgs& g, cudaStream_t s);

bool tc_attention_supported(const Dims& d, bool has_w_uv);
mla_status attention_tc(const Dims& d, const AttnArgs& a, int n_valid, cudaStream_t s);
// The tensor-core attention with the query heads computed inside it from the query latent
// (c_q [B, n_q, d_cq], w_qcat [H, D, d_cq]): d_c <= 192, D <= 256, d_cq a multiple of 64.
bool tc_attention_fused_q_supported(const Dims& d, bool has_w_uv);
mla_status attention_tc_fused_q(const Dims& d, const AttnArgs& a, int n_valid, const void* c_q,
                                const void* w_qcat, int first_frame, cudaStream_t s);
// CTA-pair tensor-core attention (attention_pair_sm100.cu): pairs of heads share each key tile.
bool tc_attention_pair_supported(const Dims& d, bool has_w_uv);
mla_status attention_tc_pair(const Dims& d, const AttnArgs& a, int n_valid, cudaStream_t s);
// The attention kernel a configuration gets (pair, single-CTA tensor-core or CUDA-core), given a
// workspace that already holds the rotated keys.
mla_status attention_dispatch(const Dims& d, const AttnArgs& a, int n_valid, cudaStream_t s);

// Attention with the scratch held in the library's built-in device array
// (attention_static_ws.cu); args.ws is ignored.
size_t static_scratch_bytes();
mla_status attention_fwd_static_scratch(const Dims& d, const AttnArgs& args,
                                        const int32_t* slot_frame, int n_valid, int first_frame,
                                        cudaStream_t s);

}  // namespace mla

#include <cuda.h>

namespace mla {

// Encodes a tiled TMA descriptor over a bf16 tensor.  dims[0] is the contiguous dimension;
// strides_bytes[i] is the byte stride of dims[i + 1]; box[i] the tile extent per dimension;
// swizzle_bytes 0, 32, 64 or 128.  Out-of-range elements of a tile read as zero.
mla_status make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                          const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes);

}  // namespace mla
