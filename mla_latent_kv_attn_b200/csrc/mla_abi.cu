// mla_abi.cu - the extern "C" entry points of include/mla.h: host-side validation, then launches
// on the caller's stream.  No allocation, no synchronisation.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <string>

#include "kernels.h"

namespace mla {

namespace {
thread_local std::string g_last_error;
}

void set_last_error(const std::string& msg) { g_last_error = msg; }

bool pdl_enabled() {
  static const bool on = std::getenv("MLA_NO_PDL") == nullptr;
  return on;
}

namespace {

constexpr int64_t kMaxElems = (int64_t{1} << 31) - 1;

mla_status check_cfg(const mla_config* cfg) {
  MLA_CHECK_ARG(cfg != nullptr, "config is null");
  const mla_config& c = *cfg;
  MLA_CHECK_ARG(c.d_model > 0 && c.n_heads > 0 && c.d_head > 0 && c.d_c > 0 && c.d_rope > 0 &&
                    c.d_cq > 0,
                "layer widths must be positive");
  MLA_CHECK_ARG(c.rope_pairs_t >= 0 && c.rope_pairs_h >= 0 && c.rope_pairs_w >= 0 &&
                    2 * (c.rope_pairs_t + c.rope_pairs_h + c.rope_pairs_w) == c.d_rope,
                "d_rope (%d) must equal 2*(rope_pairs_t+rope_pairs_h+rope_pairs_w)", c.d_rope);
  MLA_CHECK_ARG(c.rope_pairs_t + c.rope_pairs_h + c.rope_pairs_w <= kMaxRopePairs,
                "at most %d rotary pairs are supported", kMaxRopePairs);
  MLA_CHECK_ARG(std::isfinite(c.rope_base) && c.rope_base > 1.f, "rope_base must be > 1");
  MLA_CHECK_ARG(std::isfinite(c.softmax_scale) && c.softmax_scale > 0.f,
                "softmax_scale must be positive and finite");
  MLA_CHECK_ARG(c.frame_h > 0 && c.frame_w > 0 && c.chunk_frames > 0 && c.window_frames > 0 &&
                    c.batch > 0,
                "frame geometry, chunk, window and batch must be positive");
  MLA_CHECK_ARG(c.chunk_frames <= c.window_frames,
                "chunk_frames (%d) must not exceed window_frames (%d)", c.chunk_frames,
                c.window_frames);
  MLA_CHECK_ARG(c.dtype == MLA_BF16 || c.dtype == MLA_FP32, "unknown dtype %d", c.dtype);
  MLA_CHECK_ARG(c.kernel_path == MLA_PATH_AUTO || c.kernel_path == MLA_PATH_SIMT ||
                    c.kernel_path == MLA_PATH_TC_SINGLE || c.kernel_path == MLA_PATH_TC_PAIR,
                "unknown kernel_path %d", c.kernel_path);
  const int64_t tpf = int64_t{c.frame_h} * c.frame_w;
  const int64_t D = int64_t{c.d_c} + c.d_rope;
  const int64_t ring = int64_t{c.batch} * c.window_frames * tpf;
  const int64_t nq = int64_t{c.batch} * c.chunk_frames * tpf;
  MLA_CHECK_ARG(ring * D < kMaxElems && nq * c.n_heads * D < kMaxElems &&
                    nq * c.d_model < kMaxElems && nq * c.n_heads * c.d_head < kMaxElems &&
                    nq * c.n_heads * c.d_c < kMaxElems,
                "workload too large: every array must hold fewer than 2^31 elements");
  return MLA_OK;
}

// Frame indices are first_frame + (frame within the chunk) in int32; the chunk's exclusive end
// first_frame + frames must fit as well.
mla_status check_first_frame(int32_t first_frame, int64_t frames) {
  MLA_CHECK_ARG(first_frame >= 0, "first_frame must be >= 0");
  MLA_CHECK_ARG(int64_t{first_frame} + frames <= INT32_MAX,
                "first_frame (%d) + %lld frames overflows the int32 frame index", first_frame,
                static_cast<long long>(frames));
  return MLA_OK;
}

// Rejects null, misaligned, host-only or other-device pointers before anything is launched.
mla_status check_ptr(const void* p, const char* name, bool required = true) {
  if (p == nullptr) {
    if (required) MLA_FAIL(MLA_ERR_INVALID_ARG, "%s is null", name);
    return MLA_OK;
  }
  if (!aligned16(p)) MLA_FAIL(MLA_ERR_ALIGNMENT, "%s is not 16-byte aligned", name);
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    MLA_FAIL(MLA_ERR_INVALID_ARG, "%s is not a CUDA pointer (%s)", name, cudaGetErrorString(e));
  }
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    MLA_FAIL(MLA_ERR_INVALID_ARG, "%s is not device memory", name);
  int dev = -1;
  MLA_CUDA_TRY(cudaGetDevice(&dev));
  if (attr.device != dev)
    MLA_FAIL(MLA_ERR_INVALID_ARG, "%s lives on device %d, the current device is %d", name,
             attr.device, dev);
  return MLA_OK;
}

#define MLA_TRY(expr)               \
  do {                              \
    mla_status _s = (expr);         \
    if (_s != MLA_OK) return _s;    \
  } while (0)

bool use_tc(const Dims& d) { return d.dtype == MLA_BF16 && d.path != MLA_PATH_SIMT; }

// C[z](m, n) = sum_k A[z](m, k) B[z](n, k) with K contiguous in A and B; C row-major.
mla_status gemm(const Dims& d, const void* A, int64_t a_sm, int64_t a_batch, const void* B,
                int64_t b_sn, int64_t b_batch, void* C, int64_t c_sm, int64_t c_batch, int M,
                int N, int K, int batch, cudaStream_t s) {
  if (use_tc(d) && tc_gemm_supported(M, N, K, a_sm, b_sn) && a_batch % 8 == 0 &&
      b_batch % 8 == 0) {
    TcGemmArgs g{};
    g.A = A; g.a_sm = a_sm; g.a_batch = a_batch;
    g.B = B; g.b_sn = b_sn; g.b_batch = b_batch;
    g.C = C; g.c_sm = c_sm; g.c_batch = c_batch;
    g.M = M; g.N = N; g.K = K; g.batch = batch;
    g.epilogue = kEpiStore;
    return gemm_tc(g, s);
  }
  GemmArgs g{};
  g.A = A; g.a_sm = a_sm; g.a_sk = 1; g.a_batch = a_batch;
  g.B = B; g.b_sn = b_sn; g.b_sk = 1; g.b_batch = b_batch;
  g.C = C; g.c_sm = c_sm; g.c_batch = c_batch;
  g.M = M; g.N = N; g.K = K; g.batch = batch;
  return gemm_simt(g, d.dtype, s);
}

// q[m, h, :] = [w_qcat[h, 0:d_c] c_q[m] || RoPE3D(w_qcat[h, d_c:D] c_q[m], pos(m))]
mla_status query_heads(const Dims& d, const void* c_q, const void* w_qcat, void* q,
                       int first_frame, cudaStream_t s) {
  const int M = d.B * d.n_q;
  const int N = d.H * d.D;
  if (use_tc(d) && d.d_c % 2 == 0 && d.D % 8 == 0 &&
      tc_gemm_supported(M, N, d.d_cq, d.d_cq, d.d_cq)) {
    TcGemmArgs g{};
    g.A = c_q; g.a_sm = d.d_cq; g.a_batch = 0;
    g.B = w_qcat; g.b_sn = d.d_cq; g.b_batch = 0;
    g.C = q; g.c_sm = N; g.c_batch = 0;
    g.M = M; g.N = N; g.K = d.d_cq; g.batch = 1;
    g.epilogue = kEpiRopeQ; g.rope_D = d.D; g.rope_dr = d.d_rope; g.rope_n_q = d.n_q;
    g.rope_first_frame = first_frame;
    g.rope = rope_geom(d);
    return gemm_tc(g, s);
  }
  if (d.d_c % 2 == 0) {
    GemmArgs g{};
    g.A = c_q; g.a_sm = d.d_cq; g.a_sk = 1; g.a_batch = 0;
    g.B = w_qcat; g.b_sn = d.d_cq; g.b_sk = 1; g.b_batch = 0;
    g.C = q; g.c_sm = N; g.c_batch = 0;
    g.M = M; g.N = N; g.K = d.d_cq; g.batch = 1;
    g.rope_epi = 1; g.rope_D = d.D; g.rope_dc = d.d_c; g.rope_n_q = d.n_q;
    g.rope_first_frame = first_frame; g.rope = rope_geom(d);
    return gemm_simt(g, d.dtype, s);
  }
  MLA_TRY(gemm(d, c_q, d.d_cq, 0, w_qcat, d.d_cq, 0, q, N, 0, M, N, d.d_cq, 1, s));
  return rope3d_inplace(d, q, d.B, d.n_q, N, d.d_c, d.H, d.D, nullptr, 0, first_frame, s);
}

// c_q = W_down^Q x and chunk_lat = [W_down^KV x || W_R^K x]: on the tensor cores one GEMM over
// the stacked weights w_x with its columns split between the two outputs.
mla_status project_latents(const Dims& d, const void* x, const void* w_x, void* c_q,
                           void* chunk_lat, cudaStream_t s) {
  const int M = d.B * d.n_q;
  const int N = d.d_cq + d.D;
  if (use_tc(d) && d.d_cq % 32 == 0 && tc_gemm_supported(M, N, d.d_model, d.d_model, d.d_model)) {
    // one pass over x: columns 0..d_cq-1 are c_Q, the rest [c_KV || k_R]
    TcGemmArgs g{};
    g.A = x; g.a_sm = d.d_model; g.a_batch = 0;
    g.B = w_x; g.b_sn = d.d_model; g.b_batch = 0;
    g.C = c_q; g.c_sm = d.d_cq; g.c_batch = 0;
    g.C2 = chunk_lat; g.c2_sm = d.D; g.c2_batch = 0; g.n_split = d.d_cq;
    g.M = M; g.N = N; g.K = d.d_model; g.batch = 1;
    g.epilogue = kEpiStore;
    return gemm_tc(g, s);
  }
  const size_t es = dtype_size(d.dtype);
  MLA_TRY(gemm(d, x, d.d_model, 0, w_x, d.d_model, 0, c_q, d.d_cq, 0, M, d.d_cq, d.d_model, 1, s));
  return gemm(d, x, d.d_model, 0, static_cast<const char*>(w_x) + es * d.d_cq * d.d_model,
              d.d_model, 0, chunk_lat, d.D, 0, M, d.D, d.d_model, 1, s);
}

mla_status check_workspace(const Dims& d, int n_valid, const void* workspace,
                           size_t workspace_bytes) {
  const KeyWorkspace kw = key_workspace_layout(d, n_valid);
  if (workspace == nullptr || workspace_bytes < kw.bytes)
    MLA_FAIL(MLA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes,
             kw.bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    MLA_FAIL(MLA_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  return check_ptr(workspace, "workspace");
}

// project_latents plus the rotated positional keys of the chunk's attention in the key
// workspace: on the tensor cores one GEMM whose epilogue writes them (the ring's too with
// rotate_ring), otherwise the GEMMs and the rotation pass.
mla_status project_latents_rotated(const Dims& d, const void* x, const void* w_x, void* c_q,
                                   void* chunk_lat, const void* cache, const int32_t* slot_frame,
                                   int n_valid, int first_frame, int rotate_ring, void* workspace,
                                   int32_t* dev_status, cudaStream_t s) {
  const int M = d.B * d.n_q;
  const int N = d.d_cq + d.D;
  const KeyWorkspace kw = key_workspace_layout(d, n_valid);
  if (use_tc(d) && d.d_cq % 32 == 0 && (d.d_cq + d.d_c) % 32 == 0 &&
      (d.d_rope == 16 || d.d_rope == 32 || d.d_rope == 64) && d.tpf > 0 &&
      static_cast<int64_t>(d.B) * kw.rows < (int64_t{1} << 31) &&
      tc_gemm_supported(M, N, d.d_model, d.d_model, d.d_model)) {
    TcGemmArgs g{};
    g.A = x; g.a_sm = d.d_model; g.a_batch = 0;
    g.B = w_x; g.b_sn = d.d_model; g.b_batch = 0;
    g.C = c_q; g.c_sm = d.d_cq; g.c_batch = 0;
    g.C2 = chunk_lat; g.c2_sm = d.D; g.c2_batch = 0; g.n_split = d.d_cq;
    g.M = M; g.N = N; g.K = d.d_model; g.batch = 1;
    g.epilogue = kEpiStore;
    g.rope = rope_geom(d);
    g.rk = workspace; g.rk_cache = cache; g.rk_slot_frame = slot_frame;
    g.rk_dev_status = dev_status;
    g.rk_col = d.d_cq + d.d_c; g.rk_dr = d.d_rope; g.rk_D = d.D; g.rk_dc = d.d_c;
    g.rk_n_q = d.n_q; g.rk_B = d.B; g.rk_W = d.W; g.rk_nc = kw.nc; g.rk_nc_pad = kw.nc_pad;
    g.rk_rows = kw.rows; g.rk_first = first_frame; g.rk_ring = rotate_ring ? 1 : 0;
    return gemm_tc(g, s);
  }
  MLA_TRY(project_latents(d, x, w_x, c_q, chunk_lat, s));
  return build_rope_keys(d, cache, chunk_lat, slot_frame, n_valid, first_frame, workspace, s,
                         rotate_ring ? kRopeKeysAll : kRopeKeysChunk, dev_status, 1);
}

// Shared body of the attention entry points: checks, the rotated-key pre-pass (all of it, or
// only the chunk's keys when the ring's rotated keys are already in the workspace), attention.
mla_status attention_entry(const mla_config* cfg, const void* q, const void* chunk_lat,
                           const void* cache, const int32_t* slot_frame, int32_t n_valid_frames,
                           int32_t first_frame, const void* w_uv, void* out, float* lse,
                           void* workspace, size_t workspace_bytes, int32_t* dev_status,
                           void* stream, int rope_part) {
  set_last_error("");
  MLA_TRY(check_cfg(cfg));
  const Dims d = dims_of(*cfg);
  MLA_CHECK_ARG(n_valid_frames >= 0 && n_valid_frames <= d.W, "n_valid_frames must be in [0, %d]",
                d.W);
  MLA_TRY(check_first_frame(first_frame, d.C));
  MLA_TRY(check_ptr(q, "q"));
  MLA_TRY(check_ptr(chunk_lat, "chunk_lat"));
  MLA_TRY(check_ptr(slot_frame, "slot_frame"));
  MLA_TRY(check_ptr(out, "out"));
  MLA_TRY(check_ptr(cache, "cache", n_valid_frames > 0));
  MLA_TRY(check_ptr(w_uv, "w_uv", false));
  MLA_TRY(check_ptr(lse, "lse", false));
  MLA_TRY(check_ptr(dev_status, "dev_status", false));
  MLA_TRY(check_workspace(d, n_valid_frames, workspace, workspace_bytes));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MLA_TRY(build_rope_keys(d, cache, chunk_lat, slot_frame, n_valid_frames, first_frame, workspace, s,
                          rope_part, dev_status, 1));
  AttnArgs a{};
  a.q = q; a.chunk_lat = chunk_lat; a.cache = cache; a.ws = workspace; a.w_uv = w_uv;
  a.out = out; a.lse = lse; a.dev_status = dev_status;
  return attention_dispatch(d, a, n_valid_frames, s);
}

// Shared body of the attention-from-query-latent entry points (query heads formed inside the
// attention kernel); rope_part as in attention_entry.
mla_status attention_from_cq_entry(const mla_config* cfg, const void* c_q, const void* w_qcat,
                                   const void* chunk_lat, const void* cache,
                                   const int32_t* slot_frame, int32_t n_valid_frames,
                                   int32_t first_frame, const void* w_uv, void* out, float* lse,
                                   void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                   void* stream, int rope_part) {
  set_last_error("");
  MLA_TRY(check_cfg(cfg));
  const Dims d = dims_of(*cfg);
  MLA_CHECK_ARG(n_valid_frames >= 0 && n_valid_frames <= d.W, "n_valid_frames must be in [0, %d]",
                d.W);
  MLA_TRY(check_first_frame(first_frame, d.C));
  if (!(use_tc(d) && tc_attention_fused_q_supported(d, w_uv != nullptr)))
    MLA_FAIL(MLA_ERR_UNSUPPORTED,
             "attention from the query latent needs the tensor-core path (bf16, d_c <= 192, "
             "d_c + d_rope <= 256, d_cq a multiple of 64); use mla_project_chunk and "
             "mla_attention_fwd");
  MLA_TRY(check_ptr(c_q, "c_q"));
  MLA_TRY(check_ptr(w_qcat, "w_qcat"));
  MLA_TRY(check_ptr(chunk_lat, "chunk_lat"));
  MLA_TRY(check_ptr(slot_frame, "slot_frame"));
  MLA_TRY(check_ptr(out, "out"));
  MLA_TRY(check_ptr(cache, "cache", n_valid_frames > 0));
  MLA_TRY(check_ptr(w_uv, "w_uv", false));
  MLA_TRY(check_ptr(lse, "lse", false));
  MLA_TRY(check_ptr(dev_status, "dev_status", false));
  MLA_TRY(check_workspace(d, n_valid_frames, workspace, workspace_bytes));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (rope_part != kRopeKeysNone)
    MLA_TRY(build_rope_keys(d, cache, chunk_lat, slot_frame, n_valid_frames, first_frame,
                            workspace, s, rope_part, dev_status, 1));
  AttnArgs a{};
  a.q = nullptr; a.chunk_lat = chunk_lat; a.cache = cache; a.ws = workspace; a.w_uv = w_uv;
  a.out = out; a.lse = lse; a.dev_status = dev_status;
  return attention_tc_fused_q(d, a, n_valid_frames, c_q, w_qcat, first_frame, s);
}

}  // namespace

mla_status attention_dispatch(const Dims& d, const AttnArgs& a, int n_valid, cudaStream_t s) {
  const bool has_w_uv = a.w_uv != nullptr;
  if (use_tc(d) && tc_attention_supported(d, has_w_uv)) {
    if (d.path == MLA_PATH_TC_PAIR && tc_attention_pair_supported(d, has_w_uv))
      return attention_tc_pair(d, a, n_valid, s);
    return attention_tc(d, a, n_valid, s);
  }
  return attention_simt(d, a, n_valid, s);
}

}  // namespace mla

using namespace mla;

extern "C" {

const char* mla_status_string(int32_t status) {
  switch (status) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_ALIGNMENT: return "MLA_ERR_ALIGNMENT";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_DEVICE_CHECK: return "MLA_ERR_DEVICE_CHECK";
    default: return "MLA_ERR_UNKNOWN";
  }
}

const char* mla_last_error(void) { return g_last_error.c_str(); }

int32_t mla_abi_version(void) { return MLA_ABI_VERSION; }

mla_status mla_config_check(const mla_config* cfg) {
  MLA_NVTX_RANGE("mla_config_check");
  return check_cfg(cfg);
}

mla_status mla_cache_append(const mla_config* cfg, const void* x, const void* w_dkv_kr,
                            void* chunk_lat, void* cache, int32_t* slot_frame,
                            int32_t first_frame, int32_t mode, void* stream) {
  MLA_NVTX_RANGE("mla_cache_append");
  set_last_error("");
  MLA_TRY(check_cfg(cfg));
  MLA_CHECK_ARG(mode == MLA_PROJECT || mode == MLA_APPEND || mode == MLA_PROJECT_AND_APPEND,
                "unknown mode %d", mode);
  const Dims d = dims_of(*cfg);
  MLA_TRY(check_first_frame(first_frame, d.C));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MLA_TRY(check_ptr(chunk_lat, "chunk_lat"));
  if (mode & MLA_PROJECT) {
    MLA_TRY(check_ptr(x, "x"));
    MLA_TRY(check_ptr(w_dkv_kr, "w_dkv_kr"));
  }
  if (mode & MLA_APPEND) {
    MLA_TRY(check_ptr(cache, "cache"));
    MLA_TRY(check_ptr(slot_frame, "slot_frame"));
  }
  const int M = d.B * d.n_q;
  if (mode == MLA_PROJECT_AND_APPEND && use_tc(d) &&
      tc_gemm_supported(M, d.D, d.d_model, d.d_model, d.d_model)) {
    // one kernel: the GEMM's epilogue stores every row to chunk_lat and to its ring slot
    TcGemmArgs g{};
    g.A = x; g.a_sm = d.d_model; g.a_batch = 0;
    g.B = w_dkv_kr; g.b_sn = d.d_model; g.b_batch = 0;
    g.C = chunk_lat; g.c_sm = d.D; g.c_batch = 0;
    g.M = M; g.N = d.D; g.K = d.d_model; g.batch = 1;
    g.epilogue = kEpiStore;
    g.ring = cache; g.slot_frame = slot_frame;
    g.ring_W = d.W; g.ring_tpf = d.tpf; g.ring_n_q = d.n_q; g.ring_first = first_frame;
    g.ring_B = d.B;
    return gemm_tc(g, s);
  }
  if (mode & MLA_PROJECT)
    MLA_TRY(gemm(d, x, d.d_model, 0, w_dkv_kr, d.d_model, 0, chunk_lat, d.D, 0, M, d.D,
                 d.d_model, 1, s));
  if (mode & MLA_APPEND) MLA_TRY(ring_append(d, chunk_lat, cache, slot_frame, first_frame, s));
  return MLA_OK;
}

mla_status mla_rope3d(const mla_config* cfg, void* data, int32_t n_samples,
                      int32_t rows_per_sample, int32_t row_width, int32_t col_offset,
                      int32_t n_vec, int32_t vec_stride, const int32_t* frame_table,
                      int32_t frame_table_stride, int32_t first_frame, void* stream) {
  MLA_NVTX_RANGE("mla_rope3d");
  set_last_error("");
  MLA_TRY(check_cfg(cfg));
  const Dims d = dims_of(*cfg);
  MLA_CHECK_ARG(n_samples >= 0 && rows_per_sample >= 0 && n_vec >= 0, "negative size");
  MLA_CHECK_ARG(rows_per_sample % d.tpf == 0, "rows_per_sample must be a multiple of %d", d.tpf);
  MLA_CHECK_ARG(col_offset >= 0 && vec_stride >= 0 && row_width > 0, "bad row geometry");
  MLA_CHECK_ARG(n_vec == 0 || int64_t{col_offset} + int64_t{n_vec - 1} * vec_stride + d.d_rope <=
                                  row_width,
                "rotated vectors reach beyond row_width");
  MLA_CHECK_ARG(int64_t{n_samples} * rows_per_sample * row_width < kMaxElems, "array too large");
  if (frame_table == nullptr) MLA_TRY(check_first_frame(first_frame, rows_per_sample / d.tpf));
  if (int64_t{n_samples} * rows_per_sample * n_vec == 0) return MLA_OK;
  MLA_TRY(check_ptr(data, "data"));
  if (frame_table != nullptr) {
    MLA_TRY(check_ptr(frame_table, "frame_table"));
    MLA_CHECK_ARG(frame_table_stride >= rows_per_sample / d.tpf, "frame_table_stride too small");
  }
  return rope3d_inplace(d, data, n_samples, rows_per_sample, row_width, col_offset, n_vec,
                        vec_stride, frame_table, frame_table_stride, first_frame,
                        static_cast<cudaStream_t>(stream));
}

mla_status mla_key_positions(const mla_config* cfg, const int32_t* slot_frame,
                             int32_t n_valid_frames, int32_t first_frame, int32_t* pos_out,
                             void* stream) {
  MLA_NVTX_RANGE("mla_key_positions");
  set_last_error("");
  MLA_TRY(check_cfg(cfg));
  const Dims d = dims_of(*cfg);
  MLA_CHECK_ARG(n_valid_frames >= 0 && n_valid_frames <= d.W, "n_valid_frames must be in [0, %d]",
                d.W);
  MLA_TRY(check_first_frame(first_frame, d.C));
  MLA_TRY(check_ptr(slot_frame, "slot_frame"));
  MLA_TRY(check_ptr(pos_out, "pos_out"));
  return key_positions(d, slot_frame, n_valid_frames, first_frame, pos_out,
                       static_cast<cudaStream_t>(stream));
}

mla_status mla_compose_query_weights(const mla_config* cfg, const void* w_uq, const void* w_uk,
                                     const void* w_qr, void* w_qcat, void* stream) {
  MLA_NVTX_RANGE("mla_compose_query_weights");
  set_last_error("");
  MLA_TRY(check_cfg(cfg));
  const Dims d = dims_of(*cfg);
  MLA_TRY(check_ptr(w_uq, "w_uq"));
  MLA_TRY(check_ptr(w_uk, "w_uk"));
  MLA_TRY(check_ptr(w_qr, "w_qr"));
  MLA_TRY(check_ptr(w_qcat, "w_qcat"));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // w_qcat[h, c, k] = sum_d w_uk[h, d, c] w_uq[h, d, k]   (fp32 accumulation, one rounding)
  GemmArgs g{};
  g.A = w_uk; g.a_sm = 1; g.a_sk = d.d_c; g.a_batch = int64_t{d.d_head} * d.d_c;
  g.B = w_uq; g.b_sn = 1; g.b_sk = d.d_cq; g.b_batch = int64_t{d.d_head} * d.d_cq;
  g.C = w_qcat; g.c_sm = d.d_cq; g.c_batch = int64_t{d.D} * d.d_cq;
  g.M = d.d_c; g.N = d.d_cq; g.K = d.d_head; g.batch = d.H;
  MLA_TRY(gemm_simt(g, d.dtype, s));
  // w_qcat[h, d_c + r, k] = w_qr[h, r, k]
  const size_t es = dtype_size(d.dtype);
  return copy_rows(d.dtype, w_qr, d.d_cq, static_cast<char*>(w_qcat) + es * d.d_c * d.d_cq, d.d_cq,
                   d.d_rope, d.d_cq, int64_t{d.d_rope} * d.d_cq, int64_t{d.D} * d.d_cq, d.H, s);
}

mla_status mla_query_proj(const mla_config* cfg, const void* x, const void* w_dq,
                          const void* w_qcat, void* c_q, void* q, int32_t first_frame,
                          void* stream) {
  MLA_NVTX_RANGE("mla_query_proj");
  set_last_error("");
  MLA_TRY(check_cfg(cfg));
  const Dims d = dims_of(*cfg);
  MLA_TRY(check_first_frame(first_frame, d.C));
  MLA_TRY(check_ptr(x, "x"));
  MLA_TRY(check_ptr(w_dq, "w_dq"));
  MLA_TRY(check_ptr(w_qcat, "w_qcat"));
  MLA_TRY(check_ptr(c_q, "c_q"));
  MLA_TRY(check_ptr(q, "q"));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int M = d.B * d.n_q;
  MLA_TRY(gemm(d, x, d.d_model, 0, w_dq, d.d_model, 0, c_q, d.d_cq, 0, M, d.d_cq, d.d_model, 1, s));
  return query_heads(d, c_q, w_qcat, q, first_frame, s);
}

mla_status mla_project_chunk(const mla_config* cfg, const void* x, const void* w_x,
                             const void* w_qcat, void* c_q, void* q, void* chunk_lat,
                             int32_t first_frame, void* stream) {
  MLA_NVTX_RANGE("mla_project_chunk");
  set_last_error("");
  MLA_TRY(check_cfg(cfg));
  const Dims d = dims_of(*cfg);
  MLA_TRY(check_first_frame(first_frame, d.C));
  MLA_TRY(check_ptr(x, "x"));
  MLA_TRY(check_ptr(w_x, "w_x"));
  MLA_TRY(check_ptr(w_qcat, "w_qcat"));
  MLA_TRY(check_ptr(c_q, "c_q"));
  MLA_TRY(check_ptr(q, "q"));
  MLA_TRY(check_ptr(chunk_lat, "chunk_lat"));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MLA_TRY(project_latents(d, x, w_x, c_q, chunk_lat, s));
  return query_heads(d, c_q, w_qcat, q, first_frame, s);
}

mla_status mla_project_latents(const mla_config* cfg, const void* x, const void* w_x, void* c_q,
                               void* chunk_lat, void* stream) {
  MLA_NVTX_RANGE("mla_project_latents");
  set_last_error("");
  MLA_TRY(check_cfg(cfg));
  const Dims d = dims_of(*cfg);
  MLA_TRY(check_ptr(x, "x"));
  MLA_TRY(check_ptr(w_x, "w_x"));
  MLA_TRY(check_ptr(c_q, "c_q"));
  MLA_TRY(check_ptr(chunk_lat, "chunk_lat"));
  return project_latents(d, x, w_x, c_q, chunk_lat, static_cast<cudaStream_t>(stream));
}

mla_status mla_project_latents_rotated(const mla_config* cfg, const void* x, const void* w_x,
                                       void* c_q, void* chunk_lat, const void* cache,
                                       const int32_t* slot_frame, int32_t n_valid_frames,
                                       int32_t first_frame, int32_t rotate_ring, void* workspace,
                                       size_t workspace_bytes, int32_t* dev_status,
                                       void* stream) {
  MLA_NVTX_RANGE("mla_project_latents_rotated");
  set_last_error("");
  MLA_TRY(check_cfg(cfg));
  const Dims d = dims_of(*cfg);
  MLA_CHECK_ARG(n_valid_frames >= 0 && n_valid_frames <= d.W, "n_valid_frames must be in [0, %d]",
                d.W);
  MLA_CHECK_ARG(rotate_ring == 0 || rotate_ring == 1, "rotate_ring must be 0 or 1");
  MLA_TRY(check_first_frame(first_frame, d.C));
  MLA_TRY(check_ptr(x, "x"));
  MLA_TRY(check_ptr(w_x, "w_x"));
  MLA_TRY(check_ptr(c_q, "c_q"));
  MLA_TRY(check_ptr(chunk_lat, "chunk_lat"));
  MLA_TRY(check_ptr(slot_frame, "slot_frame"));
  MLA_TRY(check_ptr(cache, "cache", rotate_ring && n_valid_frames > 0));
  MLA_TRY(check_ptr(dev_status, "dev_status", false));
  MLA_TRY(check_workspace(d, n_valid_frames, workspace, workspace_bytes));
  return project_latents_rotated(d, x, w_x, c_q, chunk_lat, cache, slot_frame, n_valid_frames,
                                 first_frame, rotate_ring, workspace, dev_status,
                                 static_cast<cudaStream_t>(stream));
}

int32_t mla_attention_uses_tensor_cores(const mla_config* cfg, int32_t with_w_uv) {
  if (check_cfg(cfg) != MLA_OK) return -1;
  const Dims d = dims_of(*cfg);
  return (use_tc(d) && tc_attention_supported(d, with_w_uv != 0)) ? 1 : 0;
}

size_t mla_attention_workspace_bytes(const mla_config* cfg, int32_t n_valid_frames) {
  if (check_cfg(cfg) != MLA_OK) return 0;
  const Dims d = dims_of(*cfg);
  if (n_valid_frames < 0 || n_valid_frames > d.W) return 0;
  return key_workspace_layout(d, n_valid_frames).bytes;
}

mla_status mla_attention_fwd(const mla_config* cfg, const void* q, const void* chunk_lat,
                             const void* cache, const int32_t* slot_frame,
                             int32_t n_valid_frames, int32_t first_frame, const void* w_uv,
                             void* out, float* lse, void* workspace, size_t workspace_bytes,
                             int32_t* dev_status, void* stream) {
  MLA_NVTX_RANGE("mla_attention_fwd");
  return attention_entry(cfg, q, chunk_lat, cache, slot_frame, n_valid_frames, first_frame, w_uv,
                         out, lse, workspace, workspace_bytes, dev_status, stream, kRopeKeysAll);
}

mla_status mla_attention_fwd_from_cq(const mla_config* cfg, const void* c_q, const void* w_qcat,
                                     const void* chunk_lat, const void* cache,
                                     const int32_t* slot_frame, int32_t n_valid_frames,
                                     int32_t first_frame, const void* w_uv, void* out, float* lse,
                                     void* workspace, size_t workspace_bytes,
                                     int32_t* dev_status, void* stream) {
  MLA_NVTX_RANGE("mla_attention_fwd_from_cq");
  return attention_from_cq_entry(cfg, c_q, w_qcat, chunk_lat, cache, slot_frame, n_valid_frames,
                                 first_frame, w_uv, out, lse, workspace, workspace_bytes,
                                 dev_status, stream, kRopeKeysAll);
}

mla_status mla_attention_fwd_from_cq_cached_ring(
    const mla_config* cfg, const void* c_q, const void* w_qcat, const void* chunk_lat,
    const void* cache, const int32_t* slot_frame, int32_t n_valid_frames, int32_t first_frame,
    const void* w_uv, void* out, float* lse, void* workspace, size_t workspace_bytes,
    int32_t* dev_status, void* stream) {
  MLA_NVTX_RANGE("mla_attention_fwd_from_cq_cached_ring");
  return attention_from_cq_entry(cfg, c_q, w_qcat, chunk_lat, cache, slot_frame, n_valid_frames,
                                 first_frame, w_uv, out, lse, workspace, workspace_bytes,
                                 dev_status, stream, kRopeKeysChunk);
}

mla_status mla_attention_fwd_from_cq_prerotated(
    const mla_config* cfg, const void* c_q, const void* w_qcat, const void* chunk_lat,
    const void* cache, const int32_t* slot_frame, int32_t n_valid_frames, int32_t first_frame,
    const void* w_uv, void* out, float* lse, void* workspace, size_t workspace_bytes,
    int32_t* dev_status, void* stream) {
  MLA_NVTX_RANGE("mla_attention_fwd_from_cq_prerotated");
  return attention_from_cq_entry(cfg, c_q, w_qcat, chunk_lat, cache, slot_frame, n_valid_frames,
                                 first_frame, w_uv, out, lse, workspace, workspace_bytes,
                                 dev_status, stream, kRopeKeysNone);
}

mla_status mla_attention_fwd_cached_ring(const mla_config* cfg, const void* q,
                                         const void* chunk_lat, const void* cache,
                                         const int32_t* slot_frame, int32_t n_valid_frames,
                                         int32_t first_frame, const void* w_uv, void* out,
                                         float* lse, void* workspace, size_t workspace_bytes,
                                         int32_t* dev_status, void* stream) {
  MLA_NVTX_RANGE("mla_attention_fwd_cached_ring");
  return attention_entry(cfg, q, chunk_lat, cache, slot_frame, n_valid_frames, first_frame, w_uv,
                         out, lse, workspace, workspace_bytes, dev_status, stream,
                         kRopeKeysChunk);
}

mla_status mla_rotate_ring_keys(const mla_config* cfg, const void* cache,
                                const int32_t* slot_frame, int32_t n_valid_frames,
                                void* workspace, size_t workspace_bytes, void* stream) {
  MLA_NVTX_RANGE("mla_rotate_ring_keys");
  set_last_error("");
  MLA_TRY(check_cfg(cfg));
  const Dims d = dims_of(*cfg);
  MLA_CHECK_ARG(n_valid_frames >= 0 && n_valid_frames <= d.W, "n_valid_frames must be in [0, %d]",
                d.W);
  MLA_TRY(check_ptr(slot_frame, "slot_frame"));
  MLA_TRY(check_ptr(cache, "cache", n_valid_frames > 0));
  MLA_TRY(check_workspace(d, n_valid_frames, workspace, workspace_bytes));
  return build_rope_keys(d, cache, nullptr, slot_frame, n_valid_frames, 0, workspace,
                         static_cast<cudaStream_t>(stream), kRopeKeysRing);
}

mla_status mla_attention_fwd_static_scratch(const mla_config* cfg, const void* q,
                                            const void* chunk_lat, const void* cache,
                                            const int32_t* slot_frame, int32_t n_valid_frames,
                                            int32_t first_frame, const void* w_uv, void* out,
                                            float* lse, int32_t* dev_status, void* stream) {
  MLA_NVTX_RANGE("mla_attention_fwd_static_scratch");
  set_last_error("");
  MLA_TRY(check_cfg(cfg));
  const Dims d = dims_of(*cfg);
  MLA_CHECK_ARG(n_valid_frames >= 0 && n_valid_frames <= d.W, "n_valid_frames must be in [0, %d]",
                d.W);
  MLA_TRY(check_first_frame(first_frame, d.C));
  MLA_TRY(check_ptr(q, "q"));
  MLA_TRY(check_ptr(chunk_lat, "chunk_lat"));
  MLA_TRY(check_ptr(slot_frame, "slot_frame"));
  MLA_TRY(check_ptr(out, "out"));
  MLA_TRY(check_ptr(cache, "cache", n_valid_frames > 0));
  MLA_TRY(check_ptr(w_uv, "w_uv", false));
  MLA_TRY(check_ptr(lse, "lse", false));
  MLA_TRY(check_ptr(dev_status, "dev_status", false));
  AttnArgs a{};
  a.q = q; a.chunk_lat = chunk_lat; a.cache = cache; a.ws = nullptr; a.w_uv = w_uv;
  a.out = out; a.lse = lse; a.dev_status = dev_status;
  return attention_fwd_static_scratch(d, a, slot_frame, n_valid_frames, first_frame,
                                      static_cast<cudaStream_t>(stream));
}

size_t mla_attention_bwd_workspace_bytes(const mla_config* cfg, int32_t n_valid_frames) {
  if (check_cfg(cfg) != MLA_OK) return 0;
  const Dims d = dims_of(*cfg);
  if (n_valid_frames < 0 || n_valid_frames > d.W) return 0;
  return bwd_workspace_layout(d, n_valid_frames).bytes;
}

mla_status mla_attention_bwd(const mla_config* cfg, const void* q, const void* chunk_lat,
                             const void* cache, const int32_t* slot_frame,
                             int32_t n_valid_frames, int32_t first_frame, const void* o_lat,
                             const float* lse, const void* d_o_lat, void* d_q,
                             void* d_chunk_lat, void* d_cache, void* workspace,
                             size_t workspace_bytes, int32_t* dev_status, void* stream) {
  MLA_NVTX_RANGE("mla_attention_bwd");
  set_last_error("");
  MLA_TRY(check_cfg(cfg));
  const Dims d = dims_of(*cfg);
  MLA_CHECK_ARG(n_valid_frames >= 0 && n_valid_frames <= d.W, "n_valid_frames must be in [0, %d]",
                d.W);
  MLA_TRY(check_first_frame(first_frame, d.C));
  MLA_TRY(check_ptr(q, "q"));
  MLA_TRY(check_ptr(chunk_lat, "chunk_lat"));
  MLA_TRY(check_ptr(slot_frame, "slot_frame"));
  MLA_TRY(check_ptr(cache, "cache", n_valid_frames > 0));
  MLA_TRY(check_ptr(o_lat, "o_lat"));
  MLA_TRY(check_ptr(lse, "lse"));
  MLA_TRY(check_ptr(d_o_lat, "d_o_lat"));
  MLA_TRY(check_ptr(d_q, "d_q"));
  MLA_TRY(check_ptr(d_chunk_lat, "d_chunk_lat"));
  MLA_TRY(check_ptr(d_cache, "d_cache", n_valid_frames > 0));
  MLA_TRY(check_ptr(dev_status, "dev_status", false));
  const BwdWorkspace w = bwd_workspace_layout(d, n_valid_frames);
  if (workspace == nullptr || workspace_bytes < w.bytes)
    MLA_FAIL(MLA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes,
             w.bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    MLA_FAIL(MLA_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  MLA_TRY(check_ptr(workspace, "workspace"));
  BwdArgs a{};
  a.q = q; a.chunk_lat = chunk_lat; a.cache = cache; a.slot_frame = slot_frame; a.o_lat = o_lat;
  a.lse = lse; a.d_o_lat = d_o_lat; a.d_q = d_q; a.d_chunk_lat = d_chunk_lat; a.d_cache = d_cache;
  return attention_bwd(d, a, n_valid_frames, first_frame, workspace, dev_status,
                       static_cast<cudaStream_t>(stream));
}

mla_status mla_out_proj(const mla_config* cfg, const void* o_lat, const void* w_uv,
                        const void* w_o, void* o, void* y, void* stream) {
  MLA_NVTX_RANGE("mla_out_proj");
  set_last_error("");
  MLA_TRY(check_cfg(cfg));
  const Dims d = dims_of(*cfg);
  MLA_TRY(check_ptr(o_lat, "o_lat"));
  MLA_TRY(check_ptr(w_uv, "w_uv"));
  MLA_TRY(check_ptr(o, "o"));
  MLA_CHECK_ARG((w_o == nullptr) == (y == nullptr), "w_o and y must be given together");
  MLA_TRY(check_ptr(w_o, "w_o", false));
  MLA_TRY(check_ptr(y, "y", false));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int M = d.B * d.n_q;
  // o[m, h*d_head + e] = sum_c w_uv[h, e, c] o_lat[m, h, c]   (batched over heads)
  MLA_TRY(gemm(d, o_lat, int64_t{d.H} * d.d_c, d.d_c, w_uv, d.d_c, int64_t{d.d_head} * d.d_c, o,
               int64_t{d.H} * d.d_head, d.d_head, M, d.d_head, d.d_c, d.H, s));
  if (w_o != nullptr)
    MLA_TRY(gemm(d, o, int64_t{d.H} * d.d_head, 0, w_o, int64_t{d.H} * d.d_head, 0, y, d.d_model, 0,
                 M, d.d_model, d.H * d.d_head, 1, s));
  return MLA_OK;
}

}  // extern "C"
