// simt.cu - CUDA-core kernels: every step of the path for any shape and for fp32 / bf16.
// They serve the fp32 configurations, shapes the tensor-core kernels do not cover, and the
// elementwise steps (3D-RoPE, ring append, positions, rotated-key workspace) of every path.
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace mla {

// ============================================================================================
// Strided batched GEMM: C[z](m, n) = sum_k A[z](m, k) * B[z](n, k), fp32 accumulation.
// ============================================================================================

namespace {

constexpr int kTM = 64, kTN = 64, kTK = 16;

template <typename TA, typename TC>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs g) {
  __shared__ float As[kTK][kTM + 4];
  __shared__ float Bs[kTK][kTN + 4];
  const TA* A = static_cast<const TA*>(g.A) + static_cast<int64_t>(blockIdx.z) * g.a_batch;
  const TA* Bm = static_cast<const TA*>(g.B) + static_cast<int64_t>(blockIdx.z) * g.b_batch;
  TC* C = static_cast<TC*>(g.C) + static_cast<int64_t>(blockIdx.z) * g.c_batch;
  const int m0 = blockIdx.y * kTM, n0 = blockIdx.x * kTN;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.K; k0 += kTK) {
    for (int e = threadIdx.x; e < kTK * kTM; e += 256) {
      const int kk = e % kTK, mm = e / kTK;
      const int m = m0 + mm, k = k0 + kk;
      As[kk][mm] = (m < g.M && k < g.K)
                       ? Elem<TA>::to_f(A[static_cast<int64_t>(m) * g.a_sm + static_cast<int64_t>(k) * g.a_sk])
                       : 0.f;
    }
    for (int e = threadIdx.x; e < kTK * kTN; e += 256) {
      const int kk = e % kTK, nn = e / kTK;
      const int n = n0 + nn, k = k0 + kk;
      Bs[kk][nn] = (n < g.N && k < g.K)
                       ? Elem<TA>::to_f(Bm[static_cast<int64_t>(n) * g.b_sn + static_cast<int64_t>(k) * g.b_sk])
                       : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kTK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  if (g.rope_epi) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = m0 + ty * 4 + i;
      const int nl = m % g.rope_n_q;
      const int tok = nl % g.rope.tpf;
      const int t = g.rope_first_frame + nl / g.rope.tpf;
#pragma unroll
      for (int j = 0; j < 4; j += 2) {
        const int col = (n0 + tx * 4 + j) % g.rope_D;
        if (col >= g.rope_dc)
          rope_rotate(acc[i][j], acc[i][j + 1],
                      rope_angle(g.rope, (col - g.rope_dc) / 2, t, tok / g.rope.frame_w,
                                 tok % g.rope.frame_w));
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < g.N) C[static_cast<int64_t>(m) * g.c_sm + n] = Elem<TC>::from_f(acc[i][j]);
    }
  }
}

}  // namespace

mla_status gemm_simt(const GemmArgs& g, int dtype, cudaStream_t s) {
  if (g.M == 0 || g.N == 0) return MLA_OK;
  dim3 grid(ceil_div(g.N, kTN), ceil_div(g.M, kTM), g.batch);
  if (dtype == MLA_FP32)
    gemm_simt_kernel<float, float><<<grid, 256, 0, s>>>(g);
  else
    gemm_simt_kernel<bf16, bf16><<<grid, 256, 0, s>>>(g);
  MLA_LAUNCH_CHECK("gemm_simt");
  return MLA_OK;
}

// ============================================================================================
// 3D-RoPE in place
// ============================================================================================

namespace {

template <typename T>
__global__ void rope3d_kernel(T* data, int n_samples, int rows, int row_width, int col_offset,
                              int n_vec, int vec_stride, const int32_t* frame_table,
                              int frame_table_stride, int first_frame, int n_pairs, RopeGeom g) {
  const int64_t total = static_cast<int64_t>(n_samples) * rows * n_vec * n_pairs;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int pair = static_cast<int>(e % n_pairs);
    int64_t rest = e / n_pairs;
    const int v = static_cast<int>(rest % n_vec);
    rest /= n_vec;
    const int r = static_cast<int>(rest % rows);
    const int smp = static_cast<int>(rest / rows);
    const int fi = r / g.tpf, i = r % g.tpf;
    const int t = frame_table ? frame_table[static_cast<int64_t>(smp) * frame_table_stride + fi]
                              : first_frame + fi;
    if (t < 0) continue;
    T* p = data + (static_cast<int64_t>(smp) * rows + r) * row_width + col_offset +
           v * vec_stride + 2 * pair;
    float x0 = Elem<T>::to_f(p[0]), x1 = Elem<T>::to_f(p[1]);
    rope_rotate(x0, x1, rope_angle(g, pair, t, i / g.frame_w, i % g.frame_w));
    p[0] = Elem<T>::from_f(x0);
    p[1] = Elem<T>::from_f(x1);
  }
}

// One thread per rotated vector (d_rope values, whole 16-byte pieces): every piece is loaded
// before the first is rotated and stored, and the row's position is computed once.
template <typename T, int kPieces>
__global__ void __launch_bounds__(256)
    rope3d_vec_kernel(T* data, int n_samples, int rows, int row_width, int col_offset, int n_vec,
                      int vec_stride, const int32_t* frame_table, int frame_table_stride,
                      int first_frame, RopeGeom g) {
  constexpr int kPer = 16 / sizeof(T);
  const int64_t total = static_cast<int64_t>(n_samples) * rows * n_vec;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int v = static_cast<int>(e % n_vec);
    const int64_t rr = e / n_vec;                  // sample * rows + row
    const int r = static_cast<int>(rr % rows);
    const int smp = static_cast<int>(rr / rows);
    const int fi = r / g.tpf, i = r % g.tpf;
    const int t = frame_table ? frame_table[static_cast<int64_t>(smp) * frame_table_stride + fi]
                              : first_frame + fi;
    if (t < 0) continue;
    uint4* p = reinterpret_cast<uint4*>(data + rr * row_width + col_offset +
                                        static_cast<int64_t>(v) * vec_stride);
    uint4 raw[kPieces];
#pragma unroll
    for (int k = 0; k < kPieces; ++k) raw[k] = p[k];
    const int h = i / g.frame_w, w = i % g.frame_w;
#pragma unroll
    for (int k = 0; k < kPieces; ++k) {
      T* x = reinterpret_cast<T*>(&raw[k]);
#pragma unroll
      for (int q = 0; q < kPer; q += 2) {
        float x0 = Elem<T>::to_f(x[q]), x1 = Elem<T>::to_f(x[q + 1]);
        rope_rotate(x0, x1, rope_angle(g, (k * kPer + q) / 2, t, h, w));
        x[q] = Elem<T>::from_f(x0);
        x[q + 1] = Elem<T>::from_f(x1);
      }
      p[k] = raw[k];
    }
  }
}

template <typename T, int kPieces>
void launch_rope3d_vec(T* data, int n_samples, int rows, int row_width, int col_offset, int n_vec,
                       int vec_stride, const int32_t* frame_table, int frame_table_stride,
                       int first_frame, const RopeGeom& g, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(n_samples) * rows * n_vec;
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 148 * 16));
  rope3d_vec_kernel<T, kPieces><<<blocks, 256, 0, s>>>(data, n_samples, rows, row_width,
                                                       col_offset, n_vec, vec_stride, frame_table,
                                                       frame_table_stride, first_frame, g);
}

}  // namespace

mla_status rope3d_inplace(const Dims& d, void* data, int n_samples, int rows, int row_width,
                          int col_offset, int n_vec, int vec_stride, const int32_t* frame_table,
                          int frame_table_stride, int first_frame, cudaStream_t s) {
  const int n_pairs = d.d_rope / 2;
  const int64_t total = static_cast<int64_t>(n_samples) * rows * n_vec * n_pairs;
  if (total == 0) return MLA_OK;
  const int threads = 256;
  const int blocks = static_cast<int>(std::min<int64_t>((total + threads - 1) / threads, 148 * 16));
  const RopeGeom g = rope_geom(d);
  const int es = static_cast<int>(dtype_size(d.dtype));
  const int pieces = d.d_rope * es / 16;
  if (aligned16(data) && (d.d_rope * es) % 16 == 0 && (col_offset * es) % 16 == 0 &&
      (vec_stride * es) % 16 == 0 && (static_cast<int64_t>(row_width) * es) % 16 == 0 &&
      (pieces == 2 || pieces == 4 || pieces == 8)) {
#define MLA_ROPE_VEC(T, P)                                                                      \
  launch_rope3d_vec<T, P>(static_cast<T*>(data), n_samples, rows, row_width, col_offset, n_vec, \
                          vec_stride, frame_table, frame_table_stride, first_frame, g, s)
    if (d.dtype == MLA_FP32) {
      if (pieces == 2) MLA_ROPE_VEC(float, 2);
      else if (pieces == 4) MLA_ROPE_VEC(float, 4);
      else MLA_ROPE_VEC(float, 8);
    } else {
      if (pieces == 2) MLA_ROPE_VEC(bf16, 2);
      else if (pieces == 4) MLA_ROPE_VEC(bf16, 4);
      else MLA_ROPE_VEC(bf16, 8);
    }
#undef MLA_ROPE_VEC
    MLA_LAUNCH_CHECK("rope3d_vec");
    return MLA_OK;
  }
  if (d.dtype == MLA_FP32)
    rope3d_kernel<float><<<blocks, threads, 0, s>>>(static_cast<float*>(data), n_samples, rows,
                                                    row_width, col_offset, n_vec, vec_stride,
                                                    frame_table, frame_table_stride, first_frame,
                                                    n_pairs, g);
  else
    rope3d_kernel<bf16><<<blocks, threads, 0, s>>>(static_cast<bf16*>(data), n_samples, rows,
                                                   row_width, col_offset, n_vec, vec_stride,
                                                   frame_table, frame_table_stride, first_frame,
                                                   n_pairs, g);
  MLA_LAUNCH_CHECK("rope3d");
  return MLA_OK;
}

// ============================================================================================
// Ring append: chunk frame j -> slot (first_frame + j) mod W.  Copies 16-byte vectors.
// ============================================================================================

namespace {

__global__ void ring_append_kernel(const uint4* __restrict__ lat, uint4* __restrict__ cache,
                                   int32_t* __restrict__ slot_frame, int B, int C, int W,
                                   int vec_per_frame, int first_frame) {
  grid_dep_wait();     // launched with programmatic serialisation (launch_pdl)
  grid_dep_launch();
  const int64_t per_sample = static_cast<int64_t>(C) * vec_per_frame;
  const int64_t total = per_sample * B;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int b = static_cast<int>(e / per_sample);
    const int64_t r = e % per_sample;
    const int j = static_cast<int>(r / vec_per_frame);
    const int64_t v = r % vec_per_frame;
    const int slot = (first_frame + j) % W;
    cache[(static_cast<int64_t>(b) * W + slot) * vec_per_frame + v] = lat[e];
    if (v == 0) slot_frame[b * W + slot] = first_frame + j;
  }
}

}  // namespace

mla_status ring_append(const Dims& d, const void* chunk_lat, void* cache, int32_t* slot_frame,
                       int first_frame, cudaStream_t s) {
  const int64_t frame_bytes = static_cast<int64_t>(d.tpf) * d.D * dtype_size(d.dtype);
  if (frame_bytes % 16 != 0)
    MLA_FAIL(MLA_ERR_UNSUPPORTED, "frame of %lld bytes is not a multiple of 16",
             static_cast<long long>(frame_bytes));
  const int vec_per_frame = static_cast<int>(frame_bytes / 16);
  const int64_t total = static_cast<int64_t>(d.B) * d.C * vec_per_frame;
  const int threads = 256;
  const int blocks = static_cast<int>(std::min<int64_t>((total + threads - 1) / threads, 148 * 8));
  MLA_CUDA_TRY(launch_pdl(ring_append_kernel, dim3(blocks), dim3(threads), 0, s,
                          static_cast<const uint4*>(chunk_lat), static_cast<uint4*>(cache),
                          slot_frame, d.B, d.C, d.W, vec_per_frame, first_frame));
  return MLA_OK;
}

// ============================================================================================
// Key positions, in the walk order of the attention kernels.
// ============================================================================================


namespace {

__global__ void key_positions_kernel(const int32_t* slot_frame, int B, int W, int tpf,
                                     int frame_w, int nc, int nk, int first_frame, int32_t* out) {
  const int64_t total = static_cast<int64_t>(B) * nk;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int b = static_cast<int>(e / nk), m = static_cast<int>(e % nk);
    int t, h, w;
    key_position(slot_frame, b, W, tpf, frame_w, nc, first_frame, m, t, h, w);
    out[3 * e + 0] = t;
    out[3 * e + 1] = h;
    out[3 * e + 2] = w;
  }
}

}  // namespace

mla_status key_positions(const Dims& d, const int32_t* slot_frame, int n_valid, int first_frame,
                         int32_t* out, cudaStream_t s) {
  const int nc = n_valid * d.tpf, nk = nc + d.n_q;
  const int64_t total = static_cast<int64_t>(d.B) * nk;
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 148 * 8));
  key_positions_kernel<<<blocks, 256, 0, s>>>(slot_frame, d.B, d.W, d.tpf, d.frame_w, nc, nk,
                                              first_frame, out);
  MLA_LAUNCH_CHECK("key_positions");
  return MLA_OK;
}

// ============================================================================================
// Rotated positional keys of every attended key, tile-padded:
//   ws[b, r, :] = RoPE3D(k_R of ring slot r, pos)              r <  nc
//   ws[b, nc_pad + j, :] = RoPE3D(k_R of chunk token j, pos)   j <  n_q
//   zero elsewhere (nc <= r < nc_pad, and the rows after the chunk up to the padded end).
// ============================================================================================

namespace {

template <typename T>
__global__ void rope_keys_kernel(const T* __restrict__ cache, const T* __restrict__ chunk_lat,
                                 const int32_t* __restrict__ slot_frame, T* __restrict__ ws,
                                 int B, int W, int D, int d_c, int n_pairs, int n_q, int nc,
                                 int nc_pad, int rows_ws, int row_begin, int row_end,
                                 int first_frame, RopeGeom g, int32_t* dev_status,
                                 int check_window) {
  // rows [row_begin, row_end) of every sample's rows_ws workspace rows, one thread per pair
  // (32-bit index arithmetic: B * span * n_pairs stays far below 2^31)
  const int span = row_end - row_begin;
  const int total = B * span * n_pairs;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < total; e += gridDim.x * blockDim.x) {
    const int pair = e % n_pairs;
    const int rs = e / n_pairs;
    const int r = row_begin + rs % span;
    const int b = rs / span;
    const int64_t rr = static_cast<int64_t>(b) * rows_ws + r;
    T* dst = ws + rr * (2 * n_pairs) + 2 * pair;
    const T* src = nullptr;
    int m = -1;
    if (r < nc) {
      m = r;
      src = cache + (static_cast<int64_t>(b) * W * g.tpf + r) * D + d_c + 2 * pair;
    } else if (r >= nc_pad && r - nc_pad < n_q) {
      m = nc + (r - nc_pad);
      src = chunk_lat + (static_cast<int64_t>(b) * n_q + (r - nc_pad)) * D + d_c + 2 * pair;
    }
    if (src == nullptr) {
      dst[0] = Elem<T>::from_f(0.f);
      dst[1] = Elem<T>::from_f(0.f);
      continue;
    }
    int t, h, w;
    key_position(slot_frame, b, W, g.tpf, g.frame_w, nc, first_frame, m, t, h, w);
    if (m < nc)
      debug_check(t >= 0 && (!check_window || (t < first_frame && t >= first_frame - W)), dev_status);
    float x0 = Elem<T>::to_f(src[0]), x1 = Elem<T>::to_f(src[1]);
    rope_rotate(x0, x1, rope_angle(g, pair, t, h, w));
    dst[0] = Elem<T>::from_f(x0);
    dst[1] = Elem<T>::from_f(x1);
  }
}

// The same rows with 16-byte vectors: one thread per rotated key (rope_key_row: every piece is
// loaded before the first is rotated and stored, and the key's position is computed once).
// Needs d_c, d_rope and D at whole 16-byte multiples (host check).  Launched with programmatic
// serialisation (launch_pdl).
template <typename T, int kPieces>
__global__ void __launch_bounds__(256)
    rope_keys_vec_kernel(const T* __restrict__ cache, const T* __restrict__ chunk_lat,
                         const int32_t* __restrict__ slot_frame, T* __restrict__ ws, int B, int W,
                         int D, int d_c, int n_q, int nc, int nc_pad, int rows_ws, int row_begin,
                         int row_end, int first_frame, RopeGeom g, int32_t* dev_status,
                         int check_window) {
  grid_dep_wait();
  grid_dep_launch();
  const int span = row_end - row_begin;
  const int total = B * span;                   // < 2^31 (host check)
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < total; e += gridDim.x * blockDim.x)
    rope_key_row<T, kPieces>(cache, chunk_lat, slot_frame, ws, e / span, row_begin + e % span, W,
                             D, d_c, n_q, nc, nc_pad, rows_ws, first_frame, g, dev_status,
                             check_window);
}

}  // namespace

KeyWorkspace key_workspace_layout(const Dims& d, int n_valid) {
  KeyWorkspace k;
  k.nc = n_valid * d.tpf;
  k.nc_pad = round_up(k.nc, kKeyTile);
  k.rows = k.nc_pad + round_up(d.n_q, kKeyTile);
  k.bytes = static_cast<size_t>(d.B) * k.rows * d.d_rope * dtype_size(d.dtype);
  return k;
}

mla_status build_rope_keys(const Dims& d, const void* cache, const void* chunk_lat,
                           const int32_t* slot_frame, int n_valid, int first_frame, void* ws,
                           cudaStream_t s, int part, int32_t* dev_status, int check_window) {
  const KeyWorkspace k = key_workspace_layout(d, n_valid);
  const int n_pairs = d.d_rope / 2;
  // the ring part is rows [0, nc_pad) (its padding rows included), the chunk part the rest
  if (part == kRopeKeysNone) return MLA_OK;
  const int row_begin = part == kRopeKeysChunk ? k.nc_pad : 0;
  const int row_end = part == kRopeKeysRing ? k.nc_pad : k.rows;
  if (row_end <= row_begin) return MLA_OK;
  if (static_cast<int64_t>(d.B) * (row_end - row_begin) * (d.d_rope / 2) >= (int64_t{1} << 31))
    MLA_FAIL(MLA_ERR_UNSUPPORTED, "too many rotated keys for one launch");
  const int64_t total = static_cast<int64_t>(d.B) * (row_end - row_begin) * n_pairs;
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 148 * 16));
  const RopeGeom g = rope_geom(d);
  const size_t es = dtype_size(d.dtype);
  const bool vec = (d.d_c * es) % 16 == 0 && (d.d_rope * es) % 16 == 0 && (d.D * es) % 16 == 0 &&
                   aligned16(cache) && aligned16(chunk_lat) && aligned16(ws);
  const int pieces = d.d_rope * static_cast<int>(es) / 16;
  if (vec && (pieces == 2 || pieces == 4 || pieces == 8)) {
    const int64_t vtotal = static_cast<int64_t>(d.B) * (row_end - row_begin);
    const int vblocks = static_cast<int>(std::min<int64_t>((vtotal + 255) / 256, 148 * 16));
#define MLA_KEYS_VEC(T, P)                                                                       \
  MLA_CUDA_TRY(launch_pdl(rope_keys_vec_kernel<T, P>, dim3(vblocks), dim3(256), 0, s,          \
                          static_cast<const T*>(cache), static_cast<const T*>(chunk_lat),      \
                          slot_frame, static_cast<T*>(ws), d.B, d.W, d.D, d.d_c, d.n_q, k.nc,  \
                          k.nc_pad, k.rows, row_begin, row_end, first_frame, g, dev_status,    \
                          check_window))
    if (d.dtype == MLA_FP32) {
      if (pieces == 2) MLA_KEYS_VEC(float, 2);
      else if (pieces == 4) MLA_KEYS_VEC(float, 4);
      else MLA_KEYS_VEC(float, 8);
    } else {
      if (pieces == 2) MLA_KEYS_VEC(bf16, 2);
      else if (pieces == 4) MLA_KEYS_VEC(bf16, 4);
      else MLA_KEYS_VEC(bf16, 8);
    }
#undef MLA_KEYS_VEC
    MLA_LAUNCH_CHECK("rope_keys_vec");
    return MLA_OK;
  }
  if (d.dtype == MLA_FP32)
    rope_keys_kernel<float><<<blocks, 256, 0, s>>>(
        static_cast<const float*>(cache), static_cast<const float*>(chunk_lat), slot_frame,
        static_cast<float*>(ws), d.B, d.W, d.D, d.d_c, n_pairs, d.n_q, k.nc, k.nc_pad, k.rows,
        row_begin, row_end, first_frame, g, dev_status, check_window);
  else
    rope_keys_kernel<bf16><<<blocks, 256, 0, s>>>(
        static_cast<const bf16*>(cache), static_cast<const bf16*>(chunk_lat), slot_frame,
        static_cast<bf16*>(ws), d.B, d.W, d.D, d.d_c, n_pairs, d.n_q, k.nc, k.nc_pad, k.rows,
        row_begin, row_end, first_frame, g, dev_status, check_window);
  MLA_LAUNCH_CHECK("rope_keys");
  return MLA_OK;
}

// ============================================================================================
// Attention on CUDA cores: one warp per (sample, head, query row), online softmax over the
// keys in walk order (ring slots, then the chunk).
// ============================================================================================

namespace {

constexpr int kMaxPerLane = 16;  // supports D <= 512 and d_c <= 512

template <typename T>
__global__ void __launch_bounds__(128)
    attention_simt_kernel(AttnArgs a, int B, int H, int n_q, int D, int d_c, int d_rope,
                          int d_head, int W, int tpf, float scale_log2, int nc, int nc_pad,
                          int rows_ws) {
  extern __shared__ float o_sm[];  // [4 warps][d_c]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n = blockIdx.x * 4 + warp;
  const int h = blockIdx.y, b = blockIdx.z;
  if (n >= n_q) return;
  const T* q = static_cast<const T*>(a.q) + ((static_cast<int64_t>(b) * n_q + n) * H + h) * D;
  const T* cache = static_cast<const T*>(a.cache) + static_cast<int64_t>(b) * W * tpf * D;
  const T* lat = static_cast<const T*>(a.chunk_lat) + static_cast<int64_t>(b) * n_q * D;
  const T* ws = static_cast<const T*>(a.ws) + static_cast<int64_t>(b) * rows_ws * d_rope;

  float qv[kMaxPerLane], ov[kMaxPerLane];
#pragma unroll
  for (int j = 0; j < kMaxPerLane; ++j) {
    const int c = lane + 32 * j;
    qv[j] = c < D ? Elem<T>::to_f(q[c]) : 0.f;
    ov[j] = 0.f;
  }
  float m_run = -INFINITY, l_run = 0.f;
  const int nk = nc + n_q;
  for (int m = 0; m < nk; ++m) {
    const T* content = m < nc ? cache + static_cast<int64_t>(m) * D
                              : lat + static_cast<int64_t>(m - nc) * D;
    const T* rope = ws + static_cast<int64_t>(m < nc ? m : nc_pad + (m - nc)) * d_rope;
    float part = 0.f, cv[kMaxPerLane];
#pragma unroll
    for (int j = 0; j < kMaxPerLane; ++j) {
      const int c = lane + 32 * j;
      float k = 0.f;
      if (c < d_c) k = Elem<T>::to_f(content[c]);
      else if (c < D) k = Elem<T>::to_f(rope[c - d_c]);
      cv[j] = c < d_c ? k : 0.f;
      part = fmaf(qv[j], k, part);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    const float s = part * scale_log2;          // log2 domain
    const float m_new = fmaxf(m_run, s);
    const float corr = exp2f(m_run - m_new);    // 0 on the first key
    const float p = exp2f(s - m_new);
    l_run = l_run * corr + p;
#pragma unroll
    for (int j = 0; j < kMaxPerLane; ++j) ov[j] = fmaf(ov[j], corr, p * cv[j]);
    m_run = m_new;
  }
  const float inv_l = 1.f / l_run;
  if (a.lse != nullptr && lane == 0)
    a.lse[(static_cast<int64_t>(b) * H + h) * n_q + n] =
        (m_run + log2f(l_run)) * 0.69314718055994530942f;
  if (a.w_uv == nullptr) {
    T* o = static_cast<T*>(a.out) + ((static_cast<int64_t>(b) * n_q + n) * H + h) * d_c;
#pragma unroll
    for (int j = 0; j < kMaxPerLane; ++j) {
      const int c = lane + 32 * j;
      if (c < d_c) o[c] = Elem<T>::from_f(ov[j] * inv_l);
    }
    return;
  }
  float* orow = o_sm + warp * d_c;
#pragma unroll
  for (int j = 0; j < kMaxPerLane; ++j) {
    const int c = lane + 32 * j;
    if (c < d_c) orow[c] = ov[j] * inv_l;
  }
  __syncwarp();
  const T* wuv = static_cast<const T*>(a.w_uv) + static_cast<int64_t>(h) * d_head * d_c;
  T* o = static_cast<T*>(a.out) + (static_cast<int64_t>(b) * n_q + n) * H * d_head +
         static_cast<int64_t>(h) * d_head;
  for (int dd = lane; dd < d_head; dd += 32) {
    float acc = 0.f;
    for (int c = 0; c < d_c; ++c) acc = fmaf(Elem<T>::to_f(wuv[dd * d_c + c]), orow[c], acc);
    o[dd] = Elem<T>::from_f(acc);
  }
}

}  // namespace

mla_status attention_simt(const Dims& d, const AttnArgs& a, int n_valid, cudaStream_t s) {
  if (d.D > 32 * kMaxPerLane || d.d_c > 32 * kMaxPerLane)
    MLA_FAIL(MLA_ERR_UNSUPPORTED, "CUDA-core attention supports d_c + d_rope <= %d",
             32 * kMaxPerLane);
  const KeyWorkspace k = key_workspace_layout(d, n_valid);
  dim3 grid(ceil_div(d.n_q, 4), d.H, d.B);
  const size_t smem = 4 * d.d_c * sizeof(float);
  const float scale_log2 = d.scale * 1.4426950408889634f;
  if (d.dtype == MLA_FP32)
    attention_simt_kernel<float><<<grid, 128, smem, s>>>(a, d.B, d.H, d.n_q, d.D, d.d_c, d.d_rope,
                                                         d.d_head, d.W, d.tpf, scale_log2, k.nc,
                                                         k.nc_pad, k.rows);
  else
    attention_simt_kernel<bf16><<<grid, 128, smem, s>>>(a, d.B, d.H, d.n_q, d.D, d.d_c, d.d_rope,
                                                        d.d_head, d.W, d.tpf, scale_log2, k.nc,
                                                        k.nc_pad, k.rows);
  MLA_LAUNCH_CHECK("attention_simt");
  return MLA_OK;
}

// ============================================================================================
// Small copies
// ============================================================================================

namespace {

template <typename T>
__global__ void copy_rows_kernel(const T* src, int64_t src_stride, T* dst, int64_t dst_stride,
                                 int rows, int cols, int64_t src_batch, int64_t dst_batch,
                                 int batch) {
  const int64_t total = static_cast<int64_t>(batch) * rows * cols;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(e % cols);
    const int64_t r2 = e / cols;
    const int r = static_cast<int>(r2 % rows);
    const int z = static_cast<int>(r2 / rows);
    dst[z * dst_batch + r * dst_stride + c] = src[z * src_batch + r * src_stride + c];
  }
}

}  // namespace

mla_status copy_rows(int dtype, const void* src, int64_t src_stride, void* dst,
                     int64_t dst_stride, int rows, int cols, int64_t src_batch,
                     int64_t dst_batch, int batch, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(batch) * rows * cols;
  if (total == 0) return MLA_OK;
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 148 * 8));
  if (dtype == MLA_FP32)
    copy_rows_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(src), src_stride,
                                                   static_cast<float*>(dst), dst_stride, rows,
                                                   cols, src_batch, dst_batch, batch);
  else
    copy_rows_kernel<bf16><<<blocks, 256, 0, s>>>(static_cast<const bf16*>(src), src_stride,
                                                  static_cast<bf16*>(dst), dst_stride, rows, cols,
                                                  src_batch, dst_batch, batch);
  MLA_LAUNCH_CHECK("copy_rows");
  return MLA_OK;
}

}  // namespace mla
