// attention_bwd.cu - gradients of the latent-space attention call (training use: the VideoMLA
// pages train the latent students through these layers; hyper.ai summary, "Method").
//
// Forward, per sample b, head h, query row n and key m (walk order: valid ring slots, then the
// chunk's own tokens):  K'_m = [c_m || RoPE3D(k_R,m)],  s = scale q.K'_m,
// p = exp(s - lse),  O_lat = sum_m p c_m.  For dL/dO_lat = G:
//   dP_nm   = G_n . c_m                       Delta_n = sum_m p_nm dP_nm = G_n . O_lat,n
//   dS_nm   = p_nm (dP_nm - Delta_n)
//   dq_n    = scale sum_m dS_nm K'_m
//   dK'_m   = scale sum_{h,n} dS_nm q_n       dV_m = sum_{h,n} p_nm G_n   (V = c: content part)
//   d latent_m = [dV_m + dK'_m[0:d_c]  ||  RoPE3D^T(dK'_m[d_c:])]
// (the transpose of a rotation is the rotation by the opposite angle).
//
// CUDA-core kernels (the tensor-core path for the Wan shape is attention_bwd_sm100.cu; both use
// bwd_delta_kernel), all fp32 arithmetic, no atomics:
//   bwd_delta_kernel   one warp per (b, n, h): Delta = G . O_lat
//   bwd_dq_kernel      one warp per (b, h, n): loop over the keys
//   bwd_dkey_kernel    one warp per (b, key): loop over every head and query row
// Probabilities are recomputed from q, the keys and lse, exactly as the forward defines them.
#include "kernels.h"

namespace mla {

namespace {

constexpr int kLanesMax = 16;   // D <= 512 across 32 lanes

struct BwdParams {
  const void* q;          // [B, n_q, H, D]
  const void* chunk_lat;  // [B, n_q, D]
  const void* cache;      // [B, W*tpf, D]
  const int32_t* slot_frame;
  const void* ws_rope;    // rotated positional keys [B, rows, d_rope]
  const void* o_lat;      // [B, n_q, H, d_c]
  const float* lse;       // [B, H, n_q]
  const void* d_o_lat;    // [B, n_q, H, d_c]
  float* delta;           // [B, H, n_q]
  void* d_q;              // [B, n_q, H, D]
  void* d_chunk_lat;      // [B, n_q, D]
  void* d_cache;          // [B, W*tpf, D]
  int B, H, n_q, D, d_c, d_rope, W, tpf, frame_w, nc, nc_pad, rows_ws, first_frame;
  float scale, scale_log2;
  RopeGeom rope;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Row m of K' in fp32 across the warp: lane l holds columns l + 32 j.
template <typename T>
__device__ __forceinline__ void load_key(const BwdParams& p, int b, int m, float (&k)[kLanesMax]) {
  const int lane = threadIdx.x % 32;
  const T* content = m < p.nc
      ? static_cast<const T*>(p.cache) + (static_cast<int64_t>(b) * p.W * p.tpf + m) * p.D
      : static_cast<const T*>(p.chunk_lat) + (static_cast<int64_t>(b) * p.n_q + (m - p.nc)) * p.D;
  const T* rope = static_cast<const T*>(p.ws_rope) +
                  (static_cast<int64_t>(b) * p.rows_ws + (m < p.nc ? m : p.nc_pad + (m - p.nc))) *
                      p.d_rope;
#pragma unroll
  for (int j = 0; j < kLanesMax; ++j) {
    const int c = lane + 32 * j;
    float v = 0.f;
    if (c < p.d_c) v = Elem<T>::to_f(content[c]);
    else if (c < p.D) v = Elem<T>::to_f(rope[c - p.d_c]);
    k[j] = v;
  }
}

template <typename T>
__global__ void __launch_bounds__(128)
    bwd_delta_kernel(BwdParams p) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * 4 + warp;   // (b, n, h) row-major
  const int64_t total = static_cast<int64_t>(p.B) * p.n_q * p.H;
  if (idx >= total) return;
  const int h = static_cast<int>(idx % p.H);
  const int64_t bn = idx / p.H;
  const int n = static_cast<int>(bn % p.n_q), b = static_cast<int>(bn / p.n_q);
  const T* o = static_cast<const T*>(p.o_lat) + idx * p.d_c;
  const T* g = static_cast<const T*>(p.d_o_lat) + idx * p.d_c;
  float acc = 0.f;
  if (sizeof(T) == 2 && p.d_c % 8 == 0) {
    // bf16 rows of a multiple of 8: 16-byte pieces, one per lane (a row starts 16-byte aligned:
    // d_c * 2 bytes is a multiple of 16)
    for (int c8 = lane; c8 < p.d_c / 8; c8 += 32) {
      const uint4 ov = reinterpret_cast<const uint4*>(o)[c8];
      const uint4 gv = reinterpret_cast<const uint4*>(g)[c8];
      const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ow[i]));
        const float2 gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[i]));
        acc = fmaf(of.x, gf.x, fmaf(of.y, gf.y, acc));
      }
    }
  } else {
    for (int c = lane; c < p.d_c; c += 32) acc = fmaf(Elem<T>::to_f(o[c]), Elem<T>::to_f(g[c]), acc);
  }
  acc = warp_sum(acc);
  if (lane == 0)
    p.delta[(static_cast<int64_t>(b) * p.H + h) * p.n_q + n] = acc;
}

template <typename T>
__global__ void __launch_bounds__(128)
    bwd_dq_kernel(BwdParams p) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n = blockIdx.x * 4 + warp;
  const int h = blockIdx.y, b = blockIdx.z;
  if (n >= p.n_q) return;
  const int64_t row = (static_cast<int64_t>(b) * p.n_q + n) * p.H + h;
  const T* q = static_cast<const T*>(p.q) + row * p.D;
  const T* g = static_cast<const T*>(p.d_o_lat) + row * p.d_c;
  const int64_t sr = (static_cast<int64_t>(b) * p.H + h) * p.n_q + n;
  const float lse2 = p.lse[sr] * 1.4426950408889634f;
  const float delta = p.delta[sr];
  float qv[kLanesMax], gv[kLanesMax], acc[kLanesMax];
#pragma unroll
  for (int j = 0; j < kLanesMax; ++j) {
    const int c = lane + 32 * j;
    qv[j] = c < p.D ? Elem<T>::to_f(q[c]) : 0.f;
    gv[j] = c < p.d_c ? Elem<T>::to_f(g[c]) : 0.f;
    acc[j] = 0.f;
  }
  const int nk = p.nc + p.n_q;
  for (int m = 0; m < nk; ++m) {
    float k[kLanesMax];
    load_key<T>(p, b, m, k);
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int j = 0; j < kLanesMax; ++j) {
      s = fmaf(qv[j], k[j], s);
      dp = fmaf(gv[j], k[j], dp);          // gv is zero beyond d_c: only the content part
    }
    s = warp_sum(s);
    dp = warp_sum(dp);
    const float pr = exp2f(s * p.scale_log2 - lse2);
    const float ds = pr * (dp - delta);
#pragma unroll
    for (int j = 0; j < kLanesMax; ++j) acc[j] = fmaf(ds, k[j], acc[j]);
  }
  T* dq = static_cast<T*>(p.d_q) + row * p.D;
#pragma unroll
  for (int j = 0; j < kLanesMax; ++j) {
    const int c = lane + 32 * j;
    if (c < p.D) dq[c] = Elem<T>::from_f(acc[j] * p.scale);
  }
}

template <typename T>
__global__ void __launch_bounds__(128)
    bwd_dkey_kernel(BwdParams p) {
  extern __shared__ float grad_sm[];   // [4 warps][D]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nk = p.nc + p.n_q;
  const int m = blockIdx.x * 4 + warp, b = blockIdx.y;
  if (m >= nk) return;
  float k[kLanesMax], acc[kLanesMax];
  load_key<T>(p, b, m, k);
#pragma unroll
  for (int j = 0; j < kLanesMax; ++j) acc[j] = 0.f;
  for (int h = 0; h < p.H; ++h) {
    const float* lse_h = p.lse + (static_cast<int64_t>(b) * p.H + h) * p.n_q;
    const float* delta_h = p.delta + (static_cast<int64_t>(b) * p.H + h) * p.n_q;
    for (int n = 0; n < p.n_q; ++n) {
      const int64_t row = (static_cast<int64_t>(b) * p.n_q + n) * p.H + h;
      const T* q = static_cast<const T*>(p.q) + row * p.D;
      const T* g = static_cast<const T*>(p.d_o_lat) + row * p.d_c;
      float qv[kLanesMax], gv[kLanesMax];
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int j = 0; j < kLanesMax; ++j) {
        const int c = lane + 32 * j;
        qv[j] = c < p.D ? Elem<T>::to_f(q[c]) : 0.f;
        gv[j] = c < p.d_c ? Elem<T>::to_f(g[c]) : 0.f;
        s = fmaf(qv[j], k[j], s);
        dp = fmaf(gv[j], k[j], dp);
      }
      s = warp_sum(s);
      dp = warp_sum(dp);
      const float pr = exp2f(s * p.scale_log2 - lse_h[n] * 1.4426950408889634f);
      const float ds_scaled = pr * (dp - delta_h[n]) * p.scale;
#pragma unroll
      for (int j = 0; j < kLanesMax; ++j) acc[j] = fmaf(pr, gv[j], fmaf(ds_scaled, qv[j], acc[j]));
    }
  }
  // content part as is; the positional part back through the transposed rotation
  float* gsm = grad_sm + warp * p.D;
#pragma unroll
  for (int j = 0; j < kLanesMax; ++j) {
    const int c = lane + 32 * j;
    if (c < p.D) gsm[c] = acc[j];
  }
  __syncwarp();
  int t, hh, ww;
  key_position(p.slot_frame, b, p.W, p.tpf, p.frame_w, p.nc, p.first_frame, m, t, hh, ww);
  T* dst = m < p.nc
      ? static_cast<T*>(p.d_cache) + (static_cast<int64_t>(b) * p.W * p.tpf + m) * p.D
      : static_cast<T*>(p.d_chunk_lat) + (static_cast<int64_t>(b) * p.n_q + (m - p.nc)) * p.D;
  for (int c = lane; c < p.d_c; c += 32) dst[c] = Elem<T>::from_f(gsm[c]);
  for (int pr = lane; pr < p.d_rope / 2; pr += 32) {
    float x0 = gsm[p.d_c + 2 * pr], x1 = gsm[p.d_c + 2 * pr + 1];
    rope_rotate(x0, x1, -rope_angle(p.rope, pr, t, hh, ww));
    dst[p.d_c + 2 * pr] = Elem<T>::from_f(x0);
    dst[p.d_c + 2 * pr + 1] = Elem<T>::from_f(x1);
  }
}

template <typename T>
mla_status launch_delta(const BwdParams& p, cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(p.B) * p.n_q * p.H;
  bwd_delta_kernel<T><<<static_cast<unsigned>((rows + 3) / 4), 128, 0, s>>>(p);
  MLA_LAUNCH_CHECK("bwd_delta");
  return MLA_OK;
}

template <typename T>
mla_status launch_bwd_simt(const BwdParams& p, cudaStream_t s) {
  dim3 gq(ceil_div(p.n_q, 4), p.H, p.B);
  bwd_dq_kernel<T><<<gq, 128, 0, s>>>(p);
  MLA_LAUNCH_CHECK("bwd_dq");
  dim3 gk(ceil_div(p.nc + p.n_q, 4), p.B);
  bwd_dkey_kernel<T><<<gk, 128, 4 * p.D * sizeof(float), s>>>(p);
  MLA_LAUNCH_CHECK("bwd_dkey");
  return MLA_OK;
}

}  // namespace

BwdWorkspace bwd_workspace_layout(const Dims& d, int n_valid) {
  BwdWorkspace w;
  w.delta_bytes = static_cast<size_t>(round_up(d.B * d.H * d.n_q, 64)) * sizeof(float);
  w.keys = key_workspace_layout(d, n_valid);
  w.groups = tc_bwd_supported(d) ? bwd_tc_head_groups(d, n_valid) : 0;
  w.keys_tc_bytes = w.groups > 0 ? static_cast<size_t>(d.B) * w.keys.rows * kBwdKeyWidth * 2 : 0;
  w.partial_bytes = static_cast<size_t>(w.groups) * d.B * w.keys.rows * d.D * sizeof(float);
  w.bytes = w.delta_bytes + w.keys.bytes + w.keys_tc_bytes + w.partial_bytes;
  return w;
}

mla_status attention_bwd(const Dims& d, const BwdArgs& a, int n_valid, int first_frame,
                         void* workspace, int32_t* dev_status, cudaStream_t s) {
  if (d.D > 32 * kLanesMax) MLA_FAIL(MLA_ERR_UNSUPPORTED, "d_c + d_rope above %d", 32 * kLanesMax);
  const BwdWorkspace w = bwd_workspace_layout(d, n_valid);
  float* delta = static_cast<float*>(workspace);
  void* ws_rope = static_cast<char*>(workspace) + w.delta_bytes;
  const mla_status st = build_rope_keys(d, a.cache, a.chunk_lat, a.slot_frame, n_valid,
                                       first_frame, ws_rope, s, kRopeKeysAll, dev_status, 1);
  if (st != MLA_OK) return st;
  BwdParams p;
  p.q = a.q; p.chunk_lat = a.chunk_lat; p.cache = a.cache; p.slot_frame = a.slot_frame;
  p.ws_rope = ws_rope; p.o_lat = a.o_lat; p.lse = a.lse; p.d_o_lat = a.d_o_lat; p.delta = delta;
  p.d_q = a.d_q; p.d_chunk_lat = a.d_chunk_lat; p.d_cache = a.d_cache;
  p.B = d.B; p.H = d.H; p.n_q = d.n_q; p.D = d.D; p.d_c = d.d_c; p.d_rope = d.d_rope; p.W = d.W;
  p.tpf = d.tpf; p.frame_w = d.frame_w; p.nc = w.keys.nc; p.nc_pad = w.keys.nc_pad;
  p.rows_ws = w.keys.rows; p.first_frame = first_frame;
  p.scale = d.scale; p.scale_log2 = d.scale * 1.4426950408889634f; p.rope = rope_geom(d);
  mla_status r = d.dtype == MLA_FP32 ? launch_delta<float>(p, s) : launch_delta<bf16>(p, s);
  if (r != MLA_OK) return r;
  if (w.groups > 0) {
    void* keys_tc = static_cast<char*>(ws_rope) + w.keys.bytes;
    float* partial = reinterpret_cast<float*>(static_cast<char*>(keys_tc) + w.keys_tc_bytes);
    return attention_bwd_tc(d, a, n_valid, first_frame, delta, ws_rope, keys_tc, partial,
                            w.groups, dev_status, s);
  }
  return d.dtype == MLA_FP32 ? launch_bwd_simt<float>(p, s) : launch_bwd_simt<bf16>(p, s);
}

}  // namespace mla
