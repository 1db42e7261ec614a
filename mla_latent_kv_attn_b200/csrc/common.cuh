// common.cuh - status plumbing, dtype helpers and small device utilities shared by the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <string>

#include "mla.h"

namespace mla {

// ---- host-side error reporting ---------------------------------------------------------------

void set_last_error(const std::string& msg);  // per host thread (mla_abi.cu)

#define MLA_FAIL(code, ...)                                      \
  do {                                                           \
    char _buf[512];                                              \
    snprintf(_buf, sizeof(_buf), __VA_ARGS__);                   \
    ::mla::set_last_error(_buf);                                 \
    return (code);                                               \
  } while (0)

#define MLA_CHECK_ARG(cond, ...) \
  do {                           \
    if (!(cond)) MLA_FAIL(MLA_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

#define MLA_CUDA_TRY(expr)                                                               \
  do {                                                                                   \
    cudaError_t _e = (expr);                                                             \
    if (_e != cudaSuccess)                                                               \
      MLA_FAIL(MLA_ERR_CUDA, "%s failed: %s (%s:%d)", #expr, cudaGetErrorString(_e),     \
               __FILE__, __LINE__);                                                      \
  } while (0)

// Checks the launch just issued.
#define MLA_LAUNCH_CHECK(what)                                                           \
  do {                                                                                   \
    cudaError_t _e = cudaGetLastError();                                                 \
    if (_e != cudaSuccess)                                                               \
      MLA_FAIL(MLA_ERR_CUDA, "launch of %s failed: %s", what, cudaGetErrorString(_e));  \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- NVTX ranges (built in only with -DMLA_NVTX; header-only NVTX 3, no link dependency) -----

#ifdef MLA_NVTX
}  // namespace mla
#include <nvtx3/nvToolsExt.h>
namespace mla {
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
#define MLA_NVTX_RANGE(name) ::mla::NvtxRange mla_nvtx_range_(name)
#else
#define MLA_NVTX_RANGE(name) \
  do {                       \
  } while (0)
#endif

// ---- element types ---------------------------------------------------------------------------

using bf16 = __nv_bfloat16;

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<bf16> {
  static __device__ __forceinline__ float to_f(bf16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ bf16 from_f(float v) { return __float2bfloat16_rn(v); }
};

template <typename T> __device__ __forceinline__ float ld_f(const T* p) { return Elem<T>::to_f(*p); }
template <typename T> __device__ __forceinline__ void st_f(T* p, float v) { *p = Elem<T>::from_f(v); }

inline size_t dtype_size(int32_t dtype) { return dtype == MLA_FP32 ? 4 : 2; }

// ---- derived sizes ---------------------------------------------------------------------------

struct Dims {
  int B, H, d_model, d_head, d_c, d_rope, D, d_cq, tpf, n_q, W, C, frame_w;
  int pt, ph, pw;
  float rope_base, scale;
  int dtype, path;
};

inline Dims dims_of(const mla_config& c) {
  Dims d;
  d.B = c.batch; d.H = c.n_heads; d.d_model = c.d_model; d.d_head = c.d_head; d.d_c = c.d_c;
  d.d_rope = c.d_rope; d.D = c.d_c + c.d_rope; d.d_cq = c.d_cq;
  d.tpf = c.frame_h * c.frame_w; d.n_q = c.chunk_frames * d.tpf; d.W = c.window_frames;
  d.C = c.chunk_frames; d.frame_w = c.frame_w;
  d.pt = c.rope_pairs_t; d.ph = c.rope_pairs_h; d.pw = c.rope_pairs_w;
  d.rope_base = c.rope_base; d.scale = c.softmax_scale; d.dtype = c.dtype; d.path = c.kernel_path;
  return d;
}

// Geometry of the rotary bands, passed by value to kernels.  inv_freq[pair] =
// rope_base^(-i / n_axis) for pair i of its axis band, computed on the host in double.
constexpr int kMaxRopePairs = 64;
struct RopeGeom {
  int pt, ph, pw;        // pairs per axis
  int frame_w, tpf;
  float inv_freq[kMaxRopePairs];
};

inline RopeGeom rope_geom(const Dims& d) {
  RopeGeom g{};
  g.pt = d.pt; g.ph = d.ph; g.pw = d.pw; g.frame_w = d.frame_w; g.tpf = d.tpf;
  const int n_axis[3] = {d.pt, d.ph, d.pw};
  int pair = 0;
  for (int a = 0; a < 3; ++a)
    for (int i = 0; i < n_axis[a] && pair < kMaxRopePairs; ++i, ++pair)
      g.inv_freq[pair] = static_cast<float>(
          std::pow(static_cast<double>(d.rope_base), -static_cast<double>(i) / n_axis[a]));
  return g;
}

// Angle of rotary pair `pair` (0 .. pt+ph+pw-1) at position (t, h, w):
// pos_axis * base^(-i / n_axis), i the pair's index inside its axis band.
__device__ __forceinline__ float rope_angle(const RopeGeom& g, int pair, int t, int h, int w) {
  const int pos = pair < g.pt ? t : (pair < g.pt + g.ph ? h : w);
  return static_cast<float>(pos) * g.inv_freq[pair];
}

// sin and cos of an angle of moderate size (|a| < 2^15): Cody-Waite reduction by 2*pi
// (2*pi split into its float value and the float remainder) to r in [-pi, pi], then the
// hardware sin/cos approximations, which are accurate on that interval (error ~2^-21).
__device__ __forceinline__ void rope_sincos(float a, float* s, float* c) {
  const float k = rintf(a * 0.159154943091895336f);
  float r = fmaf(-k, 6.28318548202514648f, a);
  r = fmaf(-k, -1.74845553146951724e-7f, r);
  __sincosf(r, s, c);
}

// Rotates one pair (x0, x1) by angle a.
__device__ __forceinline__ void rope_rotate(float& x0, float& x1, float a) {
  float s, c;
  rope_sincos(a, &s, &c);
  const float y0 = x0 * c - x1 * s;
  const float y1 = x0 * s + x1 * c;
  x0 = y0;
  x1 = y1;
}

// (t, h, w) of key m in the walk order of the attention kernels: ring slots 0 .. nc-1 (their
// frame from slot_frame), then the chunk's own tokens (frame first_frame + j / tpf).
__device__ __forceinline__ void key_position(const int32_t* slot_frame, int b, int W, int tpf,
                                             int frame_w, int nc, int first_frame, int m, int& t,
                                             int& h, int& w) {
  int i;
  if (m < nc) {
    t = slot_frame[b * W + m / tpf];
    i = m % tpf;
  } else {
    const int j = m - nc;
    t = first_frame + j / tpf;
    i = j % tpf;
  }
  h = i / frame_w;
  w = i % frame_w;
}

// Device-side contract checks of the MLA_DEBUG build: a failed check writes
// MLA_ERR_DEVICE_CHECK to the caller's status word (if given) and the kernel carries on; nothing
// traps.  In the release build the check compiles to nothing.
__device__ __forceinline__ void debug_check(bool ok, int32_t* dev_status) {
#ifdef MLA_DEBUG
  if (!ok && dev_status != nullptr) atomicExch(dev_status, static_cast<int32_t>(MLA_ERR_DEVICE_CHECK));
#else
  (void)ok;
  (void)dev_status;
#endif
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int round_up(int a, int b) { return ceil_div(a, b) * b; }

}  // namespace mla
