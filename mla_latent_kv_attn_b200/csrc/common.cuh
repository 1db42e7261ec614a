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

// Rotates one pair (x0, x1) by the angle whose sine and cosine are s and c.  The rounding steps
// are spelled out (one product rounded, then one fused multiply-add), so every kernel that
// rotates gets the same bits whatever the compiler would contract.
__device__ __forceinline__ void rope_apply(float& x0, float& x1, float s, float c) {
  const float y0 = __fmaf_rn(x0, c, -__fmul_rn(x1, s));
  const float y1 = __fmaf_rn(x0, s, __fmul_rn(x1, c));
  x0 = y0;
  x1 = y1;
}

// Rotates one pair (x0, x1) by angle a.
__device__ __forceinline__ void rope_rotate(float& x0, float& x1, float a) {
  float s, c;
  rope_sincos(a, &s, &c);
  rope_apply(x0, x1, s, c);
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

// Rotated positional key of row r of sample b in the attention's key workspace (kPieces 16-byte
// pieces of d_rope values per row):
//   r <  nc                    ring slot r: RoPE3D of the cache row's k_R at its frame's position
//   nc_pad <= r < nc_pad + n_q chunk token r - nc_pad (from chunk_lat)
//   otherwise                  zeros (tile padding)
// The unrotated values are read as stored (already rounded to T); each pair is rotated in fp32
// and rounded once.  With MLA_DEBUG, ring slots must hold a frame (t >= 0) and, with
// check_window, one of the chunk's window (first_frame - W <= t < first_frame).
template <typename T, int kPieces>
__device__ __forceinline__ void rope_key_row(const T* __restrict__ cache,
                                             const T* __restrict__ chunk_lat,
                                             const int32_t* __restrict__ slot_frame,
                                             T* __restrict__ ws, int b, int r, int W, int D,
                                             int d_c, int n_q, int nc, int nc_pad, int rows_ws,
                                             int first_frame, const RopeGeom& g,
                                             int32_t* dev_status, int check_window) {
  constexpr int kPer = 16 / sizeof(T);          // elements per piece
  constexpr int kDr = kPieces * kPer;
  uint4* dst = reinterpret_cast<uint4*>(ws + (static_cast<int64_t>(b) * rows_ws + r) * kDr);
  const T* src = nullptr;
  int m = -1;
  if (r < nc) {
    m = r;
    src = cache + (static_cast<int64_t>(b) * W * g.tpf + r) * D;
  } else if (r >= nc_pad && r - nc_pad < n_q) {
    m = nc + (r - nc_pad);
    src = chunk_lat + (static_cast<int64_t>(b) * n_q + (r - nc_pad)) * D;
  }
  if (src == nullptr) {
#pragma unroll
    for (int k = 0; k < kPieces; ++k) dst[k] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  uint4 raw[kPieces];
  const uint4* s4 = reinterpret_cast<const uint4*>(src + d_c);
#pragma unroll
  for (int k = 0; k < kPieces; ++k) raw[k] = s4[k];
  int t, h, w;
  key_position(slot_frame, b, W, g.tpf, g.frame_w, nc, first_frame, m, t, h, w);
  if (m < nc)
    debug_check(t >= 0 && (!check_window || (t < first_frame && t >= first_frame - W)), dev_status);
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
    dst[k] = raw[k];
  }
}

// ---- programmatic dependent launch ---------------------------------------------------------
// The forward path's kernels are launched with programmatic stream serialisation: a kernel's
// CTAs may be scheduled while the previous kernel on the stream is still draining, set up
// shared memory, barriers and TMEM, and then block in grid_dep_wait() until that kernel has
// completed and its memory writes are visible.  Every CTA calls grid_dep_wait() before its first
// access to global memory and unconditionally (so a kernel never completes before the one it
// follows), then grid_dep_launch() to let the next kernel be scheduled.  Both are no-ops in a
// kernel launched without the attribute.
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Host: whether launches carry the programmatic-serialisation attribute (on unless the
// environment sets MLA_NO_PDL; read once per process).
bool pdl_enabled();

// Launches kernel<<<grid, block, smem, s>>>(args...) through cudaLaunchKernelEx with the
// programmatic-serialisation attribute (when pdl_enabled()).  Only for kernels that call
// grid_dep_wait() as described above.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int round_up(int a, int b) { return ceil_div(a, b) * b; }

}  // namespace mla
