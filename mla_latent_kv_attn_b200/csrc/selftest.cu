// selftest.cu - test-only kernels.
//   - The device-side failure path of the tensor-core kernels, without faulting anything: one
//     thread waits, with the kernels' bounded-wait helper, on an mbarrier that nothing ever
//     arrives on; the wait runs out and the kernel reports it in dev_status.
//   - The library's own approximations, evaluated by the very device functions the kernels
//     call, so that tests can hold them to their error bounds: the softmax's FMA-pipe
//     exponential (exp2_poly_pair, beside the SFU's ex2.approx and CUDA's exp2f), and the
//     3D-RoPE angle and sine/cosine (rope_angle, rope_sincos).
#include "exp2.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mla {

namespace {

__global__ void bounded_wait_selftest_kernel(int32_t* dev_status, long long limit_cycles) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    sm100::mbar_init(sm100::smem_u32(&bar), 1);
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    sm100::mbar_wait_or_abort(sm100::smem_u32(&bar), 0, &abort_flag, dev_status, limit_cycles);
}

// One thread per pair of arguments: (x[2i], x[2i+1]) go through exp2_poly_pair together, as
// in the softmax; an odd tail pairs the last argument with itself.
__global__ void exp2_selftest_kernel(const float* x, float* y_poly, float* y_sfu, float* y_exp2f,
                                     int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int a = 2 * i;
  if (a >= n) return;
  const int b = a + 1 < n ? a + 1 : a;
  float p0, p1;
  exp2_poly_pair(x[a], x[b], p0, p1);
  y_poly[a] = p0;
  y_sfu[a] = fast_exp2(x[a]);
  y_exp2f[a] = exp2f(x[a]);
  if (b != a) {
    y_poly[b] = p1;
    y_sfu[b] = fast_exp2(x[b]);
    y_exp2f[b] = exp2f(x[b]);
  }
}

__global__ void sincos_selftest_kernel(const float* angle, float* s, float* c, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) rope_sincos(angle[i], &s[i], &c[i]);
}

// For every position (t, h, w) and rotary pair: the angle the kernels use and its sine/cosine.
__global__ void rope_selftest_kernel(const int32_t* pos, int n, int n_pairs, RopeGeom g,
                                     float* angle, float* s, float* c) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n * n_pairs) return;
  const int i = e / n_pairs, pair = e % n_pairs;
  const float a = rope_angle(g, pair, pos[3 * i], pos[3 * i + 1], pos[3 * i + 2]);
  angle[e] = a;
  rope_sincos(a, &s[e], &c[e]);
}

// One CTA per SM: thread 0 reads the SM's cycle counter and the global nanosecond timer, spins
// on the timer for spin_ns, and reads both again: out[4 * cta] = {smid, cycles, ns, 0}.
__global__ void sm_clock_probe_kernel(unsigned long long* out, long long spin_ns) {
  if (threadIdx.x != 0) return;
  unsigned long long g0, g1, smid;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(g0));
  const long long c0 = clock64();
  // bounded: at most 2^30 polls however the timer behaves
  for (long long it = 0; it < (1LL << 30); ++it) {
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(g1));
    if (static_cast<long long>(g1 - g0) >= spin_ns) break;
  }
  const long long c1 = clock64();
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(g1));
  unsigned int id;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(id));
  smid = id;
  out[4 * blockIdx.x + 0] = smid;
  out[4 * blockIdx.x + 1] = static_cast<unsigned long long>(c1 - c0);
  out[4 * blockIdx.x + 2] = g1 - g0;
  out[4 * blockIdx.x + 3] = 0ull;
}

mla_status check_device_word(const void* p, const char* name) {
  if (p == nullptr) MLA_FAIL(MLA_ERR_INVALID_ARG, "%s is null", name);
  if ((reinterpret_cast<uintptr_t>(p) & 3u) != 0)
    MLA_FAIL(MLA_ERR_ALIGNMENT, "%s is not 4-byte aligned", name);
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess ||
      (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)) {
    cudaGetLastError();
    MLA_FAIL(MLA_ERR_INVALID_ARG, "%s is not device memory", name);
  }
  return MLA_OK;
}

}  // namespace

}  // namespace mla

#define MLA_SELFTEST_TRY(expr)      \
  do {                              \
    mla_status _s = (expr);         \
    if (_s != MLA_OK) return _s;    \
  } while (0)

extern "C" mla_status mla_selftest_exp2(const float* x, float* y_poly, float* y_sfu,
                                        float* y_exp2f, int32_t n, void* stream) {
  using namespace mla;
  set_last_error("");
  MLA_CHECK_ARG(n >= 0, "n must be >= 0");
  if (n == 0) return MLA_OK;
  MLA_SELFTEST_TRY(check_device_word(x, "x"));
  MLA_SELFTEST_TRY(check_device_word(y_poly, "y_poly"));
  MLA_SELFTEST_TRY(check_device_word(y_sfu, "y_sfu"));
  MLA_SELFTEST_TRY(check_device_word(y_exp2f, "y_exp2f"));
  const int pairs = (n + 1) / 2;
  exp2_selftest_kernel<<<ceil_div(pairs, 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, y_poly, y_sfu, y_exp2f, n);
  MLA_LAUNCH_CHECK("exp2_selftest");
  return MLA_OK;
}

extern "C" mla_status mla_selftest_sincos(const float* angle, float* sin_out, float* cos_out,
                                          int32_t n, void* stream) {
  using namespace mla;
  set_last_error("");
  MLA_CHECK_ARG(n >= 0, "n must be >= 0");
  if (n == 0) return MLA_OK;
  MLA_SELFTEST_TRY(check_device_word(angle, "angle"));
  MLA_SELFTEST_TRY(check_device_word(sin_out, "sin_out"));
  MLA_SELFTEST_TRY(check_device_word(cos_out, "cos_out"));
  sincos_selftest_kernel<<<ceil_div(n, 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      angle, sin_out, cos_out, n);
  MLA_LAUNCH_CHECK("sincos_selftest");
  return MLA_OK;
}

extern "C" mla_status mla_selftest_rope_angles(const mla_config* cfg, const int32_t* pos,
                                               int32_t n, float* angle, float* sin_out,
                                               float* cos_out, void* stream) {
  using namespace mla;
  set_last_error("");
  MLA_SELFTEST_TRY(mla_config_check(cfg));
  const Dims d = dims_of(*cfg);
  const int n_pairs = d.d_rope / 2;
  MLA_CHECK_ARG(n >= 0 && static_cast<int64_t>(n) * n_pairs < (int64_t{1} << 31),
                "n out of range");
  if (n == 0) return MLA_OK;
  MLA_SELFTEST_TRY(check_device_word(pos, "pos"));
  MLA_SELFTEST_TRY(check_device_word(angle, "angle"));
  MLA_SELFTEST_TRY(check_device_word(sin_out, "sin_out"));
  MLA_SELFTEST_TRY(check_device_word(cos_out, "cos_out"));
  const int total = n * n_pairs;
  rope_selftest_kernel<<<ceil_div(total, 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      pos, n, n_pairs, rope_geom(d), angle, sin_out, cos_out);
  MLA_LAUNCH_CHECK("rope_selftest");
  return MLA_OK;
}

extern "C" mla_status mla_selftest_wait_timeout(int32_t* dev_status, int32_t limit_us,
                                                void* stream) {
  using namespace mla;
  set_last_error("");
  MLA_CHECK_ARG(dev_status != nullptr, "dev_status is null");
  MLA_CHECK_ARG(limit_us > 0 && limit_us <= 1000000, "limit_us must be in (0, 1e6]");
  if ((reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0)
    MLA_FAIL(MLA_ERR_ALIGNMENT, "dev_status is not 4-byte aligned");
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, dev_status) != cudaSuccess ||
      (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)) {
    cudaGetLastError();
    MLA_FAIL(MLA_ERR_INVALID_ARG, "dev_status is not device memory");
  }
  int dev = 0, khz = 0;
  MLA_CUDA_TRY(cudaGetDevice(&dev));
  MLA_CUDA_TRY(cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev));
  const long long limit = static_cast<long long>(khz) * limit_us / 1000;
  bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev_status, limit);
  MLA_LAUNCH_CHECK("bounded_wait_selftest");
  return MLA_OK;
}

extern "C" mla_status mla_probe_sm_clock(unsigned long long* out, int32_t n_ctas, int32_t spin_us,
                                         void* stream) {
  using namespace mla;
  set_last_error("");
  MLA_CHECK_ARG(n_ctas > 0 && n_ctas <= 4096, "n_ctas must be in [1, 4096]");
  MLA_CHECK_ARG(spin_us > 0 && spin_us <= 100000, "spin_us must be in (0, 1e5]");
  MLA_SELFTEST_TRY(check_device_word(out, "out"));
  if ((reinterpret_cast<uintptr_t>(out) & 7u) != 0)
    MLA_FAIL(MLA_ERR_ALIGNMENT, "out is not 8-byte aligned");
  sm_clock_probe_kernel<<<n_ctas, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      out, static_cast<long long>(spin_us) * 1000);
  MLA_LAUNCH_CHECK("sm_clock_probe");
  return MLA_OK;
}
