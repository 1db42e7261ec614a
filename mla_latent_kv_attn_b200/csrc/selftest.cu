// selftest.cu - exercises the device-side failure path of the tensor-core kernels without
// faulting anything: one thread waits, with the kernels' bounded-wait helper, on an mbarrier
// that nothing ever arrives on; the wait runs out and the kernel reports it in dev_status.
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

}  // namespace

}  // namespace mla

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
