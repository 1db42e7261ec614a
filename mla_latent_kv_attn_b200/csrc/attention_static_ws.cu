// attention_static_ws.cu - mla_attention_fwd for callers that cannot allocate device memory.
//
// mla_attention_fwd needs a caller-provided scratch buffer (the rotated positional keys of every
// attended key).  Some callers have no way to provide one: code that runs while a stream is
// being captured (cudaMalloc is not allowed there), plugins whose host framework hands them only
// their input and output buffers, and deployments that forbid any device allocation after start
// up.  This entry point keeps that scratch in a fixed array that is part of the library image,
// so the call itself allocates nothing.
#include <mutex>

#include "kernels.h"

namespace mla {

namespace {

// Largest scratch the built-in array holds (16 MiB; every device that loads the library keeps it
// reserved until the process exits).  The rotated keys of a call take
// batch * (round_up(n_valid*tpf, 128) + round_up(n_q, 128)) * d_rope * sizeof(T) bytes.
constexpr size_t kStaticScratchBytes = size_t{16} << 20;

// Device-side storage.  In host code this name is only a stand-in for the symbol, never a device
// address: the address is looked up per device with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Looks up (once per device, with that device current) the device address of g_scratch.
mla_status scratch_address(void** out) {
  int dev = -1;
  MLA_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices)
    MLA_FAIL(MLA_ERR_UNSUPPORTED, "device ordinal %d beyond the %d supported", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      MLA_FAIL(MLA_ERR_CUDA, "cudaGetSymbolAddress of the built-in scratch failed: %s",
               cudaGetErrorString(e));
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MLA_OK;
}

}  // namespace

size_t static_scratch_bytes() { return kStaticScratchBytes; }

mla_status attention_fwd_static_scratch(const Dims& d, const AttnArgs& args,
                                        const int32_t* slot_frame, int n_valid, int first_frame,
                                        cudaStream_t s) {
  const KeyWorkspace kw = key_workspace_layout(d, n_valid);
  if (kw.bytes > kStaticScratchBytes)
    MLA_FAIL(MLA_ERR_WORKSPACE,
             "this call needs %zu bytes of scratch; the built-in scratch holds %zu "
             "(use mla_attention_fwd with a caller-provided workspace)",
             kw.bytes, kStaticScratchBytes);
  void* ws = nullptr;
  mla_status st = scratch_address(&ws);
  if (st != MLA_OK) return st;
  // Every row of the scratch that the attention kernels read is rewritten here (padding rows
  // with zeros), so what an earlier call left behind never matters.
  st = build_rope_keys(d, args.cache, args.chunk_lat, slot_frame, n_valid, first_frame, ws, s);
  if (st != MLA_OK) return st;
  AttnArgs a = args;
  a.ws = ws;
  if (d.dtype == MLA_BF16 && d.path == MLA_PATH_AUTO && tc_attention_supported(d, a.w_uv != nullptr))
    return attention_tc(d, a, n_valid, s);
  return attention_simt(d, a, n_valid, s);
}

}  // namespace mla
