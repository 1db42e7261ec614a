// attention_static_ws.cu - mla_attention_fwd for callers that cannot allocate device memory.
//
// mla_attention_fwd needs a caller-provided scratch buffer (the rotated positional keys of every
// attended key).  Some callers have no way to provide one: plugins whose host framework hands
// them only their input and output buffers, and deployments that forbid any device allocation
// after start-up.  This entry point keeps that scratch in a fixed array that is part of the
// library image, so the call itself allocates nothing.
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"

namespace mla {

namespace {

// Largest scratch the built-in array holds (16 MiB; every device that loads the library keeps it
// reserved until the process exits).  The rotated keys of a call take
// batch * (round_up(n_valid*tpf, 128) + round_up(n_q, 128)) * d_rope * sizeof(T) bytes.
constexpr size_t kStaticScratchBytes = size_t{16} << 20;

// Device-side storage.  In host code this name is only a stand-in for the symbol, never a device
// address: the address is looked up per CUDA context with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

// The array's device address belongs to the context the library's module was loaded into: a
// device reset, or another context made current on the same device, loads the module again at
// another address.  So the looked-up address is cached per context, keyed by the driver's
// context id (unique for the life of the process; a recreated context gets a new one).
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_ctx_once;

void load_ctx_entry_points() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  fn = nullptr;
  if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
  cudaGetLastError();
}

// Id of the calling thread's current context, or 0 when none is current yet.
mla_status current_context_id(unsigned long long* id) {
  std::call_once(g_ctx_once, load_ctx_entry_points);
  if (g_ctx_current == nullptr || g_ctx_id == nullptr)
    MLA_FAIL(MLA_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId unavailable from the driver");
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS)
    MLA_FAIL(MLA_ERR_CUDA, "cuCtxGetCurrent failed");
  *id = 0;
  if (ctx != nullptr && g_ctx_id(ctx, id) != CUDA_SUCCESS)
    MLA_FAIL(MLA_ERR_CUDA, "cuCtxGetId failed");
  return MLA_OK;
}

struct ScratchEntry {
  unsigned long long ctx_id;
  void* ptr;
};
constexpr int kMaxContexts = 64;
std::mutex g_scratch_mutex;
ScratchEntry g_scratch_ptr[kMaxContexts] = {};
int g_scratch_next = 0;   // next entry to fill (round robin once all are used)

// The device address of g_scratch in the current context: looked up once per context with
// cudaGetSymbolAddress (the current device is the one the context belongs to), then cached.
mla_status scratch_address(void** out) {
  unsigned long long id = 0;
  mla_status st = current_context_id(&id);
  if (st != MLA_OK) return st;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (id != 0)
    for (const ScratchEntry& e : g_scratch_ptr)
      if (e.ctx_id == id) {
        *out = e.ptr;
        return MLA_OK;
      }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
  if (e != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    MLA_FAIL(MLA_ERR_CUDA, "cudaGetSymbolAddress of the built-in scratch failed: %s",
             cudaGetErrorString(e));
  }
  if (id == 0) {   // the lookup made the device's primary context current
    st = current_context_id(&id);
    if (st != MLA_OK) return st;
  }
  if (id != 0) {
    g_scratch_ptr[g_scratch_next] = ScratchEntry{id, p};
    g_scratch_next = (g_scratch_next + 1) % kMaxContexts;
  }
  *out = p;
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
  st = build_rope_keys(d, args.cache, args.chunk_lat, slot_frame, n_valid, first_frame, ws, s,
                       kRopeKeysAll, args.dev_status, 1);
  if (st != MLA_OK) return st;
  AttnArgs a = args;
  a.ws = ws;
  return attention_dispatch(d, a, n_valid, s);
}

}  // namespace mla
