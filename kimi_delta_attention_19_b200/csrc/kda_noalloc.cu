// kda_noalloc.cu -- kda_chunk_fwd for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: code running while a CUDA graph is being
// captured (allocation is not a capturable operation), plugin hosts that give a
// library no workspace argument, and serving loops where an allocation would
// synchronise the device. kda_chunk_fwd_noalloc serves them by running the
// prefill with its scratch taken from one fixed array in device memory that
// this file defines, instead of from a caller-provided workspace.
//
// The array is a module global: every GPU that loads the library holds
// KDA_NOALLOC_SCRATCH_BYTES of it until the process exits. Every call on a
// device shares that device's array, and the array keeps whatever the previous
// call left there; the prefill clears the parts that must start at zero itself.
// Calls whose work overlaps on the GPU (different streams without ordering)
// race on the array.
#include <cuda.h>

#include <mutex>

#include "kda_internal.cuh"

namespace {

constexpr size_t kScratchBytes = KDA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 256;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// The array's device address is a property of the CUDA context that loaded this
// module, not of the device number: a device reset (a new primary context) or a
// non-primary context made current by the caller loads the module again at
// another address. So the address is cached together with the unique ID of the
// context it was looked up in, and looked up again whenever another context is
// current.
struct Cached {
  void* addr = nullptr;
  unsigned long long ctx_id = 0;
  bool valid = false;
};
std::mutex g_mu;
Cached g_cache[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// ID of the context current on this thread; false when it cannot be told (no
// context yet, or a driver without the query), and the caller then looks up the
// address again.
bool current_context_id(unsigned long long* id) {
  static std::once_flag once;
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

}  // namespace

namespace kda {

// Device address of g_scratch in the context current on this thread. In host code
// the name g_scratch is only a host-side stand-in, so the address must come from
// the runtime (cudaGetSymbolAddress), with that context current.
kda_status noalloc_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  Cached& c = g_cache[dev];
  unsigned long long id = 0;
  const bool known = current_context_id(&id);
  if (!(known && c.valid && c.ctx_id == id)) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return KDA_ERR_CUDA;
    // the lookup makes the runtime's context current if none was: ask again
    c.addr = p;
    c.valid = current_context_id(&c.ctx_id);
  }
  *out = c.addr;
  return KDA_OK;
}

}  // namespace kda

extern "C" kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                            const void* g, const void* beta,
                                            const float* initial_state,
                                            const int32_t* cu_seqlens, void* out,
                                            float* final_state, const kda_shape* shape,
                                            kda_stream_t stream) {
  const size_t need = kda_chunk_fwd_workspace_size(shape);
  if (need == 0) {
    // Invalid or unsupported shape: let the regular entry point report which.
    return kda_chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state, shape,
                         nullptr, 0, stream);
  }
  if (need > kScratchBytes) return KDA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const kda_status st = kda::noalloc_scratch_address(&scratch);
  if (st != KDA_OK) return st;
  return kda_chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state, shape,
                       scratch, kScratchBytes, stream);
}
