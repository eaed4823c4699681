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
#include <mutex>

#include "kda_internal.cuh"

namespace {

constexpr size_t kScratchBytes = KDA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 256;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device. In host code the name
// g_scratch is only a host-side stand-in, so the address must come from the
// runtime, once per device, with that device current.
kda_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return KDA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return KDA_OK;
}

}  // namespace

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
  const kda_status st = scratch_address(&scratch);
  if (st != KDA_OK) return st;
  return kda_chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state, shape,
                       scratch, kScratchBytes, stream);
}
