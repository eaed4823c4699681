// kda_api.cu -- the C ABI (include/kda.h): argument validation, workspace
// layout and dispatch to the kernels. Nothing here allocates device memory or
// synchronises a stream (except kda_workspace_status, a diagnostic).
#include <math.h>

#include "kda_internal.cuh"

namespace kda {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool dims_supported(int d) { return d == 64 || d == 128; }

// Common shape checks; fills the resolved fields used by the kernels.
kda_status check_shape(const kda_shape* s, bool prefill) {
  if (s == nullptr) return KDA_ERR_INVALID_ARG;
  if (s->dtype != KDA_F32 && s->dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (s->H <= 0 || s->B <= 0 || s->T < 0 || s->dk <= 0 || s->dv <= 0) return KDA_ERR_INVALID_ARG;
  if (!(s->scale >= 0.f) || !isfinite(s->scale)) return KDA_ERR_INVALID_ARG;
  if (!isfinite(s->g_lower_bound) || !(s->g_lower_bound < 0.f)) return KDA_ERR_INVALID_ARG;
  if (s->prologue & ~(KDA_PROLOGUE_QK_L2NORM | KDA_PROLOGUE_GATE_SIGMOID))
    return KDA_ERR_INVALID_ARG;
  if (!dims_supported(s->dk) || !dims_supported(s->dv)) return KDA_ERR_UNSUPPORTED;
  if (prefill) {
    if (s->chunk != kChunk) return KDA_ERR_UNSUPPORTED;
    // exp(-cumsum) over a chunk must stay finite in fp32 and bf16.
    if ((double)s->g_lower_bound * kChunk < -80.0) return KDA_ERR_UNSUPPORTED;
  }
  return KDA_OK;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Packed-token view of a shape: cu_seqlens mode when n_seqs > 0, batch mode otherwise.
void resolve(const kda_shape& s, int64_t& T_total, int& n_seqs, int64_t& max_len) {
  if (s.n_seqs > 0) {
    T_total = s.T;
    n_seqs = s.n_seqs;
    max_len = s.max_seqlen > 0 ? s.max_seqlen : s.T;
  } else {
    T_total = s.T * static_cast<int64_t>(s.B);
    n_seqs = s.B;
    max_len = s.T;
  }
}

}  // namespace
}  // namespace kda

using namespace kda;

extern "C" {

size_t kda_chunk_fwd_workspace_size(const kda_shape* shape) {
  if (check_shape(shape, true) != KDA_OK) return 0;
  if (shape->n_seqs < 0 || shape->max_seqlen < 0 || (shape->n_seqs > 0 && shape->B != 1)) return 0;
  int64_t T_total, max_len;
  int n_seqs;
  resolve(*shape, T_total, n_seqs, max_len);
  if (tc_path_applies(*shape, T_total))
    return align_up(tc_plan(T_total, n_seqs, shape->H, max_len).ws_bytes, 256);
  return align_up(kWorkspaceHeader, 256);
}

}  // extern "C"

namespace kda {
namespace {

// kda_chunk_fwd, with chunk-boundary snapshots when snaps != nullptr (snap_every >= 1,
// checked by the caller).
kda_status chunk_fwd(const void* q, const void* k, const void* v, const void* g,
                     const void* beta, const float* initial_state, const int32_t* cu_seqlens,
                     void* out, float* final_state, int snap_every, float* snaps,
                     int64_t n_snaps, const kda_shape* shape, void* workspace,
                     size_t workspace_bytes, kda_stream_t stream) {
  kda_status st = check_shape(shape, true);
  if (st != KDA_OK) return st;
  const kda_shape& s = *shape;
  // cu_seqlens mode needs B == 1 and n_seqs > 0; batch mode needs n_seqs == 0
  if ((cu_seqlens != nullptr) != (s.n_seqs > 0)) return KDA_ERR_INVALID_ARG;
  if (cu_seqlens != nullptr && s.B != 1) return KDA_ERR_INVALID_ARG;
  if (s.n_seqs < 0 || s.max_seqlen < 0) return KDA_ERR_INVALID_ARG;
  int n_seqs;
  int64_t T_total, max_len;
  resolve(s, T_total, n_seqs, max_len);
  const void* tensors[] = {q, k, v, g, beta, out};
  for (const void* p : tensors) {
    if (T_total > 0 && p == nullptr) return KDA_ERR_INVALID_ARG;
    if (!aligned16(p)) return KDA_ERR_INVALID_ARG;
  }
  if (!aligned16(initial_state) || !aligned16(final_state) || !aligned16(cu_seqlens))
    return KDA_ERR_INVALID_ARG;
  if (cu_seqlens != nullptr && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return KDA_ERR_INVALID_ARG;
  if (snap_every > 0) {
    const int64_t need_snaps = T_total / (static_cast<int64_t>(snap_every) * kChunk);
    if (n_snaps < need_snaps || (need_snaps > 0 && snaps == nullptr) || !aligned16(snaps))
      return KDA_ERR_INVALID_ARG;
    if (need_snaps == 0) snaps = nullptr;
  }
  const size_t need = kda_chunk_fwd_workspace_size(shape);
  if (workspace == nullptr || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return KDA_ERR_INVALID_ARG;

  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, kWorkspaceHeader, cs) != cudaSuccess) return KDA_ERR_CUDA;

  PrefillArgs a{};
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta;
  a.s0 = initial_state;
  a.cu = cu_seqlens;
  a.out = out;
  a.sT = final_state;
  a.snap = snap_every > 0 ? snaps : nullptr;
  a.snap_every = snap_every > 0 ? snap_every : 1;
  a.status = static_cast<int32_t*>(workspace);
  a.ws = static_cast<unsigned char*>(workspace);
  a.ws_bytes = workspace_bytes;
  a.T = s.T;
  a.T_total = T_total;
  a.max_len = max_len;
  a.n_seqs = n_seqs;
  a.H = s.H; a.dk = s.dk; a.dv = s.dv;
  a.scale = s.scale > 0.f ? s.scale : 1.0f / sqrtf((float)s.dk);
  a.lb = s.g_lower_bound;
  a.prologue = s.prologue;

  cudaError_t e = tc_path_applies(s, T_total) ? launch_prefill_tc(a, cs)
                                              : launch_prefill_simt(a, s.dtype, cs);
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace
}  // namespace kda

extern "C" {

kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const void* g,
                         const void* beta, const float* initial_state,
                         const int32_t* cu_seqlens, void* out, float* final_state,
                         const kda_shape* shape, void* workspace, size_t workspace_bytes,
                         kda_stream_t stream) {
  return chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state, 0, nullptr,
                   0, shape, workspace, workspace_bytes, stream);
}

kda_status kda_chunk_fwd_snapshots(const void* q, const void* k, const void* v, const void* g,
                                   const void* beta, const float* initial_state,
                                   const int32_t* cu_seqlens, void* out, float* final_state,
                                   int32_t snapshot_chunks, float* snapshots,
                                   int64_t n_snapshots, const kda_shape* shape,
                                   void* workspace, size_t workspace_bytes,
                                   kda_stream_t stream) {
  if (snapshot_chunks < 1) return KDA_ERR_INVALID_ARG;
  return chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state,
                   snapshot_chunks, snapshots, n_snapshots, shape, workspace, workspace_bytes,
                   stream);
}

}  // extern "C"

namespace kda {
namespace {

// Backward workspace: [forward workspace (status word first) | per-chunk snapshots |
// forward output scratch], each 256-byte aligned. The fp32 accumulators of dq, dk, dg,
// dbeta reuse the forward workspace after its status header: they are zeroed only after
// the forward has run (same stream), when its tiles are dead; the first region is as large
// as the larger of the two.
struct BwdPlan {
  size_t snaps, out, acc_q, acc_k, acc_g, acc_b, total;
  int64_t n_snaps;
};

bool bwd_plan(const kda_shape* shape, BwdPlan& p) {
  if (check_shape(shape, true) != KDA_OK) return false;
  const size_t fwd = kda_chunk_fwd_workspace_size(shape);
  if (fwd == 0) return false;
  int64_t T_total, max_len;
  int n_seqs;
  resolve(*shape, T_total, n_seqs, max_len);
  const size_t elem = shape->dtype == KDA_F32 ? 4 : 2;
  const size_t th = static_cast<size_t>(T_total) * shape->H;
  p.n_snaps = T_total / kChunk;
  p.acc_q = align_up(kWorkspaceHeader, 256);
  p.acc_k = p.acc_q + align_up(th * shape->dk * 4, 256);
  p.acc_g = p.acc_k + align_up(th * shape->dk * 4, 256);
  p.acc_b = p.acc_g + align_up(th * shape->dk * 4, 256);
  const size_t acc_end = p.acc_b + align_up(th * 4, 256);
  p.snaps = align_up(fwd > acc_end ? fwd : acc_end, 256);
  p.out = align_up(p.snaps + static_cast<size_t>(p.n_snaps) * shape->H * shape->dk * shape->dv * 4, 256);
  p.total = align_up(p.out + th * shape->dv * elem, 256);
  return true;
}

}  // namespace
}  // namespace kda

extern "C" {

size_t kda_chunk_bwd_workspace_size(const kda_shape* shape) {
  BwdPlan p;
  return bwd_plan(shape, p) ? p.total : 0;
}

kda_status kda_chunk_bwd(const void* q, const void* k, const void* v, const void* g,
                         const void* beta, const float* initial_state,
                         const int32_t* cu_seqlens, const void* d_out,
                         const float* d_final_state, void* dq, void* dk, void* dv, void* dg,
                         void* dbeta, float* d_initial_state, const kda_shape* shape,
                         void* workspace, size_t workspace_bytes, kda_stream_t stream) {
  kda_status st = check_shape(shape, true);
  if (st != KDA_OK) return st;
  const kda_shape& s = *shape;
  if ((cu_seqlens != nullptr) != (s.n_seqs > 0)) return KDA_ERR_INVALID_ARG;
  if (cu_seqlens != nullptr && s.B != 1) return KDA_ERR_INVALID_ARG;
  if (s.n_seqs < 0 || s.max_seqlen < 0) return KDA_ERR_INVALID_ARG;
  int n_seqs;
  int64_t T_total, max_len;
  resolve(s, T_total, n_seqs, max_len);
  const void* tensors[] = {q, k, v, g, beta, dq, dk, dv, dg, dbeta};
  for (const void* p : tensors) {
    if (T_total > 0 && p == nullptr) return KDA_ERR_INVALID_ARG;
    if (!aligned16(p)) return KDA_ERR_INVALID_ARG;
  }
  if (!aligned16(initial_state) || !aligned16(d_out) || !aligned16(d_final_state) ||
      !aligned16(d_initial_state) || !aligned16(cu_seqlens))
    return KDA_ERR_INVALID_ARG;
  BwdPlan p;
  if (!bwd_plan(shape, p)) return KDA_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < p.total ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return KDA_ERR_INVALID_ARG;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  // forward pass keeping the state after every chunk (its outputs go to scratch)
  float* snaps = reinterpret_cast<float*>(ws + p.snaps);
  st = chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, ws + p.out, nullptr, 1, snaps,
                 p.n_snaps, shape, ws, p.snaps, stream);
  if (st != KDA_OK) return st;
  if (cudaMemsetAsync(ws + p.acc_q, 0, p.snaps - p.acc_q, cs) != cudaSuccess) return KDA_ERR_CUDA;

  BackwardArgs a{};
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta;
  a.dout = d_out;
  a.s0 = initial_state;
  a.dsT = d_final_state;
  a.snap = snaps;
  a.cu = cu_seqlens;
  a.acc_q = reinterpret_cast<float*>(ws + p.acc_q);
  a.acc_k = reinterpret_cast<float*>(ws + p.acc_k);
  a.acc_g = reinterpret_cast<float*>(ws + p.acc_g);
  a.acc_b = reinterpret_cast<float*>(ws + p.acc_b);
  a.dv_out = dv;
  a.ds0 = d_initial_state;
  a.status = static_cast<int32_t*>(workspace);
  a.T = s.T;
  a.T_total = T_total;
  a.n_seqs = n_seqs;
  a.H = s.H; a.dk = s.dk; a.dv = s.dv;
  a.scale = s.scale > 0.f ? s.scale : 1.0f / sqrtf((float)s.dk);
  a.lb = s.g_lower_bound;
  a.prologue = s.prologue;
  cudaError_t e = launch_backward(a, s.dtype, cs);
  if (e == cudaSuccess) e = launch_backward_finish(a, dq, dk, dg, dbeta, s.dtype, cs);
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int64_t kda_snapshot_count(const kda_shape* shape, int32_t snapshot_chunks) {
  if (snapshot_chunks < 1 || kda_chunk_fwd_workspace_size(shape) == 0) return -1;
  int64_t T_total, max_len;
  int n_seqs;
  resolve(*shape, T_total, n_seqs, max_len);
  return T_total / (static_cast<int64_t>(snapshot_chunks) * kChunk);
}

kda_status kda_decode_step(const void* q, const void* k, const void* v, const void* g,
                           const void* beta, float* state, const int32_t* state_slots,
                           int64_t n_slots, void* out, const kda_shape* shape,
                           int32_t* status, kda_stream_t stream) {
  kda_status st = check_shape(shape, false);
  if (st != KDA_OK) return st;
  const kda_shape& s = *shape;
  if (s.T != 1) return KDA_ERR_INVALID_ARG;
  if (n_slots <= 0 || (state_slots == nullptr && n_slots < s.B)) return KDA_ERR_INVALID_ARG;
  const void* tensors[] = {q, k, v, g, beta, out, state};
  for (const void* p : tensors)
    if (p == nullptr || !aligned16(p)) return KDA_ERR_INVALID_ARG;
  if (state_slots != nullptr && (reinterpret_cast<uintptr_t>(state_slots) & 3u))
    return KDA_ERR_INVALID_ARG;
  if (status != nullptr && (reinterpret_cast<uintptr_t>(status) & 3u)) return KDA_ERR_INVALID_ARG;

  DecodeArgs a{};
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta;
  a.state = state;
  a.slots = state_slots;
  a.n_slots = n_slots;
  a.out = out;
  a.status = status;
  a.N = s.B; a.H = s.H; a.dk = s.dk; a.dv = s.dv;
  a.scale = s.scale > 0.f ? s.scale : 1.0f / sqrtf((float)s.dk);
  a.lb = s.g_lower_bound;
  a.prologue = s.prologue;
  cudaError_t e = launch_decode(a, s.dtype, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_workspace_status(const void* workspace, size_t workspace_bytes,
                                kda_stream_t stream, int32_t* device_code) {
  if (workspace == nullptr) {
    // the status word of kda_chunk_fwd_noalloc's fixed array on the current device
    void* p = nullptr;
    const kda_status st = noalloc_scratch_address(&p);
    if (st != KDA_OK) return st;
    workspace = p;
  } else if (workspace_bytes < sizeof(int32_t)) {
    return KDA_ERR_INVALID_ARG;
  }
  int32_t code = 0;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&code, workspace, sizeof code, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return KDA_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return KDA_ERR_CUDA;
  if (device_code) *device_code = code;
  return code == kDevOk ? KDA_OK : KDA_ERR_DEVICE;
}

const char* kda_status_string(kda_status status) {
  switch (status) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: invalid argument";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: unsupported shape or parameter";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: CUDA launch or query failed";
    case KDA_ERR_DEVICE: return "KDA_ERR_DEVICE: device-side check failed";
  }
  return "KDA_ERR_UNKNOWN";
}

const char* kda_version(void) { return "0.1.0"; }

}  // extern "C"
