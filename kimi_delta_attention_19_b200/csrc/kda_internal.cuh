// kda_internal.cuh -- declarations shared by the library's translation units.
// Not part of the public ABI (that is include/kda.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

constexpr int kChunk = 64;          // chunk length C of the chunked form
constexpr int kWorkspaceHeader = 256;  // bytes: status word + scheduler counters

// Device status word values (first int32 of the workspace).
constexpr int32_t kDevOk = 0;
constexpr int32_t kDevBadSeqlens = 1;   // cu_seqlens not monotone / out of [0, T]
constexpr int32_t kDevWaitTimeout = 2;  // a bounded wait on another CTA gave up
constexpr int32_t kDevBadSlot = 3;      // a decode state_slots entry outside [0, n_slots)

// Everything a prefill launch needs, resolved on the host.
struct PrefillArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* g;
  const void* beta;
  const float* s0;          // [n, H, dk, dv] or null
  const int32_t* cu;        // [n+1] or null (then sequences are [b*T, (b+1)*T))
  void* out;                // [T_total, H, dv]
  float* sT;                // [n, H, dk, dv] or null
  float* snap;              // [floor(T_total / (snap_every C)), H, dk, dv] or null
  int snap_every;           // chunks between snapshots (>= 1 when snap is set)
  int32_t* status;          // device status word (workspace header)
  unsigned char* ws;        // workspace base
  size_t ws_bytes;
  int64_t T;                // tokens per sequence (no cu) or total tokens (cu)
  int64_t T_total;          // total packed tokens
  int64_t max_len;          // bound on one sequence's length
  int n_seqs;
  int H, dk, dv;
  float scale;
  float lb;
  int prologue;             // KDA_PROLOGUE_* flags
};

struct DecodeArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* g;
  const void* beta;
  float* state;
  const int32_t* slots;
  int64_t n_slots;
  void* out;
  int32_t* status;          // caller's device status word, or null
  int N, H, dk, dv;
  float scale;
  float lb;
  int prologue;             // KDA_PROLOGUE_* flags
};

// Everything the backward launch needs, resolved on the host.
struct BackwardArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* g;
  const void* beta;
  const void* dout;         // dL/dout [T_total, H, dv] or null (zeros)
  const float* s0;          // [n, H, dk, dv] or null
  const float* dsT;         // dL/dS_final [n, H, dk, dv] or null (zeros)
  const float* snap;        // state after every full chunk: [floor(T_total / C), H, dk, dv]
  const int32_t* cu;        // [n+1] or null
  float* acc_q;             // fp32 accumulators of the d_v slices' contributions:
  float* acc_k;             //   dq, dk, dg [T_total, H, dk]
  float* acc_g;
  float* acc_b;             //   dbeta [T_total, H]
  void* dv_out;             // dL/dv [T_total, H, dv] (dtype)
  float* ds0;               // dL/dS0 [n, H, dk, dv] or null
  int32_t* status;          // device status word
  int64_t T;
  int64_t T_total;
  int n_seqs;
  int H, dk, dv;
  float scale;
  float lb;
  int prologue;             // KDA_PROLOGUE_* flags (raw inputs)
};

// Sequence bounds [t0, t1) of sequence s; false (and status set) when the
// device-visible cu_seqlens entry is malformed.
template <typename Args>
__device__ __forceinline__ bool seq_bounds(const Args& a, int s, int64_t& t0, int64_t& t1) {
  if (a.cu == nullptr) {
    t0 = (int64_t)s * a.T;
    t1 = t0 + a.T;
    return true;
  }
  const int64_t c0 = a.cu[s], c1 = a.cu[s + 1];
  const bool ok = (c0 >= 0) && (c1 >= c0) && (c1 <= a.T_total) &&
                  (s != 0 || c0 == 0) && (s + 1 != a.n_seqs || c1 == a.T_total);
  if (!ok) {
    atomicExch(a.status, kDevBadSeqlens);
    return false;
  }
  t0 = c0;
  t1 = c1;
  return true;
}

template <typename T>
__device__ __forceinline__ float ld_in(const T* p);
template <>
__device__ __forceinline__ float ld_in<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld_in<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(__ldg(p));
}

// The raw-input prologue (KDA_PROLOGUE_*): log decay from a gate pre-activation,
// lb * sigmoid(a), evaluated without overflow for any a.
__device__ __forceinline__ float gate_from_preact(float a_pre, float lb) {
  const float e = __expf(-fabsf(a_pre));     // in (0, 1]
  const float s = 1.f / (1.f + e);           // sigmoid(|a|)
  return lb * (a_pre >= 0.f ? s : e * s);    // sigmoid(a) = 1 - sigmoid(-a)
}
// 1 / max(||row||, 1e-12) from the row's sum of squares
__device__ __forceinline__ float inv_l2(float sumsq) { return 1.f / fmaxf(sqrtf(sumsq), 1e-12f); }

template <typename T>
__device__ __forceinline__ void st_out(T* p, float x);
template <>
__device__ __forceinline__ void st_out<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void st_out<__nv_bfloat16>(__nv_bfloat16* p, float x) {
  *p = __float2bfloat16_rn(x);
}

// Segment plan of the tensor-core prefill (a pure function of the shape).
struct TcPlan {
  int first_tokens;  // tokens of a sequence's first segment (a multiple of the chunk length)
  int seg_tokens;    // tokens of segment 1 (a multiple of the chunk length)
  int seg_dec;       // segment j >= 1 holds seg_tokens - (j - 1) seg_dec tokens
  int max_segs;      // segments of the longest sequence
  int64_t pairs;     // (sequence, head) pairs
  int64_t n_slots;   // chunk slots: ceil(T_total / chunk) + n_seqs
  bool streamed;      // walk beside the intra-chunk kernel, one CTA per (sequence, head)
  size_t ready_off;   // workspace offset of the per-tile ready flags (streamed schedule)
  size_t tiles_off;  // workspace offset of the per-chunk tiles
  size_t ws_bytes;   // workspace it needs, header included
};
TcPlan tc_plan(int64_t T_total, int n_seqs, int H, int64_t max_len);
bool tc_path_applies(const kda_shape& s, int64_t T_total);

// Launchers (return the cudaGetLastError() of their launches).
cudaError_t launch_prefill_simt(const PrefillArgs& a, kda_dtype dtype, cudaStream_t st);
cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t st);
cudaError_t launch_decode(const DecodeArgs& a, kda_dtype dtype, cudaStream_t st);
cudaError_t launch_backward(const BackwardArgs& a, kda_dtype dtype, cudaStream_t st);
// dq, dk, dg, dbeta from the fp32 accumulators, through the prologue when it is on
cudaError_t launch_backward_finish(const BackwardArgs& a, void* dq, void* dk, void* dg,
                                   void* dbeta, kda_dtype dtype, cudaStream_t st);
// Device address of the no-alloc entry point's fixed scratch array in the current context.
kda_status noalloc_scratch_address(void** out);

}  // namespace kda
