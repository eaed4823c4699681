// kda_decode.cu -- one-token KDA state update, streamed from HBM.
//
// Per (sequence, head), with D = Diag(exp max(g, lb)):
//   w = (D S)^T k,  y = (D S)^T q,  u = beta (v - w)
//   S' = D S + k u^T                 (written back in place)
//   o  = scale S'^T q = scale (y + u (k . q))
// ("Kimi K3 深度拆解", section 4.2: a fixed-size state, O(d_k d_v) work per token
// independent of the position; channel-wise decay per "Kimi K3 技術報告：三個架構
// 改動", section "長度".)
//
// The state is read once and written once: each thread keeps its part of S in
// registers between the column reductions and the rank-1 update. One CTA of
// 8 warps owns one (sequence, head); warp w holds rows w, w+8, ...; lane l
// holds columns [l*V, l*V+V) with V = d_v/32 (a 128-bit access for d_v = 128).
// No tensor cores: 8 bytes of state traffic per ~7 flops is HBM-bound.
// The optional raw-input prologue (q/k L2 normalisation, log decay lb * sigmoid(a))
// is applied to the token's inputs on the fly.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int NW = 8;

template <int V>
struct Vec;
template <>
struct Vec<4> {
  using T = float4;
  __device__ static void ld(const float* p, float (&x)[4]) {
    const float4 t = __ldcs(reinterpret_cast<const float4*>(p));
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
  }
  __device__ static void st(float* p, const float (&x)[4]) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
  }
};
template <>
struct Vec<2> {
  __device__ static void ld(const float* p, float (&x)[2]) {
    const float2 t = __ldcs(reinterpret_cast<const float2*>(p));
    x[0] = t.x; x[1] = t.y;
  }
  __device__ static void st(float* p, const float (&x)[2]) {
    __stcs(reinterpret_cast<float2*>(p), make_float2(x[0], x[1]));
  }
};

// PRO: the raw-input prologue flags (KDA_PROLOGUE_*), a template parameter so the plain
// instance carries no trace of it.
template <typename Tin, int DK, int DV, int PRO>
__global__ void __launch_bounds__(NW * 32, 2) decode_kernel(DecodeArgs a) {
  constexpr int V = DV / 32;    // columns per lane
  constexpr int R = DK / NW;    // rows per warp
  __shared__ float sk[DK], sq[DK], sdec[DK], sv[DV];
  __shared__ float red[2][NW][DV];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n = blockIdx.x / a.H, h = blockIdx.x % a.H;
  const int64_t slot = a.slots ? (int64_t)a.slots[n] : (int64_t)n;
  if (slot < 0 || slot >= a.n_slots) {
    // a state_slots entry the host could not see: no state is touched, the output row
    // becomes NaN (never stale values) and the caller's status word, if any, says why
    if (warp == 0) {
      Tin* o = static_cast<Tin*>(a.out) + ((int64_t)n * a.H + h) * DV + lane * V;
#pragma unroll
      for (int c = 0; c < V; ++c) st_out(o + c, __int_as_float(0x7fc00000));
      if (lane == 0 && a.status != nullptr) atomicExch(a.status, kDevBadSlot);
    }
    return;
  }
  float* S = a.state + (slot * a.H + h) * (int64_t)DK * DV;

  // Issue the state loads first so they are in flight while the token loads land.
  float x[R][V];
#pragma unroll
  for (int rr = 0; rr < R; ++rr) Vec<V>::ld(S + (int64_t)(warp + NW * rr) * DV + lane * V, x[rr]);

  const int64_t tok = (int64_t)n * a.H + h;
  const Tin* q = static_cast<const Tin*>(a.q) + tok * DK;
  const Tin* k = static_cast<const Tin*>(a.k) + tok * DK;
  const Tin* g = static_cast<const Tin*>(a.g) + tok * DK;
  const Tin* v = static_cast<const Tin*>(a.v) + tok * DV;
  for (int i = threadIdx.x; i < DK; i += NW * 32) {
    sk[i] = ld_in(k + i);
    sq[i] = ld_in(q + i);
    float gi = ld_in(g + i);
    if (PRO & KDA_PROLOGUE_GATE_SIGMOID) gi = gate_from_preact(gi, a.lb);
    sdec[i] = expf(fmaxf(gi, a.lb));
  }
  for (int j = threadIdx.x; j < DV; j += NW * 32) sv[j] = ld_in(v + j);
  const float b = ld_in(static_cast<const Tin*>(a.beta) + tok);
  __syncthreads();
  // prologue: raw q and k rows are used divided by their L2 norms (every warp forms
  // the two norms itself, from shared memory)
  float rk = 1.f, rq = 1.f;
  if (PRO & KDA_PROLOGUE_QK_L2NORM) {
    float ssk = 0.f, ssq = 0.f;
    for (int i = lane; i < DK; i += 32) {
      ssk = fmaf(sk[i], sk[i], ssk);
      ssq = fmaf(sq[i], sq[i], ssq);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      ssk += __shfl_xor_sync(0xffffffffu, ssk, off);
      ssq += __shfl_xor_sync(0xffffffffu, ssq, off);
    }
    rk = inv_l2(ssk);
    rq = inv_l2(ssq);
  }

  float pw[V], py[V];
#pragma unroll
  for (int c = 0; c < V; ++c) pw[c] = py[c] = 0.f;
#pragma unroll
  for (int rr = 0; rr < R; ++rr) {
    const int i = warp + NW * rr;
    const float d = sdec[i], ki = sk[i] * rk, qi = sq[i] * rq;
#pragma unroll
    for (int c = 0; c < V; ++c) {
      x[rr][c] *= d;
      pw[c] = fmaf(ki, x[rr][c], pw[c]);
      py[c] = fmaf(qi, x[rr][c], py[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < V; ++c) {
    red[0][warp][lane * V + c] = pw[c];
    red[1][warp][lane * V + c] = py[c];
  }
  __syncthreads();

  float u[V];
#pragma unroll
  for (int c = 0; c < V; ++c) {
    float w = 0.f;
#pragma unroll
    for (int ww = 0; ww < NW; ++ww) w += red[0][ww][lane * V + c];
    u[c] = b * (sv[lane * V + c] - w);
  }
#pragma unroll
  for (int rr = 0; rr < R; ++rr) {
    const float ki = sk[warp + NW * rr] * rk;
#pragma unroll
    for (int c = 0; c < V; ++c) x[rr][c] = fmaf(ki, u[c], x[rr][c]);
    Vec<V>::st(S + (int64_t)(warp + NW * rr) * DV + lane * V, x[rr]);
  }

  if (warp == 0) {
    float kq = 0.f;
    for (int i = lane; i < DK; i += 32) kq = fmaf(sk[i], sq[i], kq);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
    kq *= rk * rq;
    Tin* o = static_cast<Tin*>(a.out) + tok * DV + lane * V;
#pragma unroll
    for (int c = 0; c < V; ++c) {
      float y = 0.f;
#pragma unroll
      for (int ww = 0; ww < NW; ++ww) y += red[1][ww][lane * V + c];
      st_out(o + c, a.scale * (y + u[c] * kq));
    }
  }
}

template <typename Tin, int PRO>
void launch_dims(const DecodeArgs& a, dim3 grid, dim3 block, cudaStream_t st) {
  if (a.dk == 128 && a.dv == 128) decode_kernel<Tin, 128, 128, PRO><<<grid, block, 0, st>>>(a);
  else if (a.dk == 128 && a.dv == 64) decode_kernel<Tin, 128, 64, PRO><<<grid, block, 0, st>>>(a);
  else if (a.dk == 64 && a.dv == 128) decode_kernel<Tin, 64, 128, PRO><<<grid, block, 0, st>>>(a);
  else decode_kernel<Tin, 64, 64, PRO><<<grid, block, 0, st>>>(a);
}

template <typename Tin>
cudaError_t launch_typed(const DecodeArgs& a, cudaStream_t st) {
  const int64_t blocks = (int64_t)a.N * a.H;
  if (blocks == 0) return cudaSuccess;
  const dim3 grid((unsigned)blocks), block(NW * 32);
  switch (a.prologue) {
    case 0: launch_dims<Tin, 0>(a, grid, block, st); break;
    case 1: launch_dims<Tin, 1>(a, grid, block, st); break;
    case 2: launch_dims<Tin, 2>(a, grid, block, st); break;
    default: launch_dims<Tin, 3>(a, grid, block, st); break;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, kda_dtype dtype, cudaStream_t st) {
  return dtype == KDA_F32 ? launch_typed<float>(a, st) : launch_typed<__nv_bfloat16>(a, st);
}

}  // namespace kda
