// kda_prefill_simt.cu -- fp32 CUDA-core chunked prefill.
//
// The chunk-parallel form of the gated delta rule ("Kimi K3 深度拆解", section
// 4.2: chunk-parallel with an inter-chunk recurrence; bounded log decay per
// "3 分钟看懂 Kimi K3", Figure 3), evaluated entirely in fp32 on CUDA cores.
// It serves fp32 inputs, whose accuracy target (relative L2 1e-4) rules out
// bf16/tf32 tensor-core operands.
//
// One CTA owns one (sequence, head, 32-column slice of d_v) and walks the
// sequence's chunks in order. Columns of S evolve independently, so slices
// share nothing but read-only inputs. Per chunk of L <= 64 tokens, with
// Gamma_r the inclusive prefix sum of the clamped log decays:
//   K~ = K*exp(Gamma), K^ = K*exp(-Gamma), Q~ = Q*exp(Gamma)
//   A  = Diag(beta) strict_lower(K~ K^^T),  P = lower_incl(Q~ K^^T)
//   T  = (I + A)^{-1} Diag(beta)                (forward substitution)
//   U  = T (V - K~ S)
//   O  = scale (Q~ S + P U)
//   S  = Diag(exp Gamma_L) S + (K^ * exp Gamma_L)^T U
// When asked, the state after every snap_every-th full chunk of a sequence is also
// written out (prefix-cache snapshots), and raw inputs go through the prologue
// (q/k rows L2-normalised, log decay lb * sigmoid(a) from gate pre-activations).
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int C = kChunk;
constexpr int DVS = 32;   // d_v columns per CTA
constexpr int NT = 256;   // threads per CTA

template <int DK>
struct SimtSmem {
  float Kt[C][DK + 1];  // K~   (rows padded to avoid bank conflicts)
  float Kh[C][DK + 1];  // K^
  float Qt[C][DK + 1];  // Q~
  float A[C][C + 1];
  float P[C][C + 1];
  float Tm[C][C + 1];
  alignas(16) float S[DK][DVS];  // state slice
  alignas(16) float Y[C][DVS];   // V slice, then V - K~ S
  alignas(16) float U[C][DVS];
  float gl[DK];         // exp(Gamma_L) per channel
  float bet[C];
};

// acc[0..3] += a * v (S, Y and U rows are 32 floats, 16-byte aligned: float4 reads)
__device__ __forceinline__ void axpy4(float a, const float* v, float* acc) {
  const float4 x = *reinterpret_cast<const float4*>(v);
  acc[0] = fmaf(a, x.x, acc[0]);
  acc[1] = fmaf(a, x.y, acc[1]);
  acc[2] = fmaf(a, x.z, acc[2]);
  acc[3] = fmaf(a, x.w, acc[3]);
}

// A 16-byte vector of inputs as floats
template <typename T>
__device__ __forceinline__ void unpack_vec(const uint4& u, float (&f)[16 / sizeof(T)]);
template <>
__device__ __forceinline__ void unpack_vec<float>(const uint4& u, float (&f)[4]) {
  f[0] = __uint_as_float(u.x);
  f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z);
  f[3] = __uint_as_float(u.w);
}
template <>
__device__ __forceinline__ void unpack_vec<__nv_bfloat16>(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(w[e] << 16);
    f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
  }
}

template <typename Tin, int DK>
__global__ void __launch_bounds__(NT, 1) prefill_simt_kernel(PrefillArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SimtSmem<DK>& sm = *reinterpret_cast<SimtSmem<DK>*>(smem_raw);
  const int n_slices = a.dv / DVS;
  const int slice = blockIdx.x % n_slices;
  const int h = (blockIdx.x / n_slices) % a.H;
  const int s = blockIdx.x / (n_slices * a.H);
  const int tid = threadIdx.x;
  const int j0 = slice * DVS;
  const int H = a.H, DV = a.dv;

  int64_t t0, t1;
  if (!seq_bounds(a, s, t0, t1)) return;

  const Tin* q = static_cast<const Tin*>(a.q);
  const Tin* k = static_cast<const Tin*>(a.k);
  const Tin* v = static_cast<const Tin*>(a.v);
  const Tin* g = static_cast<const Tin*>(a.g);
  const Tin* beta = static_cast<const Tin*>(a.beta);
  Tin* out = static_cast<Tin*>(a.out);
  const int64_t state_base = ((int64_t)s * H + h) * DK * DV + j0;

  for (int e = tid; e < DK * DVS; e += NT) {
    const int i = e / DVS, c = e % DVS;
    sm.S[i][c] = a.s0 ? a.s0[state_base + (int64_t)i * DV + c] : 0.f;
  }
  __syncthreads();

  for (int64_t c0 = t0; c0 < t1; c0 += C) {
    const int L = (t1 - c0) < C ? (int)(t1 - c0) : C;

    const bool l2n = (a.prologue & KDA_PROLOGUE_QK_L2NORM) != 0;
    const bool gsig = (a.prologue & KDA_PROLOGUE_GATE_SIGMOID) != 0;
    // 1. Stage the chunk's k, q (unit rows with the prologue) and clamped log decays, the V
    //    slice and beta: 16-byte vectors, every load issued before any store; rows past L
    //    are zero (no key, no decay). Then the decay tiles in place, one channel per thread.
    {
      constexpr int EV = 16 / sizeof(Tin), VR = DK / EV, NV = C * VR / NT;
      constexpr int OV = DVS / EV, NO = (C * OV + NT - 1) / NT;
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      uint4 kq[NV], qq[NV], gq[NV], vq[NO];
#pragma unroll
      for (int m = 0; m < NV; ++m) {
        const int e = tid + NT * m, r = e / VR, vi = e % VR;
        const int64_t off = ((c0 + r) * H + h) * DK + vi * EV;
        kq[m] = r < L ? *reinterpret_cast<const uint4*>(k + off) : z;
        qq[m] = r < L ? *reinterpret_cast<const uint4*>(q + off) : z;
        gq[m] = r < L ? *reinterpret_cast<const uint4*>(g + off) : z;
      }
#pragma unroll
      for (int m = 0; m < NO; ++m) {
        const int e = tid + NT * m, r = e / OV, vj = e % OV;
        const bool in = e < C * OV && r < L;
        vq[m] = in ? *reinterpret_cast<const uint4*>(v + ((c0 + r) * H + h) * DV + j0 + vj * EV) : z;
      }
      if (tid < C) sm.bet[tid] = tid < L ? ld_in(beta + (c0 + tid) * H + h) : 0.f;
#pragma unroll
      for (int m = 0; m < NV; ++m) {
        const int e = tid + NT * m, r = e / VR, i0 = (e % VR) * EV;
        float kf[EV], qf[EV], gf[EV];
        unpack_vec<Tin>(kq[m], kf);
        unpack_vec<Tin>(qq[m], qf);
        unpack_vec<Tin>(gq[m], gf);
        if (l2n) {  // a row is VR consecutive lanes (VR divides 32): norms by shuffles
          float sk = 0.f, sq2 = 0.f;
#pragma unroll
          for (int x = 0; x < EV; ++x) {
            sk = fmaf(kf[x], kf[x], sk);
            sq2 = fmaf(qf[x], qf[x], sq2);
          }
#pragma unroll
          for (int o2 = VR / 2; o2 > 0; o2 >>= 1) {
            sk += __shfl_xor_sync(0xffffffffu, sk, o2);
            sq2 += __shfl_xor_sync(0xffffffffu, sq2, o2);
          }
          const float rk = inv_l2(sk), rq = inv_l2(sq2);
#pragma unroll
          for (int x = 0; x < EV; ++x) {
            kf[x] *= rk;
            qf[x] *= rq;
          }
        }
#pragma unroll
        for (int x = 0; x < EV; ++x) {
          const float gx = gsig ? gate_from_preact(gf[x], a.lb) : gf[x];
          sm.Kt[r][i0 + x] = kf[x];
          sm.Qt[r][i0 + x] = qf[x];
          sm.Kh[r][i0 + x] = r < L ? fmaxf(gx, a.lb) : 0.f;
        }
      }
#pragma unroll
      for (int m = 0; m < NO; ++m) {
        const int e = tid + NT * m, r = e / OV, j = (e % OV) * EV;
        if (e < C * OV) {
          float vf[EV];
          unpack_vec<Tin>(vq[m], vf);
#pragma unroll
          for (int x = 0; x < EV; ++x) sm.Y[r][j + x] = vf[x];
        }
      }
    }
    __syncthreads();
    if (tid < DK) {
      const int i = tid;
      float G = 0.f;
#pragma unroll 8
      for (int r = 0; r < C; ++r) {
        G += sm.Kh[r][i];
        const float e = expf(G), ei = expf(-G);
        const float kv = sm.Kt[r][i];
        sm.Kt[r][i] = kv * e;
        sm.Kh[r][i] = kv * ei;
        sm.Qt[r][i] *= e;
      }
      sm.gl[i] = expf(G);
    }
    __syncthreads();

    // 2. A = Diag(beta) strict_lower(K~ K^^T) and P = lower_incl(Q~ K^^T).
    {
      const int tx = tid % 16, ty = tid / 16;
      float accA[4][4], accP[4][4];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) accA[x][y] = accP[x][y] = 0.f;
      for (int i = 0; i < DK; ++i) {
        float kt[4], qt[4], kh[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          kt[x] = sm.Kt[ty * 4 + x][i];
          qt[x] = sm.Qt[ty * 4 + x][i];
          kh[x] = sm.Kh[tx + 16 * x][i];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) {
            accA[x][y] = fmaf(kt[x], kh[y], accA[x][y]);
            accP[x][y] = fmaf(qt[x], kh[y], accP[x][y]);
          }
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int r = ty * 4 + x, c = tx + 16 * y;
          sm.A[r][c] = (c < r) ? sm.bet[r] * accA[x][y] : 0.f;
          sm.P[r][c] = (c <= r) ? accP[x][y] : 0.f;
        }
    }
    __syncthreads();

    // 3. N = (I + A)^{-1} into Tm (T = N Diag(beta) is applied in step 5): the four 16x16
    //    diagonal blocks by forward substitution, one per half-warp; then 16 -> 32 and
    //    32 -> 64 merges N21 = -N22 (A21 N11) by all threads (A21 is overwritten by A21 N11;
    //    A is not needed afterwards). Rows past L: A is zero there, N the identity.
    for (int e = tid; e < C * C; e += NT) {
      const int rr = e / C, cc = e % C;
      if ((rr >> 4) != (cc >> 4)) sm.Tm[rr][cc] = 0.f;
    }
    if (tid < 64) {
      const int base = 16 * (tid >> 4), c = tid & 15;
      for (int rr = 0; rr < 16; ++rr) {
        float val = (c == rr) ? 1.f : 0.f;
        for (int s2 = c; s2 < rr; ++s2)
          val = fmaf(-sm.A[base + rr][base + s2], sm.Tm[base + s2][base + c], val);
        sm.Tm[base + rr][base + c] = (c <= rr) ? val : 0.f;
        __syncwarp();
      }
    }
    __syncthreads();
    {
      const int o = 32 * (tid >> 7);
      float xv[2];
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int idx = (tid & 127) + 128 * m, rr = idx >> 4, cc = idx & 15;
        float acc = 0.f;
        for (int s2 = cc; s2 < 16; ++s2) acc = fmaf(sm.A[o + 16 + rr][o + s2], sm.Tm[o + s2][o + cc], acc);
        xv[m] = acc;
      }
      __syncthreads();
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int idx = (tid & 127) + 128 * m;
        sm.A[o + 16 + (idx >> 4)][o + (idx & 15)] = xv[m];
      }
      __syncthreads();
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int idx = (tid & 127) + 128 * m, rr = idx >> 4, cc = idx & 15;
        float acc = 0.f;
        for (int s2 = 0; s2 <= rr; ++s2)
          acc = fmaf(sm.Tm[o + 16 + rr][o + 16 + s2], sm.A[o + 16 + s2][o + cc], acc);
        sm.Tm[o + 16 + rr][o + cc] = -acc;
      }
    }
    __syncthreads();
    {
      float xv[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int idx = tid + NT * m, rr = idx >> 5, cc = idx & 31;
        float acc = 0.f;
        for (int s2 = cc; s2 < 32; ++s2) acc = fmaf(sm.A[32 + rr][s2], sm.Tm[s2][cc], acc);
        xv[m] = acc;
      }
      __syncthreads();
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int idx = tid + NT * m;
        sm.A[32 + (idx >> 5)][idx & 31] = xv[m];
      }
      __syncthreads();
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int idx = tid + NT * m, rr = idx >> 5, cc = idx & 31;
        float acc = 0.f;
        for (int s2 = 0; s2 <= rr; ++s2) acc = fmaf(sm.Tm[32 + rr][32 + s2], sm.A[32 + s2][cc], acc);
        sm.Tm[32 + rr][cc] = -acc;
      }
    }
    __syncthreads();

    const int r = tid / 4, cb = (tid % 4) * 8;
    // 4. Y = V - K~ S
    {
      float acc[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = 0.f;
      for (int i = 0; i < DK; ++i) {
        const float kt = sm.Kt[r][i];
        axpy4(kt, &sm.S[i][cb], acc);
        axpy4(kt, &sm.S[i][cb + 4], acc + 4);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) sm.Y[r][cb + c] -= acc[c];
    }
    __syncthreads();
    // 5. U = T Y
    {
      float acc[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = 0.f;
      for (int s2 = 0; s2 <= r; ++s2) {
        const float t = sm.Tm[r][s2] * sm.bet[s2];  // T = N Diag(beta)
        axpy4(t, &sm.Y[s2][cb], acc);
        axpy4(t, &sm.Y[s2][cb + 4], acc + 4);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) sm.U[r][cb + c] = acc[c];
    }
    __syncthreads();
    // 6. O = scale (Q~ S + P U)
    {
      float acc[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = 0.f;
      for (int i = 0; i < DK; ++i) {
        const float qt = sm.Qt[r][i];
        axpy4(qt, &sm.S[i][cb], acc);
        axpy4(qt, &sm.S[i][cb + 4], acc + 4);
      }
      for (int s2 = 0; s2 <= r; ++s2) {
        const float p = sm.P[r][s2];
        axpy4(p, &sm.U[s2][cb], acc);
        axpy4(p, &sm.U[s2][cb + 4], acc + 4);
      }
      if (r < L) {
        Tin* o = out + ((c0 + r) * H + h) * DV + j0 + cb;
#pragma unroll
        for (int c = 0; c < 8; ++c) st_out(o + c, a.scale * acc[c]);
      }
    }
    __syncthreads();
    // 7. S = Diag(exp Gamma_L) S + (K^ * exp Gamma_L)^T U
    {
      constexpr int PER = DK * DVS / NT;       // entries per thread
      const int i = tid / (DVS / PER), cs = (tid % (DVS / PER)) * PER;
      const float gli = sm.gl[i];
      float acc[PER];
#pragma unroll
      for (int c = 0; c < PER; ++c) acc[c] = gli * sm.S[i][cs + c];
      for (int rr = 0; rr < L; ++rr) {
        const float kb = sm.Kh[rr][i] * gli;
#pragma unroll
        for (int c = 0; c < PER; c += 4) axpy4(kb, &sm.U[rr][cs + c], acc + c);
      }
      __syncthreads();
#pragma unroll
      for (int c = 0; c < PER; ++c) sm.S[i][cs + c] = acc[c];
      // the state after a full chunk that closes a snapshot interval of the sequence
      const int64_t done = (c0 - t0) / C + 1;  // chunks of the sequence walked
      if (a.snap != nullptr && L == C && done % a.snap_every == 0) {
        const int64_t idx = t0 / (static_cast<int64_t>(C) * a.snap_every) + done / a.snap_every - 1;
        float* d = a.snap + (idx * H + h) * DK * DV + j0 + static_cast<int64_t>(i) * DV + cs;
#pragma unroll
        for (int c = 0; c < PER; ++c) d[c] = acc[c];
      }
    }
    __syncthreads();
  }

  if (a.sT) {
    for (int e = tid; e < DK * DVS; e += NT) {
      const int i = e / DVS, c = e % DVS;
      a.sT[state_base + (int64_t)i * DV + c] = sm.S[i][c];
    }
  }
}

template <typename Tin, int DK>
cudaError_t launch_typed(const PrefillArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(SimtSmem<DK>);
  cudaError_t e = cudaFuncSetAttribute(prefill_simt_kernel<Tin, DK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)a.n_seqs * a.H * (a.dv / DVS);
  if (blocks == 0) return cudaSuccess;
  prefill_simt_kernel<Tin, DK><<<(unsigned)blocks, NT, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_simt(const PrefillArgs& a, kda_dtype dtype, cudaStream_t st) {
  if (dtype == KDA_F32) {
    return a.dk == 64 ? launch_typed<float, 64>(a, st) : launch_typed<float, 128>(a, st);
  }
  return a.dk == 64 ? launch_typed<__nv_bfloat16, 64>(a, st)
                    : launch_typed<__nv_bfloat16, 128>(a, st);
}

}  // namespace kda
