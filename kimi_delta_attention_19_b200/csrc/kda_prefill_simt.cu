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
  float S[DK][DVS];     // state slice
  float Y[C][DVS];      // V slice, then V - K~ S
  float U[C][DVS];
  float gl[DK];         // exp(Gamma_L) per channel
  float bet[C];
  float rk[C], rq[C];   // prologue: 1 / |k row|, 1 / |q row|
};

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
    if (l2n) {
      // prologue: inverse L2 norms of the chunk's raw k and q rows, one warp per row
      const int warp = tid >> 5, lane = tid & 31;
      for (int rr = warp; rr < 2 * C; rr += NT / 32) {
        const int r = rr % C;
        const bool isq = rr >= C;
        float ss = 0.f;
        if (r < L) {
          const Tin* src = (isq ? q : k) + ((c0 + r) * H + h) * DK;
          for (int i = lane; i < DK; i += 32) {
            const float x = ld_in(src + i);
            ss = fmaf(x, x, ss);
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) (isq ? sm.rq : sm.rk)[r] = inv_l2(ss);
      }
      __syncthreads();
    }

    // 1. Prefix sums of the clamped log decay and the decayed operands.
    if (tid < DK) {
      const int i = tid;
      float G = 0.f;
      for (int r = 0; r < C; ++r) {
        float kt = 0.f, kh = 0.f, qt = 0.f;
        if (r < L) {
          const int64_t off = ((c0 + r) * H + h) * DK + i;
          float gr = ld_in(g + off);
          if (gsig) gr = gate_from_preact(gr, a.lb);
          G += fmaxf(gr, a.lb);
          const float e = expf(G), ei = expf(-G);
          const float kv = ld_in(k + off) * (l2n ? sm.rk[r] : 1.f);
          kt = kv * e;
          kh = kv * ei;
          qt = ld_in(q + off) * (l2n ? sm.rq[r] : 1.f) * e;
        }
        sm.Kt[r][i] = kt;
        sm.Kh[r][i] = kh;
        sm.Qt[r][i] = qt;
      }
      sm.gl[i] = expf(G);
    } else {
      for (int e = tid - DK; e < C * DVS; e += NT - DK) {
        const int r = e / DVS, c = e % DVS;
        sm.Y[r][c] = (r < L) ? ld_in(v + ((c0 + r) * H + h) * DV + j0 + c) : 0.f;
      }
      for (int r = tid - DK; r < C; r += NT - DK)
        sm.bet[r] = (r < L) ? ld_in(beta + (c0 + r) * H + h) : 0.f;
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
          kh[x] = sm.Kh[tx * 4 + x][i];
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
          const int r = ty * 4 + x, c = tx * 4 + y;
          sm.A[r][c] = (c < r) ? sm.bet[r] * accA[x][y] : 0.f;
          sm.P[r][c] = (c <= r) ? accP[x][y] : 0.f;
        }
    }
    __syncthreads();

    // 3. T = (I + A)^{-1} Diag(beta) by forward substitution, one row at a time.
    if (tid < C) {
      for (int r = L; r < C; ++r) sm.Tm[r][tid] = 0.f;
    }
    for (int r = 0; r < L; ++r) {
      if (tid < C) {
        const int c = tid;
        float val = 0.f;
        if (c <= r) {
          val = (c == r) ? sm.bet[r] : 0.f;
          for (int s2 = c; s2 < r; ++s2) val = fmaf(-sm.A[r][s2], sm.Tm[s2][c], val);
        }
        sm.Tm[r][c] = val;
      }
      __syncthreads();
    }

    const int r = tid / 4, cb = (tid % 4) * 8;
    // 4. Y = V - K~ S
    {
      float acc[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = 0.f;
      for (int i = 0; i < DK; ++i) {
        const float kt = sm.Kt[r][i];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = fmaf(kt, sm.S[i][cb + c], acc[c]);
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
        const float t = sm.Tm[r][s2];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = fmaf(t, sm.Y[s2][cb + c], acc[c]);
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
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = fmaf(qt, sm.S[i][cb + c], acc[c]);
      }
      for (int s2 = 0; s2 <= r; ++s2) {
        const float p = sm.P[r][s2];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = fmaf(p, sm.U[s2][cb + c], acc[c]);
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
        for (int c = 0; c < PER; ++c) acc[c] = fmaf(kb, sm.U[rr][cs + c], acc[c]);
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
