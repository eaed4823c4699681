// kda_backward.cu -- gradients of the chunked prefill, fp32 on CUDA cores.
//
// Reverse mode through the chunk-parallel form ("Kimi K3 深度拆解", section 4.2:
// chunk-parallel with an inter-chunk recurrence; the bounded log decay of
// "3 分钟看懂 Kimi K3", Figure 3, keeps exp(-Gamma) finite over a chunk). Per chunk of
// L <= 64 tokens with start state S, end-state gradient dS' and output gradient dO:
//
//   forward pieces (recomputed): Gamma = cumsum max(g, lb), E = exp Gamma,
//     K~ = K E, K^ = K / E, Q~ = Q E, gl = E_last, A = Diag(beta) strict_lower(K~ K^^T),
//     N = (I + A)^-1, T = N Diag(beta), Y = V - K~ S, U = T Y, P = lower_incl(Q~ K^^T)
//   dU  = (K^ gl) dS' + scale P^T dO
//   dT  = dU Y^T,        Z = T^T dU = dV
//   dS  = Diag(gl) dS' + scale Q~^T dO - K~^T Z          (carried to the previous chunk)
//   dN  = dT Diag(beta), dA = -N^T dN N^T,  dG = strict_lower(Diag(beta) dA)
//   dbeta_r = sum_c N_cr dT_cr + sum_{s<r} (K~ K^^T)_rs dA_rs = ... + K~_r . (dA K^)_r
//   dP  = scale lower_incl(dO U^T)
//   dQ~ = scale dO S^T + dP K^,   dK~ = -Z S^T + dG K^
//   dK^ = dP^T Q~ + dG^T K~ + (U dS'^T) gl,   dgl = rowsum(S dS') + colsum(K^ (U dS'^T))
//   dGamma = dK~ K~ - dK^ K^ + dQ~ Q~ (+ dgl gl on the last row), dg' = reverse cumsum,
//   dg = dg' where g >= lb,   dq = dQ~ E,   dk = dK~ E + dK^ / E
//
// One CTA per (sequence, head, slice of 32 or 16 columns of d_v) walks the chunks backwards. The
// columns of S and dS evolve independently, so dv, dS and dS0 of a slice are complete in
// its CTA; dq, dk, dg and dbeta are sums over the slices and are added, in fp32, into
// accumulators that a finishing pass converts to the input dtype (carrying them through
// the raw-input prologue when it is on). The chunk start states come from a forward pass
// that keeps the state after every chunk.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int C = kChunk;
constexpr int NT = 256;   // threads per CTA

// DVS: the d_v columns of one CTA (32, or 16 when the sequences and heads alone give too
// few CTAs to fill the GPU)
template <int DK, int DVS>
struct BwdSmem {
  float Kt[C][DK + 1];   // K~
  float Kh[C][DK + 1];   // K^
  float Qt[C][DK + 1];   // Q~
  float BA[C][C + 1];    // A, then N^T dN, then dP
  float BN[C][C + 1];    // N = (I + A)^-1
  float BP[C][C + 1];    // P, then dT -> dN -> dA (strict lower; dG = Diag(beta) dA is
                         // applied where it is used)
  // d_v-slice arrays: rows of DVS + 4 floats, 16-byte aligned, so products over the slice's
  // columns read float4s (conflict-free with the stride of 36 words)
  alignas(16) float S[DK][DVS + 4];  // chunk start state (slice)
  alignas(16) float dS[DK][DVS + 4]; // dL/d(chunk end state), updated in place to the start
  alignas(16) float Y[C][DVS + 4];   // V - K~ S, then Z = T^T dU (= dL/dV)
  alignas(16) float U[C][DVS + 4];
  alignas(16) float dO[C][DVS + 4];
  alignas(16) float dU[C][DVS + 4];
  float gl[DK];
  float sdS[DK];         // sum_j S[i][j] dS'[i][j]: the decay of S's part of dgl
  float bet[C];
  float dbet[C];
};
static_assert(2 * 16 * 128 <= C * (C + 1), "row-group scans fit in the N buffer");

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

// PRO: the raw-input prologue flags (KDA_PROLOGUE_*); the kernel then works on the
// normalised q, k and the gate's log decays, and the finishing pass carries the gradients
// through the prologue to the raw inputs.
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float dot4(const float4& a, const float4& b, float c) {
  return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, fmaf(a.x, b.x, c))));
}

template <typename Tin, int DK, int DVS, int PRO>
__global__ void __launch_bounds__(NT, 1) bwd_simt_kernel(BackwardArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BwdSmem<DK, DVS>& sm = *reinterpret_cast<BwdSmem<DK, DVS>*>(smem_raw);
  constexpr int CT = DK / 16;   // channels per thread in the per-element pass
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
  const Tin* dout = static_cast<const Tin*>(a.dout);
  Tin* dvo = static_cast<Tin*>(a.dv_out);
  const int64_t state_base = ((int64_t)s * H + h) * DK * DV + j0;
  const float scale = a.scale, lb = a.lb;

  for (int e = tid; e < DK * DVS; e += NT) {
    const int i = e / DVS, c = e % DVS;
    sm.dS[i][c] = a.dsT ? a.dsT[state_base + (int64_t)i * DV + c] : 0.f;
  }

  const int64_t n_chunks = (t1 - t0 + C - 1) / C;
  const int64_t snap0 = t0 / C;  // snapshot index of this sequence's first chunk end
  // C x DVS tiles: RR rows from rcr, columns rcc + RCW x (x < 4)
  constexpr int RCW = DVS / 4, RR = C * DVS / (NT * 4);
  const int rcr = RR * (tid / RCW), rcc = tid % RCW;
  const int tx = tid % 16, ty = tid / 16;         // C x C tiles: rows 4 ty + x, columns
                                                  // tx + 16 y (conflict-free loads)

  for (int64_t cc = n_chunks - 1; cc >= 0; --cc) {
    const int64_t c0 = t0 + cc * C;
    const int L = (t1 - c0) < C ? (int)(t1 - c0) : C;
    __syncthreads();  // the previous chunk's reads are done

    // ---- 0. stage the chunk's k, q and clamped log decays (normalised and gated with the
    //         prologue; all threads, coalesced; rows past L are zero: no key, no decay) and
    //         the slice's S, V, dO and beta; then the decay tiles in place, one channel per
    //         thread
    {
      // k, q, g rows: 16-byte vectors, all of a thread's loads issued before any store
      constexpr int EV = 16 / sizeof(Tin);        // elements per vector
      constexpr int VR = DK / EV;                 // vectors per row
      constexpr int NV = C * VR / NT;             // vectors per thread per tensor
      uint4 kq[NV], qq[NV], gq[NV];
#pragma unroll
      for (int m = 0; m < NV; ++m) {
        const int e = tid + NT * m, r = e / VR, vi = e % VR;
        const int64_t off = ((c0 + r) * H + h) * DK + vi * EV;
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        kq[m] = r < L ? *reinterpret_cast<const uint4*>(k + off) : z;
        qq[m] = r < L ? *reinterpret_cast<const uint4*>(q + off) : z;
        gq[m] = r < L ? *reinterpret_cast<const uint4*>(g + off) : z;
      }
      // the slice's S (fp32 rows of DVS), V and dO rows (DVS elements), beta
      constexpr int SV = DVS / 4, NS = DK * SV / NT;          // S: float4 vectors
      constexpr int OV = DVS / EV, NO = (C * OV + NT - 1) / NT; // V, dO vectors
      const float* src = nullptr;
      if (cc > 0) src = a.snap + ((snap0 + cc - 1) * H + h) * (int64_t)DK * DV + j0;
      else if (a.s0) src = a.s0 + state_base;
      float4 sq[NS];
#pragma unroll
      for (int m = 0; m < NS; ++m) {
        const int e = tid + NT * m, i = e / SV, vj = e % SV;
        sq[m] = src ? *reinterpret_cast<const float4*>(src + (int64_t)i * DV + 4 * vj)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      uint4 vq[NO], oq[NO];
#pragma unroll
      for (int m = 0; m < NO; ++m) {
        const int e = tid + NT * m, r = e / OV, vj = e % OV;
        const int64_t off = ((c0 + r) * H + h) * DV + j0 + vj * EV;
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        const bool in = e < C * OV && r < L;
        vq[m] = in ? *reinterpret_cast<const uint4*>(v + off) : z;
        oq[m] = (in && dout) ? *reinterpret_cast<const uint4*>(dout + off) : z;
      }
      if (tid < C) sm.bet[tid] = tid < L ? ld_in(beta + (c0 + tid) * H + h) : 0.f;
      // unpack into shared memory (k -> Kt, q -> Qt, clamped log decay -> Kh; rows past
      // L are zero: no key, no decay)
#pragma unroll
      for (int m = 0; m < NV; ++m) {
        const int e = tid + NT * m, r = e / VR, i0 = (e % VR) * EV;
        float kf[EV], qf[EV], gf[EV];
        unpack_vec<Tin>(kq[m], kf);
        unpack_vec<Tin>(qq[m], qf);
        unpack_vec<Tin>(gq[m], gf);
        if (PRO & KDA_PROLOGUE_QK_L2NORM) {
          // a row is VR consecutive lanes (VR divides 32): its norms by shuffles
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
          float gx = gf[x];
          if (PRO & KDA_PROLOGUE_GATE_SIGMOID) gx = gate_from_preact(gx, lb);
          sm.Kt[r][i0 + x] = kf[x];
          sm.Qt[r][i0 + x] = qf[x];
          sm.Kh[r][i0 + x] = r < L ? fmaxf(gx, lb) : 0.f;
        }
      }
#pragma unroll
      for (int m = 0; m < NS; ++m) {
        const int e = tid + NT * m, i = e / SV, j = 4 * (e % SV);
        *reinterpret_cast<float4*>(&sm.S[i][j]) = sq[m];
      }
#pragma unroll
      for (int m = 0; m < NO; ++m) {
        const int e = tid + NT * m, r = e / OV, j = (e % OV) * EV;
        if (e < C * OV) {
          float vf[EV], of[EV];
          unpack_vec<Tin>(vq[m], vf);
          unpack_vec<Tin>(oq[m], of);
#pragma unroll
          for (int x = 0; x < EV; ++x) {
            sm.Y[r][j + x] = vf[x];
            sm.dO[r][j + x] = of[x];
          }
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

    // ---- 1. A = Diag(beta) strict_lower(K~ K^^T) and P = lower_incl(Q~ K^^T)
    {
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
          sm.BA[r][c] = (c < r) ? sm.bet[r] * accA[x][y] : 0.f;
          sm.BP[r][c] = (c <= r) ? accP[x][y] : 0.f;
        }
    }
    __syncthreads();

    // ---- 2. N = (I + A)^-1 (lower triangular): the four 16x16 diagonal blocks by forward
    //         substitution, one per half-warp; then 16 -> 32 and 32 -> 64 merges
    //         N21 = -N22 (A21 N11), each product by all threads. A21 is overwritten by
    //         A21 N11 (A is not needed afterwards); the upper blocks of N stay zero.
    for (int e = tid; e < C * C; e += NT) {
      const int r = e / C, c = e % C;
      if ((r >> 4) != (c >> 4)) sm.BN[r][c] = 0.f;
    }
    if (tid < 64) {
      const int base = 16 * (tid >> 4), c = tid & 15;
      for (int r = 0; r < 16; ++r) {
        float val = (c == r) ? 1.f : 0.f;
        for (int s2 = c; s2 < r; ++s2)
          val = fmaf(-sm.BA[base + r][base + s2], sm.BN[base + s2][base + c], val);
        sm.BN[base + r][base + c] = (c <= r) ? val : 0.f;
        __syncwarp();
      }
    }
    __syncthreads();
    {  // 16 -> 32, both 32-blocks at once: thread -> block o = 32 (tid >> 7), two elements
      const int o = 32 * (tid >> 7);
      float xv[2];
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int idx = (tid & 127) + 128 * m, r = idx >> 4, c = idx & 15;
        float acc = 0.f;
        for (int s2 = c; s2 < 16; ++s2)
          acc = fmaf(sm.BA[o + 16 + r][o + s2], sm.BN[o + s2][o + c], acc);
        xv[m] = acc;
      }
      __syncthreads();
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int idx = (tid & 127) + 128 * m;
        sm.BA[o + 16 + (idx >> 4)][o + (idx & 15)] = xv[m];
      }
      __syncthreads();
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int idx = (tid & 127) + 128 * m, r = idx >> 4, c = idx & 15;
        float acc = 0.f;
        for (int s2 = 0; s2 <= r; ++s2)
          acc = fmaf(sm.BN[o + 16 + r][o + 16 + s2], sm.BA[o + 16 + s2][o + c], acc);
        sm.BN[o + 16 + r][o + c] = -acc;
      }
    }
    __syncthreads();
    {  // 32 -> 64: four elements per thread
      float xv[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int idx = tid + NT * m, r = idx >> 5, c = idx & 31;
        float acc = 0.f;
        for (int s2 = c; s2 < 32; ++s2) acc = fmaf(sm.BA[32 + r][s2], sm.BN[s2][c], acc);
        xv[m] = acc;
      }
      __syncthreads();
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int idx = tid + NT * m;
        sm.BA[32 + (idx >> 5)][idx & 31] = xv[m];
      }
      __syncthreads();
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int idx = tid + NT * m, r = idx >> 5, c = idx & 31;
        float acc = 0.f;
        for (int s2 = 0; s2 <= r; ++s2) acc = fmaf(sm.BN[32 + r][32 + s2], sm.BA[32 + s2][c], acc);
        sm.BN[32 + r][c] = -acc;
      }
    }
    __syncthreads();

    // ---- 3. Y = V - K~ S, then U = N Diag(beta) Y            (C x DVS tiles, RR x 4)
    {
      float acc[RR][4] = {};
      for (int i = 0; i < DK; ++i) {
        float kr[RR];
#pragma unroll
        for (int y = 0; y < RR; ++y) kr[y] = sm.Kt[rcr + y][i];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float sv = sm.S[i][rcc + RCW * x];
#pragma unroll
          for (int y = 0; y < RR; ++y) acc[y][x] = fmaf(kr[y], sv, acc[y][x]);
        }
      }
#pragma unroll
      for (int y = 0; y < RR; ++y)
#pragma unroll
        for (int x = 0; x < 4; ++x) sm.Y[rcr + y][rcc + RCW * x] -= acc[y][x];
    }
    __syncthreads();
    {
      float acc[RR][4] = {};
      for (int s2 = 0; s2 < rcr + RR; ++s2) {  // N is lower triangular
        const float b = sm.bet[s2];
        float nr[RR];
#pragma unroll
        for (int y = 0; y < RR; ++y) nr[y] = sm.BN[rcr + y][s2] * b;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float yv = sm.Y[s2][rcc + RCW * x];
#pragma unroll
          for (int y = 0; y < RR; ++y) acc[y][x] = fmaf(nr[y], yv, acc[y][x]);
        }
      }
#pragma unroll
      for (int y = 0; y < RR; ++y)
#pragma unroll
        for (int x = 0; x < 4; ++x) sm.U[rcr + y][rcc + RCW * x] = acc[y][x];
    }
    __syncthreads();

    // ---- 4. dU = (K^ gl) dS' + scale P^T dO
    {
      float acc[RR][4] = {}, acc2[RR][4] = {};
      for (int i = 0; i < DK; ++i) {
        const float gi = sm.gl[i];
        float kr[RR];
#pragma unroll
        for (int y = 0; y < RR; ++y) kr[y] = sm.Kh[rcr + y][i] * gi;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float dv0 = sm.dS[i][rcc + RCW * x];
#pragma unroll
          for (int y = 0; y < RR; ++y) acc[y][x] = fmaf(kr[y], dv0, acc[y][x]);
        }
      }
      for (int t = rcr; t < C; ++t) {  // P[t][r] = 0 for t < r
        float pr[RR];
#pragma unroll
        for (int y = 0; y < RR; ++y) pr[y] = sm.BP[t][rcr + y];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float o = sm.dO[t][rcc + RCW * x];
#pragma unroll
          for (int y = 0; y < RR; ++y) acc2[y][x] = fmaf(pr[y], o, acc2[y][x]);
        }
      }
#pragma unroll
      for (int y = 0; y < RR; ++y)
#pragma unroll
        for (int x = 0; x < 4; ++x)
          sm.dU[rcr + y][rcc + RCW * x] = fmaf(scale, acc2[y][x], acc[y][x]);
    }
    __syncthreads();

    // ---- 5. dT = dU Y^T (over P, which is dead)                 (C x C tiles, 4 x 4)
    {
      float acc[4][4] = {};
      for (int j = 0; j < DVS; j += 4) {
        float4 du[4], yy[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          du[x] = ld4(&sm.dU[ty * 4 + x][j]);
          yy[x] = ld4(&sm.Y[tx + 16 * x][j]);
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[x][y] = dot4(du[x], yy[y], acc[x][y]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) sm.BP[ty * 4 + x][tx + 16 * y] = acc[x][y];
      // sum_j S[i][j] dS'[i][j], NT / DK threads per channel
      constexpr int TPR = NT / DK, JPT = DVS / TPR;
      const int i = tid / TPR, j0p = (tid % TPR) * JPT;
      float sd = 0.f;
#pragma unroll
      for (int j = 0; j < JPT; ++j) sd = fmaf(sm.S[i][j0p + j], sm.dS[i][j0p + j], sd);
#pragma unroll
      for (int o2 = 1; o2 < TPR; o2 <<= 1) sd += __shfl_xor_sync(0xffffffffu, sd, o2);
      if (tid % TPR == 0) sm.sdS[i] = sd;
    }
    __syncthreads();

    // ---- 6. Z = Diag(beta) N^T dU (= dL/dV, over Y); dbeta from T = N Diag(beta)
    {
      float acc[RR][4] = {};
      for (int t = rcr; t < C; ++t) {  // N[t][r] = 0 for t < r
        float nr[RR];
#pragma unroll
        for (int y = 0; y < RR; ++y) nr[y] = sm.BN[t][rcr + y];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float d = sm.dU[t][rcc + RCW * x];
#pragma unroll
          for (int y = 0; y < RR; ++y) acc[y][x] = fmaf(nr[y], d, acc[y][x]);
        }
      }
#pragma unroll
      for (int y = 0; y < RR; ++y) {
        const int r = rcr + y;
        const float b = sm.bet[r];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          sm.Y[r][rcc + RCW * x] = b * acc[y][x];
          if (r < L) st_out(dvo + ((c0 + r) * H + h) * DV + j0 + rcc + RCW * x, b * acc[y][x]);
        }
      }
      if (tid < C) {
        const int r = tid;
        float db = 0.f;
        for (int c = r; c < C; ++c) db = fmaf(sm.BN[c][r], sm.BP[c][r], db);
        sm.dbet[r] = db;
      }
    }
    __syncthreads();

    // ---- 7. dN = dT Diag(beta) (in place), then N^T dN (over A), then dA = -(N^T dN) N^T
    for (int e = tid; e < C * C; e += NT) {
      const int r = e / C, c = e % C;
      sm.BP[r][c] *= sm.bet[c];
    }
    __syncthreads();
    {
      float acc[4][4] = {};
      for (int c = 0; c < C; ++c) {  // (N^T dN)[r][s] = sum_c N[c][r] dN[c][s]
        float nv[4], dn[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          nv[x] = sm.BN[c][ty * 4 + x];
          dn[x] = sm.BP[c][tx + 16 * x];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(nv[x], dn[y], acc[x][y]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) sm.BA[ty * 4 + x][tx + 16 * y] = acc[x][y];
    }
    __syncthreads();
    {
      float acc[4][4] = {};
      for (int c = 0; c < C; ++c) {  // dA[r][s] = -sum_c (N^T dN)[r][c] N[s][c]
        float tv[4], nv[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          tv[x] = sm.BA[ty * 4 + x][c];
          nv[x] = sm.BN[tx + 16 * x][c];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(tv[x], nv[y], acc[x][y]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) sm.BP[ty * 4 + x][tx + 16 * y] = -acc[x][y];
    }
    __syncthreads();

    // ---- 8. dA keeps its strict lower part (dG = Diag(beta) dA is applied where it is used);
    //         dP = scale lower_incl(dO U^T) over (N^T dN)
    {
      float accP[4][4] = {};
      for (int j = 0; j < DVS; j += 4) {
        float4 d[4], u[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          d[x] = ld4(&sm.dO[ty * 4 + x][j]);
          u[x] = ld4(&sm.U[tx + 16 * x][j]);
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) accP[x][y] = dot4(d[x], u[y], accP[x][y]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int r = ty * 4 + x;
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int c = tx + 16 * y;
          if (c >= r) sm.BP[r][c] = 0.f;
          sm.BA[r][c] = (c <= r) ? scale * accP[x][y] : 0.f;
        }
      }
    }
    __syncthreads();
    if (tid < L) atomicAdd(a.acc_b + (c0 + tid) * H + h, sm.dbet[tid]);

    // ---- 9. per element of the C x DK tiles (4 rows x CT channels per thread): dQ~, dK~,
    //         dK^ -> dq, dk; dGamma -> dg. N is dead: its buffer holds the row-group scans.
    {
      float* scan = &sm.BN[0][0];           // [16][DK]: prefix / suffix totals per row group
      float* dglp_all = scan + 16 * DK;     // [16][DK]: dgl parts per row group
      const int rg = tid >> 4, cg = tid & 15, rb = 4 * rg;
      // 9a. Gamma of the thread's rows: its rows' clamped decay sums, then the earlier groups'
      float gsum[CT] = {}, graw[4][CT];
#pragma unroll
      for (int y = 0; y < 4; ++y)
#pragma unroll
        for (int x = 0; x < CT; ++x) {
          const int r = rb + y, c = cg + 16 * x;
          graw[y][x] = r < L ? ld_in(g + ((c0 + r) * H + h) * DK + c) : 0.f;
          if ((PRO & KDA_PROLOGUE_GATE_SIGMOID) && r < L) graw[y][x] = gate_from_preact(graw[y][x], lb);
          gsum[x] += r < L ? fmaxf(graw[y][x], lb) : 0.f;
        }
#pragma unroll
      for (int x = 0; x < CT; ++x) scan[rg * DK + cg + 16 * x] = gsum[x];
      __syncthreads();
      float E[4][CT];
      uint32_t live = 0;  // bit y * CT + x: g >= lb (the clamp passes the gradient)
#pragma unroll
      for (int x = 0; x < CT; ++x) {
        float G = 0.f;
        for (int q2 = 0; q2 < rg; ++q2) G += scan[q2 * DK + cg + 16 * x];
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          G += rb + y < L ? fmaxf(graw[y][x], lb) : 0.f;
          E[y][x] = expf(G);
          if (graw[y][x] >= lb) live |= 1u << (y * CT + x);
        }
      }
      float dgam[4][CT], dkk[4][CT], acc[4][CT];
      // 9b. dQ~ = scale dO S^T + dP K^  ->  dq, dGamma
#pragma unroll
      for (int y = 0; y < 4; ++y)
#pragma unroll
        for (int x = 0; x < CT; ++x) acc[y][x] = 0.f;
      for (int j = 0; j < DVS; j += 4) {
        float4 o[4];
#pragma unroll
        for (int y = 0; y < 4; ++y) o[y] = ld4(&sm.dO[rb + y][j]);
#pragma unroll
        for (int x = 0; x < CT; ++x) {
          const float4 sv = ld4(&sm.S[cg + 16 * x][j]);
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[y][x] = dot4(o[y], sv, acc[y][x]);
        }
      }
#pragma unroll
      for (int y = 0; y < 4; ++y)
#pragma unroll
        for (int x = 0; x < CT; ++x) acc[y][x] *= scale;
      for (int t = 0; t < rb + 4; ++t) {  // dP[r][t] = 0 for t > r
        float p[4], kh[CT];
#pragma unroll
        for (int y = 0; y < 4; ++y) p[y] = sm.BA[rb + y][t];
#pragma unroll
        for (int x = 0; x < CT; ++x) kh[x] = sm.Kh[t][cg + 16 * x];
#pragma unroll
        for (int y = 0; y < 4; ++y)
#pragma unroll
          for (int x = 0; x < CT; ++x) acc[y][x] = fmaf(p[y], kh[x], acc[y][x]);
      }
#pragma unroll
      for (int y = 0; y < 4; ++y)
#pragma unroll
        for (int x = 0; x < CT; ++x) {
          const int r = rb + y, c = cg + 16 * x;
          dgam[y][x] = acc[y][x] * sm.Qt[r][c];
          if (r < L) atomicAdd(a.acc_q + ((c0 + r) * H + h) * DK + c, acc[y][x] * E[y][x]);
        }
      // 9c. dK~ = -Z S^T + Diag(beta) (dA K^)  ->  dk (first part), dGamma; and the A part
      //     of dbeta, sum_s (K~ K^^T)_rs dA_rs = K~_r . (dA K^)_r
#pragma unroll
      for (int y = 0; y < 4; ++y)
#pragma unroll
        for (int x = 0; x < CT; ++x) acc[y][x] = 0.f;
      for (int t = 0; t < rb + 3; ++t) {  // dA[r][t] = 0 for t >= r
        float da4[4], kh[CT];
#pragma unroll
        for (int y = 0; y < 4; ++y) da4[y] = sm.BP[rb + y][t];
#pragma unroll
        for (int x = 0; x < CT; ++x) kh[x] = sm.Kh[t][cg + 16 * x];
#pragma unroll
        for (int y = 0; y < 4; ++y)
#pragma unroll
          for (int x = 0; x < CT; ++x) acc[y][x] = fmaf(da4[y], kh[x], acc[y][x]);
      }
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        const int r = rb + y;
        float db = 0.f;
#pragma unroll
        for (int x = 0; x < CT; ++x) db = fmaf(sm.Kt[r][cg + 16 * x], acc[y][x], db);
#pragma unroll
        for (int o2 = 8; o2 > 0; o2 >>= 1) db += __shfl_xor_sync(0xffffffffu, db, o2);
        if (cg == 0 && r < L) atomicAdd(a.acc_b + (c0 + r) * H + h, db);
        const float br = sm.bet[r];
#pragma unroll
        for (int x = 0; x < CT; ++x) acc[y][x] *= br;
      }
      for (int j = 0; j < DVS; j += 4) {
        float4 z[4];
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          z[y] = ld4(&sm.Y[rb + y][j]);
          z[y] = make_float4(-z[y].x, -z[y].y, -z[y].z, -z[y].w);
        }
#pragma unroll
        for (int x = 0; x < CT; ++x) {
          const float4 sv = ld4(&sm.S[cg + 16 * x][j]);
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[y][x] = dot4(z[y], sv, acc[y][x]);
        }
      }
#pragma unroll
      for (int y = 0; y < 4; ++y)
#pragma unroll
        for (int x = 0; x < CT; ++x) {
          const int r = rb + y, c = cg + 16 * x;
          dkk[y][x] = acc[y][x] * E[y][x];
          dgam[y][x] = fmaf(acc[y][x], sm.Kt[r][c], dgam[y][x]);
        }
      // 9d. dK^ = (U dS'^T) gl + dP^T Q~ + dG^T K~  ->  dk, dGamma, dgl parts
#pragma unroll
      for (int y = 0; y < 4; ++y)
#pragma unroll
        for (int x = 0; x < CT; ++x) acc[y][x] = 0.f;
      for (int j = 0; j < DVS; j += 4) {
        float4 u[4];
#pragma unroll
        for (int y = 0; y < 4; ++y) u[y] = ld4(&sm.U[rb + y][j]);
#pragma unroll
        for (int x = 0; x < CT; ++x) {
          const float4 d = ld4(&sm.dS[cg + 16 * x][j]);
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[y][x] = dot4(u[y], d, acc[y][x]);
        }
      }
      float dglp[CT];
#pragma unroll
      for (int x = 0; x < CT; ++x) {
        const int c = cg + 16 * x;
        const float gi = sm.gl[c];
        float part = rg == 0 ? sm.sdS[c] : 0.f;  // the decay of S itself
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          part = fmaf(sm.Kh[rb + y][c], acc[y][x], part);  // K^ (U dS'^T)
          acc[y][x] *= gi;
        }
        dglp[x] = part;
      }
      for (int t = rb; t < C; ++t) {  // dP[t][r] = 0 for t < r, dA[t][r] = 0 for t <= r
        float p[4], dg4[4], qt[CT], kt[CT];
        const float bt = sm.bet[t];  // dG = Diag(beta) dA
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          p[y] = sm.BA[t][rb + y];
          dg4[y] = bt * sm.BP[t][rb + y];
        }
#pragma unroll
        for (int x = 0; x < CT; ++x) {
          qt[x] = sm.Qt[t][cg + 16 * x];
          kt[x] = sm.Kt[t][cg + 16 * x];
        }
#pragma unroll
        for (int y = 0; y < 4; ++y)
#pragma unroll
          for (int x = 0; x < CT; ++x)
            acc[y][x] = fmaf(p[y], qt[x], fmaf(dg4[y], kt[x], acc[y][x]));
      }
#pragma unroll
      for (int y = 0; y < 4; ++y)
#pragma unroll
        for (int x = 0; x < CT; ++x) {
          const int r = rb + y, c = cg + 16 * x;
          dgam[y][x] = fmaf(-acc[y][x], sm.Kh[r][c], dgam[y][x]);
          if (r < L)
            atomicAdd(a.acc_k + ((c0 + r) * H + h) * DK + c, dkk[y][x] + acc[y][x] / E[y][x]);
        }
#pragma unroll
      for (int x = 0; x < CT; ++x) dglp_all[rg * DK + cg + 16 * x] = dglp[x];
      __syncthreads();
      // 9e. gl = E[L - 1] feeds the last live row; then the reverse cumulative sum over the
      //     live rows: local suffix sums plus the later groups' totals
#pragma unroll
      for (int x = 0; x < CT; ++x) {
        const int c = cg + 16 * x;
        float dgl = 0.f;
        for (int q2 = 0; q2 < 16; ++q2) dgl += dglp_all[q2 * DK + c];
        float suf = 0.f;
#pragma unroll
        for (int y = 3; y >= 0; --y) {
          const int r = rb + y;
          if (r == L - 1) dgam[y][x] = fmaf(dgl, sm.gl[c], dgam[y][x]);
          if (r < L) suf += dgam[y][x];
          dgam[y][x] = suf;
        }
        scan[rg * DK + c] = suf;
      }
      __syncthreads();
#pragma unroll
      for (int x = 0; x < CT; ++x) {
        const int c = cg + 16 * x;
        float later = 0.f;
        for (int q2 = rg + 1; q2 < 16; ++q2) later += scan[q2 * DK + c];
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int r = rb + y;
          if (r < L)
            atomicAdd(a.acc_g + ((c0 + r) * H + h) * DK + c,
                      ((live >> (y * CT + x)) & 1u) ? dgam[y][x] + later : 0.f);
        }
      }
    }
    __syncthreads();  // dS' and S are read above; dS is updated below

    // ---- 10. dS <- Diag(gl) dS' + scale Q~^T dO - K~^T Z        (DK x DVS tiles, IT x 4)
    {
      constexpr int JG = DVS / 4, IT = DK * DVS / (NT * 4);
      const int ib = (tid / JG) * IT, jc = tid % JG;
      float a1[IT][4] = {}, a2[IT][4] = {};
      for (int r = 0; r < C; ++r) {
        float qt[IT], kt[IT], o[4], z[4];
#pragma unroll
        for (int y = 0; y < IT; ++y) {
          qt[y] = sm.Qt[r][ib + y];
          kt[y] = sm.Kt[r][ib + y];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          o[x] = sm.dO[r][jc + JG * x];
          z[x] = sm.Y[r][jc + JG * x];
        }
#pragma unroll
        for (int y = 0; y < IT; ++y)
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            a1[y][x] = fmaf(qt[y], o[x], a1[y][x]);
            a2[y][x] = fmaf(kt[y], z[x], a2[y][x]);
          }
      }
#pragma unroll
      for (int y = 0; y < IT; ++y) {
        const int i = ib + y;
        const float gi = sm.gl[i];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int j = jc + JG * x;
          sm.dS[i][j] = fmaf(gi, sm.dS[i][j], fmaf(scale, a1[y][x], -a2[y][x]));
        }
      }
    }
  }
  __syncthreads();
  if (a.ds0) {
    for (int e = tid; e < DK * DVS; e += NT) {
      const int i = e / DVS, c = e % DVS;
      a.ds0[state_base + (int64_t)i * DV + c] = sm.dS[i][c];
    }
  }
}

// dq, dk, dg, dbeta in the input dtype from the fp32 accumulators
template <typename Tout>
__global__ void bwd_convert_kernel(const float* __restrict__ acc, Tout* __restrict__ out,
                                   int64_t n) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x)
    st_out(out + e, acc[e]);
}

// Through q = r / max(|r|, 1e-12): dr = (dq - q (q . dq)) / |r| (dq / 1e-12 at the floor).
// One warp per (token, head) row of the raw input r.
template <typename Tin, int DK>
__global__ void bwd_l2norm_kernel(const float* __restrict__ acc, const Tin* __restrict__ raw,
                                  Tin* __restrict__ out, int64_t rows) {
  constexpr int PL = DK / 32;
  const int lane = threadIdx.x & 31;
  for (int64_t row = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; row < rows;
       row += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    float x[PL], d[PL], ss = 0.f, dot = 0.f;
#pragma unroll
    for (int p = 0; p < PL; ++p) {
      x[p] = ld_in(raw + row * DK + lane + 32 * p);
      d[p] = acc[row * DK + lane + 32 * p];
      ss = fmaf(x[p], x[p], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float n = fmaxf(sqrtf(ss), 1e-12f), rn = 1.f / n;
#pragma unroll
    for (int p = 0; p < PL; ++p) dot = fmaf(x[p] * rn, d[p], dot);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (sqrtf(ss) <= 1e-12f) dot = 0.f;
#pragma unroll
    for (int p = 0; p < PL; ++p) st_out(out + row * DK + lane + 32 * p, (d[p] - x[p] * rn * dot) * rn);
  }
}

// Through g = lb * sigmoid(a): da = dg lb sigmoid(a) (1 - sigmoid(a)).
template <typename Tin>
__global__ void bwd_gate_kernel(const float* __restrict__ acc, const Tin* __restrict__ raw,
                                Tin* __restrict__ out, int64_t n, float lb) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    const float a = ld_in(raw + e);
    const float ex = __expf(-fabsf(a)), s = 1.f / (1.f + ex);
    const float sg = a >= 0.f ? s : ex * s;  // sigmoid(a)
    st_out(out + e, acc[e] * lb * sg * (1.f - sg));
  }
}

template <typename Tin, int DK, int DVS, int PRO>
cudaError_t launch_kernel(const BackwardArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(BwdSmem<DK, DVS>);
  cudaError_t e = cudaFuncSetAttribute(bwd_simt_kernel<Tin, DK, DVS, PRO>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)a.n_seqs * a.H * (a.dv / DVS);
  if (blocks == 0) return cudaSuccess;
  bwd_simt_kernel<Tin, DK, DVS, PRO><<<(unsigned)blocks, NT, smem, st>>>(a);
  return cudaGetLastError();
}

template <typename Tin, int DK, int DVS>
cudaError_t launch_width(const BackwardArgs& a, cudaStream_t st) {
  switch (a.prologue) {
    case 0: return launch_kernel<Tin, DK, DVS, 0>(a, st);
    case 1: return launch_kernel<Tin, DK, DVS, 1>(a, st);
    case 2: return launch_kernel<Tin, DK, DVS, 2>(a, st);
    default: return launch_kernel<Tin, DK, DVS, 3>(a, st);
  }
}

// One CTA per SM at most: 32-column slices unless they leave more than half the SMs idle,
// then 16-column slices (twice the CTAs; each recomputes the chunk's decay tiles and inverse)
template <typename Tin, int DK>
cudaError_t launch_typed(const BackwardArgs& a, cudaStream_t st) {
  const int64_t wide = (int64_t)a.n_seqs * a.H * (a.dv / 32);
  return 2 * wide <= 148 ? launch_width<Tin, DK, 16>(a, st) : launch_width<Tin, DK, 32>(a, st);
}

unsigned grid_for(int64_t n, int threads) {
  const int64_t want = (n + threads - 1) / threads;
  return (unsigned)(want < 148 * 16 ? (want > 0 ? want : 1) : 148 * 16);
}

template <typename Tin>
cudaError_t finish_typed(const BackwardArgs& a, void* dq, void* dk, void* dg, void* dbeta,
                         cudaStream_t st) {
  const int64_t rows = a.T_total * a.H, nk = rows * a.dk;
  if (rows == 0) return cudaSuccess;
  const int threads = 256;
  Tin* oq = static_cast<Tin*>(dq);
  Tin* ok = static_cast<Tin*>(dk);
  Tin* og = static_cast<Tin*>(dg);
  if (a.prologue & KDA_PROLOGUE_QK_L2NORM) {
    const unsigned gr = grid_for(rows * 32, threads);
    if (a.dk == 64) {
      bwd_l2norm_kernel<Tin, 64><<<gr, threads, 0, st>>>(a.acc_q, static_cast<const Tin*>(a.q), oq, rows);
      bwd_l2norm_kernel<Tin, 64><<<gr, threads, 0, st>>>(a.acc_k, static_cast<const Tin*>(a.k), ok, rows);
    } else {
      bwd_l2norm_kernel<Tin, 128><<<gr, threads, 0, st>>>(a.acc_q, static_cast<const Tin*>(a.q), oq, rows);
      bwd_l2norm_kernel<Tin, 128><<<gr, threads, 0, st>>>(a.acc_k, static_cast<const Tin*>(a.k), ok, rows);
    }
  } else {
    bwd_convert_kernel<Tin><<<grid_for(nk, threads), threads, 0, st>>>(a.acc_q, oq, nk);
    bwd_convert_kernel<Tin><<<grid_for(nk, threads), threads, 0, st>>>(a.acc_k, ok, nk);
  }
  if (a.prologue & KDA_PROLOGUE_GATE_SIGMOID)
    bwd_gate_kernel<Tin><<<grid_for(nk, threads), threads, 0, st>>>(
        a.acc_g, static_cast<const Tin*>(a.g), og, nk, a.lb);
  else
    bwd_convert_kernel<Tin><<<grid_for(nk, threads), threads, 0, st>>>(a.acc_g, og, nk);
  bwd_convert_kernel<Tin><<<grid_for(rows, threads), threads, 0, st>>>(
      a.acc_b, static_cast<Tin*>(dbeta), rows);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_backward(const BackwardArgs& a, kda_dtype dtype, cudaStream_t st) {
  if (dtype == KDA_F32)
    return a.dk == 64 ? launch_typed<float, 64>(a, st) : launch_typed<float, 128>(a, st);
  return a.dk == 64 ? launch_typed<__nv_bfloat16, 64>(a, st)
                    : launch_typed<__nv_bfloat16, 128>(a, st);
}

cudaError_t launch_backward_finish(const BackwardArgs& a, void* dq, void* dk, void* dg,
                                   void* dbeta, kda_dtype dtype, cudaStream_t st) {
  return dtype == KDA_F32 ? finish_typed<float>(a, dq, dk, dg, dbeta, st)
                          : finish_typed<__nv_bfloat16>(a, dq, dk, dg, dbeta, st);
}

}  // namespace kda
