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
//   dbeta_r = sum_c N_cr dT_cr + sum_{s<r} (K~ K^^T)_rs dA_rs
//   dP  = scale lower_incl(dO U^T)
//   dQ~ = scale dO S^T + dP K^,   dK~ = -Z S^T + dG K^
//   dK^ = dP^T Q~ + dG^T K~ + (U dS'^T) gl,   dgl = rowsum(S dS') + colsum(K^ (U dS'^T))
//   dGamma = dK~ K~ - dK^ K^ + dQ~ Q~ (+ dgl gl on the last row), dg' = reverse cumsum,
//   dg = dg' where g >= lb,   dq = dQ~ E,   dk = dK~ E + dK^ / E
//
// One CTA per (sequence, head, 32-column slice of d_v) walks the chunks backwards. The
// columns of S and dS evolve independently, so dv, dS and dS0 of a slice are complete in
// its CTA; dq, dk, dg and dbeta are sums over the slices and are added, in fp32, into
// accumulators that a final pass converts to the input dtype. The chunk start states
// come from a forward pass that keeps the state after every chunk.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int C = kChunk;
constexpr int DVS = 32;   // d_v columns per CTA
constexpr int NT = 256;   // threads per CTA

template <int DK>
struct BwdSmem {
  float Kt[C][DK + 1];   // K~
  float Kh[C][DK + 1];   // K^
  float Qt[C][DK + 1];   // Q~
  float BA[C][C + 1];    // A, then N^T dN, then dP
  float BN[C][C + 1];    // N = (I + A)^-1
  float BP[C][C + 1];    // P, then dT -> dN -> dA -> dG
  float S[DK][DVS + 1];  // chunk start state (slice)
  float dS[DK][DVS + 1]; // dL/d(chunk end state), updated in place to the chunk start
  float Y[C][DVS + 1];   // V - K~ S, then Z = T^T dU (= dL/dV)
  float U[C][DVS + 1];
  float dO[C][DVS + 1];
  float dU[C][DVS + 1];
  float gl[DK];
  float bet[C];
  float dbet[C];
  float part[NT / DK][DK];  // per row group: dgl parts, then suffix totals of dGamma
};

template <typename Tin, int DK>
__global__ void __launch_bounds__(NT, 1) bwd_simt_kernel(BackwardArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BwdSmem<DK>& sm = *reinterpret_cast<BwdSmem<DK>*>(smem_raw);
  constexpr int RG = NT / DK;   // row groups in the per-element pass
  constexpr int RPT = C / RG;   // rows per thread there
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
  const int r4 = tid / 4, cb = (tid % 4) * 8;  // (row, 8-column group) of C x DVS tiles
  const int tx = tid % 16, ty = tid / 16;      // 4x4 blocks of C x C tiles

  for (int64_t cc = n_chunks - 1; cc >= 0; --cc) {
    const int64_t c0 = t0 + cc * C;
    const int L = (t1 - c0) < C ? (int)(t1 - c0) : C;
    __syncthreads();  // the previous chunk's reads are done

    // ---- 0. decay tiles (threads < DK, one channel each); the slice's S, V, dO and beta
    if (tid < DK) {
      const int i = tid;
      float G = 0.f;
      for (int r = 0; r < C; ++r) {
        float kt = 0.f, kh = 0.f, qt = 0.f;
        if (r < L) {
          const int64_t off = ((c0 + r) * H + h) * DK + i;
          G += fmaxf(ld_in(g + off), lb);
          const float e = expf(G), ei = expf(-G);
          const float kv = ld_in(k + off);
          kt = kv * e;
          kh = kv * ei;
          qt = ld_in(q + off) * e;
        }
        sm.Kt[r][i] = kt;
        sm.Kh[r][i] = kh;
        sm.Qt[r][i] = qt;
      }
      sm.gl[i] = expf(G);
    } else {
      const float* src = nullptr;
      if (cc > 0) src = a.snap + ((snap0 + cc - 1) * H + h) * (int64_t)DK * DV + j0;
      else if (a.s0) src = a.s0 + state_base;
      for (int e = tid - DK; e < DK * DVS; e += NT - DK) {
        const int i = e / DVS, c = e % DVS;
        sm.S[i][c] = src ? src[(int64_t)i * DV + c] : 0.f;
      }
      for (int e = tid - DK; e < C * DVS; e += NT - DK) {
        const int r = e / DVS, c = e % DVS;
        const int64_t off = ((c0 + r) * H + h) * DV + j0 + c;
        sm.Y[r][c] = r < L ? ld_in(v + off) : 0.f;
        sm.dO[r][c] = (r < L && dout) ? ld_in(dout + off) : 0.f;
      }
      for (int r = tid - DK; r < C; r += NT - DK)
        sm.bet[r] = r < L ? ld_in(beta + (c0 + r) * H + h) : 0.f;
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
          sm.BA[r][c] = (c < r) ? sm.bet[r] * accA[x][y] : 0.f;
          sm.BP[r][c] = (c <= r) ? accP[x][y] : 0.f;
        }
    }
    __syncthreads();

    // ---- 2. N = (I + A)^-1 by forward substitution, one row at a time (rows past L:
    //         A is zero there, so N is the identity)
    if (tid < C) {
      for (int r = L; r < C; ++r) sm.BN[r][tid] = (r == tid) ? 1.f : 0.f;
    }
    for (int r = 0; r < L; ++r) {
      if (tid < C) {
        const int c = tid;
        float val = (c == r) ? 1.f : 0.f;
        for (int s2 = c; s2 < r; ++s2) val = fmaf(-sm.BA[r][s2], sm.BN[s2][c], val);
        sm.BN[r][c] = (c <= r) ? val : 0.f;
      }
      __syncthreads();
    }

    // ---- 3. Y = V - K~ S, then U = N Diag(beta) Y
    {
      float acc[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = 0.f;
      for (int i = 0; i < DK; ++i) {
        const float kt = sm.Kt[r4][i];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = fmaf(kt, sm.S[i][cb + c], acc[c]);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) sm.Y[r4][cb + c] -= acc[c];
    }
    __syncthreads();
    {
      float acc[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = 0.f;
      for (int s2 = 0; s2 <= r4; ++s2) {
        const float t = sm.BN[r4][s2] * sm.bet[s2];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = fmaf(t, sm.Y[s2][cb + c], acc[c]);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) sm.U[r4][cb + c] = acc[c];
    }
    __syncthreads();

    // ---- 4. dU = (K^ gl) dS' + scale P^T dO
    {
      float acc[8], acc2[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = acc2[c] = 0.f;
      for (int i = 0; i < DK; ++i) {
        const float kb = sm.Kh[r4][i] * sm.gl[i];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = fmaf(kb, sm.dS[i][cb + c], acc[c]);
      }
      for (int t = r4; t < C; ++t) {
        const float p = sm.BP[t][r4];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc2[c] = fmaf(p, sm.dO[t][cb + c], acc2[c]);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) sm.dU[r4][cb + c] = fmaf(scale, acc2[c], acc[c]);
    }
    __syncthreads();

    // ---- 5. dT = dU Y^T (over P, which is dead)
    {
      float acc[4][4];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
      for (int j = 0; j < DVS; ++j) {
        float du[4], yy[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          du[x] = sm.dU[ty * 4 + x][j];
          yy[x] = sm.Y[tx * 4 + x][j];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(du[x], yy[y], acc[x][y]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) sm.BP[ty * 4 + x][tx * 4 + y] = acc[x][y];
    }
    __syncthreads();

    // ---- 6. Z = Diag(beta) N^T dU (= dL/dV, over Y); dbeta from T = N Diag(beta)
    {
      float acc[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = 0.f;
      for (int t = r4; t < C; ++t) {
        const float nv = sm.BN[t][r4];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = fmaf(nv, sm.dU[t][cb + c], acc[c]);
      }
      const float b = sm.bet[r4];
#pragma unroll
      for (int c = 0; c < 8; ++c) sm.Y[r4][cb + c] = b * acc[c];
      if (r4 < L) {
        Tin* o = dvo + ((c0 + r4) * H + h) * DV + j0 + cb;
#pragma unroll
        for (int c = 0; c < 8; ++c) st_out(o + c, b * acc[c]);
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
      float acc[4][4];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
      for (int c = 0; c < C; ++c) {  // (N^T dN)[r][s] = sum_c N[c][r] dN[c][s]
        float nv[4], dn[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          nv[x] = sm.BN[c][ty * 4 + x];
          dn[x] = sm.BP[c][tx * 4 + x];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(nv[x], dn[y], acc[x][y]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) sm.BA[ty * 4 + x][tx * 4 + y] = acc[x][y];
    }
    __syncthreads();
    {
      float acc[4][4];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
      for (int c = 0; c < C; ++c) {  // dA[r][s] = -sum_c (N^T dN)[r][c] N[s][c]
        float tv[4], nv[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          tv[x] = sm.BA[ty * 4 + x][c];
          nv[x] = sm.BN[tx * 4 + x][c];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(tv[x], nv[y], acc[x][y]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) sm.BP[ty * 4 + x][tx * 4 + y] = -acc[x][y];
    }
    __syncthreads();

    // ---- 8. dG = strict_lower(Diag(beta) dA) in place, with dbeta += sum_s G dA (G = K~ K^^T
    //         recomputed); dP = scale lower_incl(dO U^T) over (N^T dN)
    {
      float accG[4][4], accP[4][4];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) accG[x][y] = accP[x][y] = 0.f;
      for (int i = 0; i < DK; ++i) {
        float kt[4], kh[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          kt[x] = sm.Kt[ty * 4 + x][i];
          kh[x] = sm.Kh[tx * 4 + x][i];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) accG[x][y] = fmaf(kt[x], kh[y], accG[x][y]);
      }
      for (int j = 0; j < DVS; ++j) {
        float d[4], u[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          d[x] = sm.dO[ty * 4 + x][j];
          u[x] = sm.U[tx * 4 + x][j];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) accP[x][y] = fmaf(d[x], u[y], accP[x][y]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int r = ty * 4 + x;
        const float br = sm.bet[r];
        float db = 0.f;
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int c = tx * 4 + y;
          const float da = sm.BP[r][c];
          if (c < r) db = fmaf(accG[x][y], da, db);
          sm.BP[r][c] = (c < r) ? br * da : 0.f;
          sm.BA[r][c] = (c <= r) ? scale * accP[x][y] : 0.f;
        }
        atomicAdd(&sm.dbet[r], db);
      }
    }
    __syncthreads();
    if (tid < L) atomicAdd(a.acc_b + (c0 + tid) * H + h, sm.dbet[tid]);

    // ---- 9. per (row group, channel i): dQ~, dK~, dK^ -> dq, dk; dGamma -> dg
    {
      const int i = tid % DK, rg = tid / DK, rb = rg * RPT;
      float E[RPT], dgam[RPT], dkk[RPT];
      uint32_t live = 0;  // bit rr: g >= lb (the clamp passes the gradient)
      {
        float G = 0.f;
        for (int r = 0; r < rb + RPT; ++r) {
          float gr = 0.f;
          if (r < L) gr = ld_in(g + ((c0 + r) * H + h) * DK + i);
          G += r < L ? fmaxf(gr, lb) : 0.f;
          if (r >= rb) {
            E[r - rb] = expf(G);
            if (gr >= lb) live |= 1u << (r - rb);
          }
        }
      }
      const float gli = sm.gl[i];
      float dglp = 0.f;
#pragma unroll 1
      for (int rr = 0; rr < RPT; ++rr) {
        const int r = rb + rr;
        // dQ~ = scale dO S^T + dP K^
        float a1 = 0.f, a2 = 0.f;
        for (int j = 0; j < DVS; ++j) a1 = fmaf(sm.dO[r][j], sm.S[i][j], a1);
        for (int t = 0; t <= r; ++t) a2 = fmaf(sm.BA[r][t], sm.Kh[t][i], a2);
        const float dqt = fmaf(scale, a1, a2);
        // dK~ = -Z S^T + dG K^
        float b1 = 0.f, b2 = 0.f;
        for (int j = 0; j < DVS; ++j) b1 = fmaf(sm.Y[r][j], sm.S[i][j], b1);
        for (int t = 0; t < r; ++t) b2 = fmaf(sm.BP[r][t], sm.Kh[t][i], b2);
        const float dkt = b2 - b1;
        // dK^ = dP^T Q~ + dG^T K~ + (U dS'^T) gl
        float c1 = 0.f, c2 = 0.f, dkb = 0.f;
        for (int t = r; t < C; ++t) c1 = fmaf(sm.BA[t][r], sm.Qt[t][i], c1);
        for (int t = r + 1; t < C; ++t) c2 = fmaf(sm.BP[t][r], sm.Kt[t][i], c2);
        for (int j = 0; j < DVS; ++j) dkb = fmaf(sm.U[r][j], sm.dS[i][j], dkb);
        const float dkh = c1 + c2 + dkb * gli;
        const float kh = sm.Kh[r][i];
        dglp = fmaf(kh, dkb, dglp);
        dgam[rr] = dkt * sm.Kt[r][i] - dkh * kh + dqt * sm.Qt[r][i];
        dkk[rr] = dkt * E[rr] + dkh / E[rr];
        if (r < L) atomicAdd(a.acc_q + ((c0 + r) * H + h) * DK + i, dqt * E[rr]);
      }
      if (rg == 0) {
        for (int j = 0; j < DVS; ++j) dglp = fmaf(sm.S[i][j], sm.dS[i][j], dglp);
      }
      sm.part[rg][i] = dglp;
      __syncthreads();
      float dgl = 0.f;
#pragma unroll
      for (int q2 = 0; q2 < RG; ++q2) dgl += sm.part[q2][i];
      // the end-of-chunk decay gl = E[L - 1] feeds the last live row's dGamma
      if (L - 1 >= rb && L - 1 < rb + RPT) dgam[L - 1 - rb] = fmaf(dgl, gli, dgam[L - 1 - rb]);
      // reverse cumulative sum over the live rows: local suffix sums, then the later groups
      float suf = 0.f;
#pragma unroll
      for (int rr = RPT - 1; rr >= 0; --rr) {
        if (rb + rr < L) suf += dgam[rr];
        dgam[rr] = suf;
      }
      __syncthreads();  // every group has read part[] as dgl parts
      sm.part[rg][i] = suf;
      __syncthreads();
      float later = 0.f;
      for (int q2 = rg + 1; q2 < RG; ++q2) later += sm.part[q2][i];
#pragma unroll 1
      for (int rr = 0; rr < RPT; ++rr) {
        const int r = rb + rr;
        if (r >= L) break;
        const int64_t off = ((c0 + r) * H + h) * DK + i;
        atomicAdd(a.acc_k + off, dkk[rr]);
        atomicAdd(a.acc_g + off, ((live >> rr) & 1u) ? dgam[rr] + later : 0.f);
      }
    }
    __syncthreads();  // dS' is read above; it is updated below

    // ---- 10. dS <- Diag(gl) dS' + scale Q~^T dO - K~^T Z (the start state's gradient)
    for (int e = tid; e < DK * DVS; e += NT) {
      const int i = e / DVS, j = e % DVS;
      float a1 = 0.f, a2 = 0.f;
      for (int r = 0; r < C; ++r) {
        a1 = fmaf(sm.Qt[r][i], sm.dO[r][j], a1);
        a2 = fmaf(sm.Kt[r][i], sm.Y[r][j], a2);
      }
      sm.dS[i][j] = fmaf(sm.gl[i], sm.dS[i][j], fmaf(scale, a1, -a2));
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

template <typename Tin, int DK>
cudaError_t launch_typed(const BackwardArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(BwdSmem<DK>);
  cudaError_t e = cudaFuncSetAttribute(bwd_simt_kernel<Tin, DK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)a.n_seqs * a.H * (a.dv / DVS);
  if (blocks == 0) return cudaSuccess;
  bwd_simt_kernel<Tin, DK><<<(unsigned)blocks, NT, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_backward(const BackwardArgs& a, kda_dtype dtype, cudaStream_t st) {
  if (dtype == KDA_F32)
    return a.dk == 64 ? launch_typed<float, 64>(a, st) : launch_typed<float, 128>(a, st);
  return a.dk == 64 ? launch_typed<__nv_bfloat16, 64>(a, st)
                    : launch_typed<__nv_bfloat16, 128>(a, st);
}

cudaError_t launch_backward_convert(const float* acc, void* out, int64_t n, kda_dtype dtype,
                                    cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t want = (n + threads - 1) / threads;
  const unsigned blocks = (unsigned)(want < 148 * 16 ? want : 148 * 16);
  if (dtype == KDA_F32)
    bwd_convert_kernel<float><<<blocks, threads, 0, st>>>(acc, static_cast<float*>(out), n);
  else
    bwd_convert_kernel<__nv_bfloat16><<<blocks, threads, 0, st>>>(
        acc, static_cast<__nv_bfloat16*>(out), n);
  return cudaGetLastError();
}

}  // namespace kda
