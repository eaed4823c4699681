// kda_prefill_tc.cu -- bf16 chunked prefill on the sm_100a tensor cores.
//
// Method: the chunk-parallel gated delta rule ("Kimi K3 深度拆解", section 4.2:
// chunk-parallel with an inter-chunk recurrence, tensor-core friendly blocking),
// with the log decay clamped from below ("3 分钟看懂 Kimi K3", Figure 3) so that
// exp(+-cumsum) over a 64-token chunk stays finite and every intra-chunk
// product is a dense matmul. Channel-wise decay per "Kimi K3 技術報告：三個架構改動",
// section "長度".
//
// Per chunk of L <= 64 tokens, with Gamma_r the inclusive prefix sum of the
// clamped log decays and gl = exp(Gamma_last):
//   K~ = K*exp(Gamma), K^ = K*exp(-Gamma), Q~ = Q*exp(Gamma), Kb = K^*gl
//   A  = Diag(beta) strict_lower(K~ K^^T)        P = lower_incl(Q~ K^^T)
//   T  = (I + A)^{-1} Diag(beta)                 (blocked forward substitution)
//   U  = T (V - K~ S)                            O = scale (Q~ S + P U)
//   S <- Diag(gl) S + Kb^T U
// Everything is computed in the transposed frame so every MMA has M = 128
// (the d_v index of S): X^T = S^T K~^T, U^T = (V - X)^T T^T, O^T += U^T P^T,
// Z = U^T Kb. Operands are bf16 tiles in shared memory, accumulators fp32 in
// tensor memory, and the state S stays fp32 in tensor memory for the whole walk.
//
// Long sequences are split into segments that run in parallel (two passes):
//   summary pass: per segment, the affine map S_end = M S_start + L, found by
//                 walking the segment with the 256-column state [M | L] started
//                 at [I | 0] (the M half sees V = 0);
//   combine:      S_start of every segment, sequentially per (sequence, head), fp32;
//   output pass:  per segment, the walk from its true S_start, writing outputs.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kda_internal.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = kChunk;  // 64
constexpr int D = 128;     // d_k = d_v on this path
constexpr int NT = 256;
constexpr uint32_t K8 = 8192, K16 = 16384, K32 = 32768;
constexpr int kTmemCols = 512;

struct TcArgs {
  CUtensorMap tm_q, tm_k, tm_g, tm_v;
  const __nv_bfloat16* beta;
  __nv_bfloat16* out;
  const float* s0;
  float* sT;
  const int32_t* cu;
  int32_t* status;
  float* mbuf;    // [pairs, max_segs-1, D, D]  summary: M (row-major [i][j])
  float* lbuf;    // [pairs, max_segs-1, D, D]  summary: L
  float* sstart;  // [pairs, max_segs, D, D]    start state of every segment
  int64_t T, T_total;
  int n_seqs, H;
  int seg_tokens, max_segs;
  float scale, lb;
};

// Shared-memory map (byte offsets from a 1024-aligned base). PC = output pass.
template <bool PC>
struct Sm {
  static constexpr int NB = PC ? 1 : 2;  // 128-column state blocks
  // KQ region: [K~ atom0 | X atom0 | K~ atom1 | X atom1] (8 KB each), X = Q~ (output
  // pass) or K^ (summary pass), so rows 0..127 form one M=128 operand.
  static constexpr uint32_t KQ = 0;
  static constexpr uint32_t KH = PC ? K32 : K8;        // K^ tile
  static constexpr uint32_t KH_AS = PC ? K8 : K16;     // its atom stride
  static constexpr uint32_t KB = PC ? K32 + K16 : K32;  // Kb tile (atom stride 8 KB)
  static constexpr uint32_t S = KB + K16;              // bf16 S^T blocks, 32 KB each
  static constexpr uint32_t Y = S + NB * K32;          // (V - X)^T, then U^T; 16 KB each
  static constexpr uint32_t T = Y + NB * K16;          // T (8 KB)
  static constexpr uint32_t P = T + K8;                // P (8 KB, output pass)
  static constexpr uint32_t NS = P + (PC ? K8 : 0);    // fp32 (I + A)^{-1}, 16 KB
  static constexpr uint32_t SQ = NS + K16;             // TMA staging q (output pass)
  static constexpr uint32_t SK = SQ + (PC ? K16 : 0);
  static constexpr uint32_t SG = SK + K16;
  static constexpr uint32_t SV = SG + K16;
  static constexpr uint32_t GL = SV + K16;             // float[128]
  static constexpr uint32_t TOT = GL + 512;            // float[4][128]
  static constexpr uint32_t BET = TOT + 2048;          // float[64]
  static constexpr uint32_t BT = BET + 256;            // float[3][256]
  static constexpr uint32_t BARS = BT + 3072;          // 3 mbarriers
  static constexpr uint32_t TPTR = BARS + 64;          // tensor-memory base
  static constexpr uint32_t BYTES = TPTR + 64;
  // fp32 A (strictly lower, beta-scaled) lives in the K^ tile once MMA-g has read it
  __device__ static constexpr uint32_t as_piece(int p) {
    return PC ? KH + p * K8 : KQ + K8 + p * K16;
  }
  // tensor-memory columns
  __device__ static constexpr uint32_t st(int b) { return PC ? 320 : 128 * b; }      // fp32 S^T
  __device__ static constexpr uint32_t xu(int b) { return PC ? 0 : 256 + 64 * b; }   // X^T, U^T
  static constexpr uint32_t YO = 64;                                                  // O^T
  static constexpr uint32_t G = PC ? 128 : 384;                                       // K~K^^T|Q~K^^T
  __device__ static constexpr uint32_t z(int b) { return PC ? 192 : 256 + 128 * b; }  // Kb^T U
};
static_assert(Sm<true>::BYTES + 1024 <= 232448, "output pass shared memory");
static_assert(Sm<false>::BYTES + 1024 <= 232448, "summary pass shared memory");

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  __nv_bfloat162 t = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(t);
}

__device__ __forceinline__ bool tc_seq_bounds(const TcArgs& a, int s, int64_t& t0, int64_t& t1) {
  if (a.cu == nullptr) {
    t0 = (int64_t)s * a.T;
    t1 = t0 + a.T;
    return true;
  }
  const int64_t c0 = a.cu[s], c1 = a.cu[s + 1];
  const bool ok = (c0 >= 0) && (c1 >= c0) && (c1 <= a.T_total) && (s != 0 || c0 == 0) &&
                  (s + 1 != a.n_seqs || c1 == a.T_total);
  if (!ok) {
    atomicExch(a.status, kDevBadSeqlens);
    return false;
  }
  t0 = c0;
  t1 = c1;
  return true;
}

// fp32 64x64 tile with a per-row XOR swizzle (conflict-free row and column access).
__device__ __forceinline__ float* f64x64(unsigned char* base, int r, int s) {
  return reinterpret_cast<float*>(base) + r * 64 + (s ^ (r & 31));
}

template <bool PC>
__global__ void __launch_bounds__(NT, 1) kda_tc_pass(const __grid_constant__ TcArgs a) {
  using L_ = Sm<PC>;
  constexpr int NB = L_::NB;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- which (sequence, head, segment) this CTA owns
  const int per = PC ? a.max_segs : a.max_segs - 1;
  const int seg = blockIdx.x % per;
  const int pair = blockIdx.x / per;
  const int s = pair / a.H, h = pair % a.H;
  int64_t t0, t1;
  if (!tc_seq_bounds(a, s, t0, t1)) return;
  const int64_t len = t1 - t0;
  const int nseg = len > 0 ? (int)((len + a.seg_tokens - 1) / a.seg_tokens) : 1;
  if (nseg > a.max_segs) {  // the caller's max_seqlen bound was too small
    if (seg == 0 && tid == 0) atomicExch(a.status, kDevBadSeqlens);
    return;
  }
  if (PC ? (seg >= nseg) : (seg >= nseg - 1)) return;
  const int64_t c_begin = t0 + (int64_t)seg * a.seg_tokens;
  const int64_t c_end = (c_begin + a.seg_tokens < t1) ? c_begin + a.seg_tokens : t1;

  float* gl = reinterpret_cast<float*>(sm + L_::GL);
  float* tot = reinterpret_cast<float*>(sm + L_::TOT);
  float* bet = reinterpret_cast<float*>(sm + L_::BET);
  float* bt = reinterpret_cast<float*>(sm + L_::BT);
  uint64_t* bar_qkg = reinterpret_cast<uint64_t*>(sm + L_::BARS);
  uint64_t* bar_v = bar_qkg + 1;
  uint64_t* bar_mma = bar_qkg + 2;
  uint32_t* tptr = reinterpret_cast<uint32_t*>(sm + L_::TPTR);

  if (warp == 0) {
    tmem_alloc(tptr, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_qkg, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    tma_prefetch_desc(&a.tm_k);
    tma_prefetch_desc(&a.tm_g);
    tma_prefetch_desc(&a.tm_v);
    if (PC) tma_prefetch_desc(&a.tm_q);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = *tptr;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const int row = tid & 127;   // TMEM lane = state column j for the state-side work
  const int half = tid >> 7;   // which warpgroup

  uint32_t ph_qkg = 0, ph_v = 0, ph_mma = 0;
  bool pend_qkg = false, pend_v = false, pend_mma = false;
  constexpr uint32_t qkg_bytes = (PC ? 3 : 2) * K16;

  auto issue_qkg = [&](int64_t cs) {
    mbar_arrive_expect_tx(bar_qkg, qkg_bytes);
    for (int bx = 0; bx < 2; ++bx) {
      const int x = h * D + 64 * bx;
      tma_load_2d(sm + L_::SK + bx * K8, &a.tm_k, bar_qkg, x, (int)cs);
      tma_load_2d(sm + L_::SG + bx * K8, &a.tm_g, bar_qkg, x, (int)cs);
      if (PC) tma_load_2d(sm + L_::SQ + bx * K8, &a.tm_q, bar_qkg, x, (int)cs);
    }
  };
  auto issue_v = [&](int64_t cs) {
    mbar_arrive_expect_tx(bar_v, K16);
    for (int bx = 0; bx < 2; ++bx)
      tma_load_2d(sm + L_::SV + bx * K8, &a.tm_v, bar_v, h * D + 64 * bx, (int)cs);
  };

  if (tid == 0 && c_begin < c_end) {
    issue_qkg(c_begin);
    issue_v(c_begin);
  }
  pend_qkg = pend_v = (c_begin < c_end);

  // ---- initial state: fp32 into tensor memory, bf16 copy as the MMA operand
  {
    const float* src = nullptr;
    if (PC) {
      if (nseg > 1) src = a.sstart + ((int64_t)pair * a.max_segs + seg) * D * D;
      else if (a.s0) src = a.s0 + (int64_t)pair * D * D;
    }
    for (int b = 0; b < NB; ++b) {
      if (!PC && b != half) continue;
      for (int c = (PC ? half * 64 : 0); c < (PC ? half * 64 + 64 : D); c += 32) {
        uint32_t v[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          float x;
          if (PC) x = src ? src[(int64_t)(c + t) * D + row] : 0.f;
          else x = (b == 0 && c + t == row) ? 1.f : 0.f;
          v[t] = __float_as_uint(x);
        }
        tmem_st32(tb + lane_base + L_::st(b) + c, v);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint4 pk;
          pk.x = pack_bf16(__uint_as_float(v[8 * q8 + 0]), __uint_as_float(v[8 * q8 + 1]));
          pk.y = pack_bf16(__uint_as_float(v[8 * q8 + 2]), __uint_as_float(v[8 * q8 + 3]));
          pk.z = pack_bf16(__uint_as_float(v[8 * q8 + 4]), __uint_as_float(v[8 * q8 + 5]));
          pk.w = pack_bf16(__uint_as_float(v[8 * q8 + 6]), __uint_as_float(v[8 * q8 + 7]));
          *reinterpret_cast<uint4*>(sm + L_::S + b * K32 + sw128_chunk(row, c / 8 + q8, K16)) =
              pk;
        }
      }
    }
    tmem_st_wait();
  }

  // beta for the first chunk (threads 0..63 keep the next chunk's value in a register)
  float bnext = 0.f;
  if (tid < C && c_begin + tid < c_end) bnext = __bfloat162float(a.beta[(c_begin + tid) * a.H + h]);

  tc_fence_before();
  fence_async_smem();
  __syncthreads();

  const int p = tid & 63, qr = tid >> 6;  // elementwise: channel pair, row quarter
  const int ch = 2 * p, bx = p >> 5, cofs = (p & 31) * 4;
  bool failed = false;

  for (int64_t c0 = c_begin; c0 < c_end && !failed; c0 += C) {
    const int L = (c_end - c0) < C ? (int)(c_end - c0) : C;
    const bool has_next = c0 + C < c_end;

    // ---------------- [A] decay prefix sums and the decayed operand tiles
    if (tid < C) {
      bet[tid] = bnext;
      bnext = 0.f;
      if (has_next && c0 + C + tid < c_end)
        bnext = __bfloat162float(a.beta[(c0 + C + tid) * a.H + h]);
    }
    {
      const bool ok = mbar_wait(bar_qkg, ph_qkg) && mbar_wait(bar_v, ph_v);
      if (__syncthreads_or(!ok)) { failed = true; break; }
      ph_qkg ^= 1;
      ph_v ^= 1;
      pend_qkg = pend_v = false;
    }
    float G0[16], G1[16];
    {
      float r0 = 0.f, r1 = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * qr + i;
        const float2 gg =
            unpack_bf16(*reinterpret_cast<const uint32_t*>(sm + L_::SG + bx * K8 + r * 128 + cofs));
        if (r < L) {
          r0 += fmaxf(gg.x, a.lb);
          r1 += fmaxf(gg.y, a.lb);
        }
        G0[i] = r0;
        G1[i] = r1;
      }
      tot[qr * 128 + ch] = r0;
      tot[qr * 128 + ch + 1] = r1;
    }
    __syncthreads();
    float kh0[16], kh1[16];
    {
      float o0 = 0.f, o1 = 0.f;
      for (int q = 0; q < qr; ++q) {
        o0 += tot[q * 128 + ch];
        o1 += tot[q * 128 + ch + 1];
      }
      if (qr == 3) {
        gl[ch] = expf(G0[15] + o0);
        gl[ch + 1] = expf(G1[15] + o1);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * qr + i;
        const float g0 = G0[i] + o0, g1 = G1[i] + o1;
        const float e0 = __expf(g0), e1 = __expf(g1);
        const float ei0 = __expf(-g0), ei1 = __expf(-g1);
        float2 kk = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm + L_::SK + bx * K8 + r * 128 + cofs));
        if (r >= L) kk = make_float2(0.f, 0.f);
        *reinterpret_cast<uint32_t*>(sm + L_::KQ + sw128_off(r, ch, K16)) =
            pack_bf16(kk.x * e0, kk.y * e1);
        kh0[i] = kk.x * ei0;
        kh1[i] = kk.y * ei1;
        *reinterpret_cast<uint32_t*>(sm + L_::KH + sw128_off(r, ch, L_::KH_AS)) =
            pack_bf16(kh0[i], kh1[i]);
        if (PC) {
          float2 qq =
              unpack_bf16(*reinterpret_cast<const uint32_t*>(sm + L_::SQ + bx * K8 + r * 128 + cofs));
          if (r >= L) qq = make_float2(0.f, 0.f);
          *reinterpret_cast<uint32_t*>(sm + L_::KQ + K8 + sw128_off(r, ch, K16)) =
              pack_bf16(qq.x * e0, qq.y * e1);
        }
      }
    }
    __syncthreads();  // gl ready; every read of the q/k/g staging is done
    if (tid == 0 && has_next) {
      issue_qkg(c0 + C);
      pend_qkg = true;
    }
    {
      const float gl0 = gl[ch], gl1 = gl[ch + 1];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * qr + i;
        *reinterpret_cast<uint32_t*>(sm + L_::KB + sw128_off(r, ch, K8)) =
            pack_bf16(kh0[i] * gl0, kh1[i] * gl1);
      }
    }
    fence_async_smem();
    __syncthreads();

    // ---------------- [B] MMA-g: [K~;Q~|K^] K^^T  and  MMA-a: S^T [K~;Q~]^T
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ig = idesc_bf16(128, 64, 0, 0);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t ko = (k >> 2) * K16 + (k & 3) * 32;
        const uint32_t kho = (k >> 2) * L_::KH_AS + (k & 3) * 32;
        umma_bf16(tb + L_::G, sdesc_sw128(sb + L_::KQ + ko, 16, 1024),
                  sdesc_sw128(sb + L_::KH + kho, 16, 1024), ig, k > 0);
      }
      const uint32_t ia = idesc_bf16(128, PC ? 128 : 64, 0, 0);
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t ko = (k >> 2) * K16 + (k & 3) * 32;
          umma_bf16(tb + L_::xu(b), sdesc_sw128(sb + L_::S + b * K32 + ko, 16, 1024),
                    sdesc_sw128(sb + L_::KQ + ko, 16, 1024), ia, k > 0);
        }
      umma_commit(bar_mma);
    }
    pend_mma = true;
    {
      const bool ok = mbar_wait(bar_mma, ph_mma);
      if (__syncthreads_or(!ok)) { failed = true; break; }
      ph_mma ^= 1;
      pend_mma = false;
    }
    tc_fence_after();

    // ---------------- [C] warpgroup 0: T = (I + A)^{-1} Diag(beta), P;  warpgroup 1: (V - X)^T
    if (half == 0) {
      if (tid < 64) {
        const int r = tid;
        const float br = bet[r];
#pragma unroll
        for (int cb = 0; cb < 64; cb += 32) {
          uint32_t v[32];
          tmem_ld32(tb + lane_base + L_::G + cb, v);
          tmem_ld_wait(v);
          float* arow = reinterpret_cast<float*>(sm + L_::as_piece(r >> 5)) + (r & 31) * 64;
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const int sc = cb + t;
            arow[sc ^ (r & 31)] = (sc < r) ? br * __uint_as_float(v[t]) : 0.f;
          }
        }
      } else if (PC) {
        const int r = tid - 64;
#pragma unroll
        for (int cb = 0; cb < 64; cb += 32) {
          uint32_t v[32];
          tmem_ld32(tb + lane_base + L_::G + cb, v);
          tmem_ld_wait(v);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            float f[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              const int sc = cb + 8 * q8 + t;
              f[t] = (sc <= r) ? __uint_as_float(v[8 * q8 + t]) : 0.f;
            }
            uint4 pk = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]),
                                  pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
            *reinterpret_cast<uint4*>(sm + L_::P + sw128_chunk(r, cb / 8 + q8, K8)) = pk;
          }
        }
      }
      named_bar(1, 128);
      auto As = [&](int r, int c) -> float {
        return reinterpret_cast<const float*>(sm + L_::as_piece(r >> 5))[(r & 31) * 64 + (c ^ (r & 31))];
      };
      unsigned char* ns = sm + L_::NS;
      // diagonal 16x16 blocks: lane l of warp w owns column 16w + l
      if (lane < 16) {
        const int w = warp;
        float n[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
          float val = (rr == lane) ? 1.f : 0.f;
#pragma unroll
          for (int ss = 0; ss < rr; ++ss) val -= As(16 * w + rr, 16 * w + ss) * n[ss];
          n[rr] = (rr < lane) ? 0.f : val;
        }
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) *f64x64(ns, 16 * w + rr, 16 * w + lane) = n[rr];
      }
      named_bar(1, 128);
      // off-diagonal blocks, by distance d from the diagonal:
      //   N_ij = -N_ii * sum_{k=j}^{i-1} A_ik N_kj
#pragma unroll 1
      for (int d = 1; d < 4; ++d) {
        const int nblk = 4 - d;
        for (int e = tid; e < nblk * 256; e += 128) {
          const int bj = e >> 8, bi = bj + d, rr = (e >> 4) & 15, cc = e & 15;
          const int r = 16 * bi + rr, c = 16 * bj + cc;
          float acc = 0.f;
          for (int kk = 16 * bj; kk < 16 * bi; ++kk) acc += As(r, kk) * *f64x64(ns, kk, c);
          bt[e] = acc;
        }
        named_bar(1, 128);
        for (int e = tid; e < nblk * 256; e += 128) {
          const int bj = e >> 8, bi = bj + d, rr = (e >> 4) & 15, cc = e & 15;
          float acc = 0.f;
#pragma unroll
          for (int m = 0; m < 16; ++m)
            acc += *f64x64(ns, 16 * bi + rr, 16 * bi + m) * bt[(bj << 8) + (m << 4) + cc];
          *f64x64(ns, 16 * bi + rr, 16 * bj + cc) = -acc;
        }
        named_bar(1, 128);
      }
      // T = N Diag(beta), lower triangle, bf16
      {
        const int r = tid >> 1, hf = tid & 1;
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const int c8 = hf * 4 + q8;
          float f[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int sc = 8 * c8 + t;
            f[t] = (sc <= r) ? *f64x64(ns, r, sc) * bet[sc] : 0.f;
          }
          *reinterpret_cast<uint4*>(sm + L_::T + sw128_chunk(r, c8, K8)) =
              make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                         pack_bf16(f[6], f[7]));
        }
      }
    } else {
      const int j = row;
#pragma unroll 1
      for (int b = 0; b < NB; ++b) {
        const bool use_v = PC || b == 1;
#pragma unroll
        for (int cb = 0; cb < 64; cb += 32) {
          uint32_t v[32];
          tmem_ld32(tb + lane_base + L_::xu(b) + cb, v);
          tmem_ld_wait(v);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            float f[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              const int r = cb + 8 * q8 + t;
              const float vv =
                  use_v ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                              sm + L_::SV + (j >> 6) * K8 + r * 128 + (j & 63) * 2))
                        : 0.f;
              f[t] = vv - __uint_as_float(v[8 * q8 + t]);
            }
            *reinterpret_cast<uint4*>(sm + L_::Y + b * K16 + sw128_chunk(j, cb / 8 + q8, K16)) =
                make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                           pack_bf16(f[6], f[7]));
          }
        }
      }
    }
    tc_fence_before();
    fence_async_smem();
    __syncthreads();
    if (tid == 0 && has_next) {  // every read of the v staging is done
      issue_v(c0 + C);
      pend_v = true;
    }

    // ---------------- [D] MMA-b: U^T = (V - X)^T T^T
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ib = idesc_bf16(128, 64, 0, 0);
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int k = 0; k < C / 16; ++k)
          umma_bf16(tb + L_::xu(b), sdesc_sw128(sb + L_::Y + b * K16 + k * 32, 16, 1024),
                    sdesc_sw128(sb + L_::T + k * 32, 16, 1024), ib, k > 0);
      umma_commit(bar_mma);
    }
    pend_mma = true;
    {
      const bool ok = mbar_wait(bar_mma, ph_mma);
      if (__syncthreads_or(!ok)) { failed = true; break; }
      ph_mma ^= 1;
      pend_mma = false;
    }
    tc_fence_after();

    // ---------------- [E] U^T -> bf16 operand
    {
      const int b = PC ? 0 : half;
      const int cb0 = PC ? half * 32 : 0, cb1 = PC ? half * 32 + 32 : 64;
      for (int cb = cb0; cb < cb1; cb += 32) {
        uint32_t v[32];
        tmem_ld32(tb + lane_base + L_::xu(b) + cb, v);
        tmem_ld_wait(v);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const float* f = reinterpret_cast<const float*>(v) + 8 * q8;
          *reinterpret_cast<uint4*>(sm + L_::Y + b * K16 + sw128_chunk(row, cb / 8 + q8, K16)) =
              make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                         pack_bf16(f[6], f[7]));
        }
      }
    }
    tc_fence_before();
    fence_async_smem();
    __syncthreads();

    // ---------------- [F] MMA-c: O^T += U^T P^T (output pass);  MMA-d: Z = U^T Kb
    if (tid == 0) {
      tc_fence_after();
      if (PC) {
        const uint32_t ic = idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int k = 0; k < C / 16; ++k)
          umma_bf16(tb + L_::YO, sdesc_sw128(sb + L_::Y + k * 32, 16, 1024),
                    sdesc_sw128(sb + L_::P + k * 32, 16, 1024), ic, 1);
      }
      const uint32_t id = idesc_bf16(128, 128, 0, 1);
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int k = 0; k < C / 16; ++k)
          umma_bf16(tb + L_::z(b), sdesc_sw128(sb + L_::Y + b * K16 + k * 32, 16, 1024),
                    sdesc_sw128(sb + L_::KB + k * 2048, K8, 1024), id, k > 0);
      umma_commit(bar_mma);
    }
    pend_mma = true;
    {
      const bool ok = mbar_wait(bar_mma, ph_mma);
      if (__syncthreads_or(!ok)) { failed = true; break; }
      ph_mma ^= 1;
      pend_mma = false;
    }
    tc_fence_after();

    // ---------------- [G] outputs; S <- Diag(gl) S + Z; bf16 S^T for the next chunk
    if (PC) {
      uint32_t v[32];
      tmem_ld32(tb + lane_base + L_::YO + half * 32, v);
      tmem_ld_wait(v);
      __nv_bfloat16* o = a.out + (c0 * a.H + h) * D + row;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const int r = half * 32 + t;
        if (r < L) o[(int64_t)r * a.H * D] = __float2bfloat16_rn(a.scale * __uint_as_float(v[t]));
      }
    }
    {
      const int b = PC ? 0 : half;
      const int c_lo = PC ? half * 64 : 0, c_hi = PC ? half * 64 + 64 : D;
      for (int c = c_lo; c < c_hi; c += 32) {
        uint32_t sv[32], zv[32];
        tmem_ld32(tb + lane_base + L_::st(b) + c, sv);
        tmem_ld_wait(sv);
        tmem_ld32(tb + lane_base + L_::z(b) + c, zv);
        tmem_ld_wait(zv);
#pragma unroll
        for (int t = 0; t < 32; ++t)
          sv[t] = __float_as_uint(fmaf(gl[c + t], __uint_as_float(sv[t]), __uint_as_float(zv[t])));
        tmem_st32(tb + lane_base + L_::st(b) + c, sv);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const float* f = reinterpret_cast<const float*>(sv) + 8 * q8;
          *reinterpret_cast<uint4*>(sm + L_::S + b * K32 + sw128_chunk(row, c / 8 + q8, K16)) =
              make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                         pack_bf16(f[6], f[7]));
        }
      }
      tmem_st_wait();
    }
    tc_fence_before();
    fence_async_smem();
    __syncthreads();
  }

  if (failed) {
    if (tid == 0) {
      atomicExch(a.status, kDevWaitTimeout);
      // let copies and MMAs that were issued finish before tensor memory is released
      if (pend_qkg) mbar_wait(bar_qkg, ph_qkg, 400000000LL);
      if (pend_v) mbar_wait(bar_v, ph_v, 400000000LL);
      if (pend_mma) mbar_wait(bar_mma, ph_mma, 400000000LL);
    }
  } else {
    // ---- write the final / summary state
    float* dst = nullptr;
    if (PC) {
      if (a.sT && seg == nseg - 1) dst = a.sT + (int64_t)pair * D * D;
    }
    for (int b = 0; b < NB; ++b) {
      if (!PC) {
        if (b != half) continue;
        const int64_t u = (int64_t)pair * (a.max_segs - 1) + seg;
        dst = (b == 0 ? a.mbuf : a.lbuf) + u * D * D;
      }
      if (dst == nullptr) continue;
      const int c_lo = PC ? half * 64 : 0, c_hi = PC ? half * 64 + 64 : D;
      for (int c = c_lo; c < c_hi; c += 32) {
        uint32_t v[32];
        tmem_ld32(tb + lane_base + L_::st(b) + c, v);
        tmem_ld_wait(v);
#pragma unroll
        for (int t = 0; t < 32; ++t) dst[(int64_t)(c + t) * D + row] = __uint_as_float(v[t]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tb, kTmemCols);
  }
}

// Start state of every segment: S_{j+1} = M_j S_j + L_j, fp32, one CTA per
// (sequence, head, 32-column slice).
__global__ void __launch_bounds__(256) kda_tc_combine(const __grid_constant__ TcArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* Ms = reinterpret_cast<float*>(smem_raw);  // [128][129]
  float* Ss = Ms + 128 * 129;                      // [128][32]
  const int pair = blockIdx.x >> 2, j0 = (blockIdx.x & 3) * 32;
  const int s = pair / a.H;
  int64_t t0, t1;
  if (!tc_seq_bounds(a, s, t0, t1)) return;
  const int64_t len = t1 - t0;
  const int nseg = len > 0 ? (int)((len + a.seg_tokens - 1) / a.seg_tokens) : 1;
  if (nseg <= 1 || nseg > a.max_segs) return;
  const int tid = threadIdx.x;
  float* st0 = a.sstart + (int64_t)pair * a.max_segs * D * D;
  for (int e = tid; e < D * 32; e += 256) {
    const int i = e >> 5, c = e & 31;
    const float x = a.s0 ? a.s0[(int64_t)pair * D * D + i * D + j0 + c] : 0.f;
    Ss[i * 32 + c] = x;
    st0[i * D + j0 + c] = x;
  }
  const int i = tid >> 1, cs = (tid & 1) * 16;
  for (int sg = 0; sg < nseg - 1; ++sg) {
    const int64_t u = (int64_t)pair * (a.max_segs - 1) + sg;
    const float* M = a.mbuf + u * D * D;
    const float* Lm = a.lbuf + u * D * D;
    __syncthreads();
    for (int e = tid; e < D * D / 4; e += 256) {
      const float4 m4 = reinterpret_cast<const float4*>(M)[e];
      const int r = (e * 4) >> 7, c = (e * 4) & 127;
      Ms[r * 129 + c] = m4.x;
      Ms[r * 129 + c + 1] = m4.y;
      Ms[r * 129 + c + 2] = m4.z;
      Ms[r * 129 + c + 3] = m4.w;
    }
    __syncthreads();
    float acc[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) acc[c] = Lm[i * D + j0 + cs + c];
    for (int k = 0; k < D; ++k) {
      const float m = Ms[i * 129 + k];
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[c] = fmaf(m, Ss[k * 32 + cs + c], acc[c]);
    }
    __syncthreads();
    float* dst = st0 + (int64_t)(sg + 1) * D * D;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      Ss[i * 32 + cs + c] = acc[c];
      dst[i * D + j0 + cs + c] = acc[c];
    }
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_map(CUtensorMap* m, const void* ptr, int64_t rows, int H) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(H) * D, static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(H) * D * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int64_t pow2_ceil(int64_t x) {
  int64_t p = 1;
  while (p < x) p <<= 1;
  return p;
}

}  // namespace

bool tc_path_applies(const kda_shape& s, int64_t T_total) {
  return s.dtype == KDA_BF16 && s.dk == D && s.dv == D && T_total > 0;
}

TcPlan tc_plan(int64_t T_total, int n_seqs, int H, int64_t max_len) {
  TcPlan p{};
  const int64_t chunks = (T_total + C - 1) / C + n_seqs;
  int64_t per_sm = (static_cast<int64_t>(H) * chunks + 147) / 148;
  if (per_sm < 8) per_sm = 8;
  const int64_t seg_chunks = pow2_ceil(per_sm);
  p.seg_tokens = static_cast<int>(seg_chunks * C > (int64_t(1) << 30) ? (int64_t(1) << 30)
                                                                       : seg_chunks * C);
  if (max_len < 1) max_len = 1;
  p.max_segs = static_cast<int>((max_len + p.seg_tokens - 1) / p.seg_tokens);
  if (p.max_segs < 1) p.max_segs = 1;
  p.pairs = static_cast<int64_t>(n_seqs) * H;
  const size_t state = sizeof(float) * D * D;
  p.ws_bytes = kWorkspaceHeader;
  if (p.max_segs > 1)
    p.ws_bytes += state * static_cast<size_t>(p.pairs) *
                  (2 * static_cast<size_t>(p.max_segs - 1) + static_cast<size_t>(p.max_segs));
  return p;
}

cudaError_t launch_prefill_tc(const PrefillArgs& pa, cudaStream_t st) {
  const TcPlan plan = tc_plan(pa.T_total, pa.n_seqs, pa.H, pa.max_len);
  if (pa.ws_bytes < plan.ws_bytes) return cudaErrorInvalidValue;
  TcArgs a;
  memset(&a, 0, sizeof a);
  if (!make_map(&a.tm_q, pa.q, pa.T_total, pa.H) || !make_map(&a.tm_k, pa.k, pa.T_total, pa.H) ||
      !make_map(&a.tm_g, pa.g, pa.T_total, pa.H) || !make_map(&a.tm_v, pa.v, pa.T_total, pa.H))
    return cudaErrorInvalidValue;
  a.beta = static_cast<const __nv_bfloat16*>(pa.beta);
  a.out = static_cast<__nv_bfloat16*>(pa.out);
  a.s0 = pa.s0;
  a.sT = pa.sT;
  a.cu = pa.cu;
  a.status = pa.status;
  const size_t state = static_cast<size_t>(D) * D;
  float* base = reinterpret_cast<float*>(pa.ws + kWorkspaceHeader);
  a.mbuf = base;
  a.lbuf = a.mbuf + state * plan.pairs * (plan.max_segs - 1);
  a.sstart = a.lbuf + state * plan.pairs * (plan.max_segs - 1);
  a.T = pa.T;
  a.T_total = pa.T_total;
  a.n_seqs = pa.n_seqs;
  a.H = pa.H;
  a.seg_tokens = plan.seg_tokens;
  a.max_segs = plan.max_segs;
  a.scale = pa.scale;
  a.lb = pa.lb;

  // dynamic shared memory limits are per function and per device: set them every call
  cudaError_t e = cudaFuncSetAttribute(kda_tc_pass<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Sm<true>::BYTES + 1024);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kda_tc_pass<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Sm<false>::BYTES + 1024);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kda_tc_combine, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (128 * 129 + 128 * 32) * 4);
  if (e != cudaSuccess) return e;

  if (plan.max_segs > 1) {
    kda_tc_pass<false><<<static_cast<unsigned>(plan.pairs * (plan.max_segs - 1)), NT,
                         Sm<false>::BYTES + 1024, st>>>(a);
    kda_tc_combine<<<static_cast<unsigned>(plan.pairs * 4), 256, (128 * 129 + 128 * 32) * 4,
                     st>>>(a);
  }
  kda_tc_pass<true><<<static_cast<unsigned>(plan.pairs * plan.max_segs), NT,
                      Sm<true>::BYTES + 1024, st>>>(a);
  return cudaGetLastError();
}

}  // namespace kda
