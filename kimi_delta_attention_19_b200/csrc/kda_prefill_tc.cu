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
constexpr int NT = 512;
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
  static constexpr uint32_t TOT = GL + 512;            // float[8][128]
  static constexpr uint32_t BET = TOT + 4096;          // float[64]
  static constexpr uint32_t BT = BET + 256;            // inverse scratch, float[32][36]
  static constexpr uint32_t BARS = BT + 4608;          // 3 mbarriers
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

// Global load issued where it stands (the asm keeps the compiler from sinking it
// next to its first use, one chunk later).
__device__ __forceinline__ uint16_t ldg_u16_early(const void* p) {
  unsigned short v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}
__device__ __forceinline__ uint4 pack8(const float* f) {
  return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                    pack_bf16(f[6], f[7]));
}

// One CTA of 16 warps per (sequence, head, segment). Warpgroup g = warp / 4 reaches
// every tensor-memory lane; phases split their columns over the four warpgroups.
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
  const int row = tid & 127;  // tensor-memory lane = state column j on the state side
  const int wg = tid >> 7;    // warpgroup 0..3

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

  // columns of the state this thread handles: output pass, warpgroup g takes
  // columns [32g, 32g+32); summary pass, block g/2, columns [64(g%2), +64)
  const int st_b = PC ? 0 : (wg >> 1);
  const int st_lo = PC ? 32 * wg : 64 * (wg & 1);
  const int st_hi = st_lo + (PC ? 32 : 64);

  // ---- initial state: fp32 into tensor memory, bf16 copy as the MMA operand
  {
    const float* src = nullptr;
    if (PC) {
      if (nseg > 1) src = a.sstart + ((int64_t)pair * a.max_segs + seg) * D * D;
      else if (a.s0) src = a.s0 + (int64_t)pair * D * D;
    }
    for (int c = st_lo; c < st_hi; c += 32) {
      uint32_t v[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        float x;
        if (PC) x = src ? src[(int64_t)(c + t) * D + row] : 0.f;
        else x = (st_b == 0 && c + t == row) ? 1.f : 0.f;
        v[t] = __float_as_uint(x);
      }
      tmem_st32(tb + lane_base + L_::st(st_b) + c, v);
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8)
        *reinterpret_cast<uint4*>(sm + L_::S + st_b * K32 + sw128_chunk(row, c / 8 + q8, K16)) =
            pack8(reinterpret_cast<const float*>(v) + 8 * q8);
    }
    tmem_st_wait();
  }

  // beta: threads 0..63 hold the next chunk's value (bf16 bits) in a register
  uint16_t bnext = 0;
  if (tid < C && c_begin + tid < c_end)
    bnext = ldg_u16_early(a.beta + (c_begin + tid) * a.H + h);

  tc_fence_before();
  fence_async_smem();
  __syncthreads();

  const int p = tid & 63, e8 = tid >> 6;  // elementwise: channel pair, group of 8 rows
  const int ch = 2 * p, bx = p >> 5, cofs = (p & 31) * 4;
  bool failed = false;

  for (int64_t c0 = c_begin; c0 < c_end && !failed; c0 += C) {
    const int L = (c_end - c0) < C ? (int)(c_end - c0) : C;
    const bool has_next = c0 + C < c_end;

    // ---------------- [A] decay prefix sums and the decayed operand tiles
    if (tid < C) {
      bet[tid] = bf16_bits_to_float(bnext);
      bnext = 0;
      if (has_next && c0 + C + tid < c_end)
        bnext = ldg_u16_early(a.beta + (c0 + C + tid) * a.H + h);
    }
    {
      const bool ok = mbar_wait(bar_qkg, ph_qkg) && mbar_wait(bar_v, ph_v);
      if (__syncthreads_or(!ok)) { failed = true; break; }
      ph_qkg ^= 1;
      ph_v ^= 1;
      pend_qkg = pend_v = false;
    }
    float G0[8], G1[8];
    {
      float r0 = 0.f, r1 = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 8 * e8 + i;
        const float2 gg =
            unpack_bf16(*reinterpret_cast<const uint32_t*>(sm + L_::SG + bx * K8 + r * 128 + cofs));
        if (r < L) {
          r0 += fmaxf(gg.x, a.lb);
          r1 += fmaxf(gg.y, a.lb);
        }
        G0[i] = r0;
        G1[i] = r1;
      }
      *reinterpret_cast<float2*>(tot + e8 * 128 + ch) = make_float2(r0, r1);
    }
    __syncthreads();
    {
      float o0 = 0.f, o1 = 0.f, s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float2 tq = *reinterpret_cast<const float2*>(tot + q * 128 + ch);
        if (q < e8) {
          o0 += tq.x;
          o1 += tq.y;
        }
        s0 += tq.x;
        s1 += tq.y;
      }
      // gamma at the last row of the chunk (rows past L add nothing)
      const float gl0 = expf(s0), gl1 = expf(s1);
      if (e8 == 7) *reinterpret_cast<float2*>(gl + ch) = make_float2(gl0, gl1);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 8 * e8 + i;
        const float g0 = G0[i] + o0, g1 = G1[i] + o1;
        const float e0 = __expf(g0), e1 = __expf(g1);
        const float ei0 = __expf(-g0), ei1 = __expf(-g1);
        float2 kk = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm + L_::SK + bx * K8 + r * 128 + cofs));
        if (r >= L) kk = make_float2(0.f, 0.f);
        *reinterpret_cast<uint32_t*>(sm + L_::KQ + sw128_off(r, ch, K16)) =
            pack_bf16(kk.x * e0, kk.y * e1);
        const float kh0 = kk.x * ei0, kh1 = kk.y * ei1;
        *reinterpret_cast<uint32_t*>(sm + L_::KH + sw128_off(r, ch, L_::KH_AS)) =
            pack_bf16(kh0, kh1);
        *reinterpret_cast<uint32_t*>(sm + L_::KB + sw128_off(r, ch, K8)) =
            pack_bf16(kh0 * gl0, kh1 * gl1);
        if (PC) {
          float2 qq =
              unpack_bf16(*reinterpret_cast<const uint32_t*>(sm + L_::SQ + bx * K8 + r * 128 + cofs));
          if (r >= L) qq = make_float2(0.f, 0.f);
          *reinterpret_cast<uint32_t*>(sm + L_::KQ + K8 + sw128_off(r, ch, K16)) =
              pack_bf16(qq.x * e0, qq.y * e1);
        }
      }
    }
    fence_async_smem();
    __syncthreads();  // operand tiles complete; every read of the q/k/g staging is done
    if (tid == 0 && has_next) {
      issue_qkg(c0 + C);
      pend_qkg = true;
    }

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

    // ---------------- [C] T = (I + A)^{-1} Diag(beta) and P (warps 0-3), (V - X)^T (4-15)
    // fp32 64x64 tiles A (in the K^ tile, no longer needed) and N = (I + A)^{-1}:
    // element (r, c) at r*64 + 4*((c/4) ^ (r%16)) + c%4, so 16-byte groups stay whole.
    auto a_ptr = [&](int r, int c) -> float* {
      return reinterpret_cast<float*>(sm + L_::as_piece(r >> 5)) + (r & 31) * 64 +
             ((((c >> 2) ^ (r & 15))) << 2) + (c & 3);
    };
    auto n_ptr = [&](int r, int c) -> float* {
      return reinterpret_cast<float*>(sm + L_::NS) + r * 64 + ((((c >> 2) ^ (r & 15))) << 2) +
             (c & 3);
    };
    if (warp < 2) {
      // A = Diag(beta) strict_lower(K~ K^^T): thread r owns row r (tensor-memory lanes 0..63)
      const int r = tid;
      const float br = bet[r];
#pragma unroll
      for (int cb = 0; cb < 64; cb += 32) {
        uint32_t v[32];
        tmem_ld32(tb + lane_base + L_::G + cb, v);
        tmem_ld_wait(v);
#pragma unroll
        for (int g4 = 0; g4 < 8; ++g4) {
          float4 f;
          const int c = cb + 4 * g4;
          f.x = (c + 0 < r) ? br * __uint_as_float(v[4 * g4 + 0]) : 0.f;
          f.y = (c + 1 < r) ? br * __uint_as_float(v[4 * g4 + 1]) : 0.f;
          f.z = (c + 2 < r) ? br * __uint_as_float(v[4 * g4 + 2]) : 0.f;
          f.w = (c + 3 < r) ? br * __uint_as_float(v[4 * g4 + 3]) : 0.f;
          *reinterpret_cast<float4*>(a_ptr(r, c)) = f;
        }
      }
    } else if (warp < 4) {
      if (PC) {
        // P = lower_incl(Q~ K^^T): tensor-memory lanes 64..127, bf16 operand tile
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
            *reinterpret_cast<uint4*>(sm + L_::P + sw128_chunk(r, cb / 8 + q8, K8)) = pack8(f);
          }
        }
      }
    } else {
      // (V - X)^T in 32-column units (block b, half), dealt to warpgroups 1..3
      const int j = row;
      for (int u = wg - 1; u < 2 * NB; u += 3) {
        const int b = u >> 1, cb = (u & 1) * 32;
        const bool use_v = PC || b == 1;
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
              pack8(f);
        }
      }
    }
    __syncthreads();  // A, P and (V - X)^T written; every read of the v staging is done
    if (tid == 0 && has_next) {
      issue_v(c0 + C);
      pend_v = true;
    }
    // diagonal 16x16 blocks of N by right-looking forward substitution:
    // warp w, half h -> block 2w+h; lane l -> column l of the block
    if (warp < 2) {
      const int base = 16 * (2 * warp + (lane >> 4)), l = lane & 15;
      float acc[16];
#pragma unroll
      for (int rr = 0; rr < 16; ++rr) acc[rr] = (rr == l) ? 1.f : 0.f;
#pragma unroll
      for (int rr = 0; rr < 16; ++rr) {
        const float nv = acc[rr];
        *n_ptr(base + rr, base + l) = nv;
#pragma unroll
        for (int r2 = rr + 1; r2 < 16; ++r2)
          acc[r2] = fmaf(-*a_ptr(base + r2, base + rr), nv, acc[r2]);
      }
    }
    __syncthreads();
    float* bt1 = bt;  // [2][16][16]
    float* bt2 = bt;  // [32][36]
    {
      // level 1: in each 32-block, N10 = -N11 (A10 N00) with 16x16 blocks
      const int b = tid >> 8, r = (tid >> 4) & 15, c = tid & 15;
      const int R0 = 32 * b, R1 = 32 * b + 16;
      float sacc = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) sacc = fmaf(*a_ptr(R1 + r, R0 + k), *n_ptr(R0 + k, R0 + c), sacc);
      bt1[b * 256 + r * 16 + c] = sacc;
      __syncthreads();
      float tacc = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) tacc = fmaf(*n_ptr(R1 + r, R1 + k), bt1[b * 256 + k * 16 + c], tacc);
      *n_ptr(R1 + r, R0 + c) = -tacc;
      *n_ptr(R0 + r, R1 + c) = 0.f;  // upper-right 16x16 block of each 32-block (read by level 2)
      __syncthreads();
    }
    {
      // level 2: N10 = -N11 (A10 N00) with 32x32 blocks
      const int r = tid >> 4, c = (tid & 15) * 2;
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float av = *a_ptr(32 + r, k);
        const float2 nn = *reinterpret_cast<const float2*>(n_ptr(k, c));
        s0 = fmaf(av, nn.x, s0);
        s1 = fmaf(av, nn.y, s1);
      }
      *reinterpret_cast<float2*>(bt2 + r * 36 + c) = make_float2(s0, s1);
      __syncthreads();
      float u0 = 0.f, u1 = 0.f;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float nv = *n_ptr(32 + r, 32 + k);
        const float2 bb = *reinterpret_cast<const float2*>(bt2 + k * 36 + c);
        u0 = fmaf(nv, bb.x, u0);
        u1 = fmaf(nv, bb.y, u1);
      }
      *reinterpret_cast<float2*>(n_ptr(32 + r, c)) = make_float2(-u0, -u1);
      __syncthreads();
    }
    {
      // T = N Diag(beta), lower triangle, as the bf16 operand: one 16-byte chunk per thread
      const int r = tid >> 3, c8 = tid & 7;
      float f[8];
#pragma unroll
      for (int h4 = 0; h4 < 2; ++h4) {
        const int c = 8 * c8 + 4 * h4;
        const float4 nn = *reinterpret_cast<const float4*>(n_ptr(r, c));
        const float4 bb = *reinterpret_cast<const float4*>(bet + c);
        f[4 * h4 + 0] = (c + 0 <= r) ? nn.x * bb.x : 0.f;
        f[4 * h4 + 1] = (c + 1 <= r) ? nn.y * bb.y : 0.f;
        f[4 * h4 + 2] = (c + 2 <= r) ? nn.z * bb.z : 0.f;
        f[4 * h4 + 3] = (c + 3 <= r) ? nn.w * bb.w : 0.f;
      }
      *reinterpret_cast<uint4*>(sm + L_::T + sw128_chunk(r, c8, K8)) = pack8(f);
    }
    tc_fence_before();
    fence_async_smem();
    __syncthreads();

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
    if (PC) {
      const int cb = 16 * wg;
      uint32_t v[16];
      tmem_ld16(tb + lane_base + L_::xu(0) + cb, v);
      tmem_ld_wait(v);
#pragma unroll
      for (int q8 = 0; q8 < 2; ++q8)
        *reinterpret_cast<uint4*>(sm + L_::Y + sw128_chunk(row, cb / 8 + q8, K16)) =
            pack8(reinterpret_cast<const float*>(v) + 8 * q8);
    } else {
      const int b = wg >> 1, cb = 32 * (wg & 1);
      uint32_t v[32];
      tmem_ld32(tb + lane_base + L_::xu(b) + cb, v);
      tmem_ld_wait(v);
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8)
        *reinterpret_cast<uint4*>(sm + L_::Y + b * K16 + sw128_chunk(row, cb / 8 + q8, K16)) =
            pack8(reinterpret_cast<const float*>(v) + 8 * q8);
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
      const int cb = 16 * wg;
      uint32_t v[16];
      tmem_ld16(tb + lane_base + L_::YO + cb, v);
      tmem_ld_wait(v);
      __nv_bfloat16* o = a.out + ((c0 + cb) * a.H + h) * D + row;
      const int64_t ostride = (int64_t)a.H * D;
#pragma unroll
      for (int t = 0; t < 16; ++t)
        if (cb + t < L) o[t * ostride] = __float2bfloat16_rn(a.scale * __uint_as_float(v[t]));
    }
    for (int c = st_lo; c < st_hi; c += 32) {
      uint32_t sv[32], zv[32];
      tmem_ld32(tb + lane_base + L_::st(st_b) + c, sv);
      tmem_ld32(tb + lane_base + L_::z(st_b) + c, zv);
      tmem_ld_wait(sv);
      tmem_ld_wait(zv);
#pragma unroll
      for (int t4 = 0; t4 < 8; ++t4) {
        const float4 g4 = *reinterpret_cast<const float4*>(gl + c + 4 * t4);
        sv[4 * t4 + 0] = __float_as_uint(fmaf(g4.x, __uint_as_float(sv[4 * t4 + 0]), __uint_as_float(zv[4 * t4 + 0])));
        sv[4 * t4 + 1] = __float_as_uint(fmaf(g4.y, __uint_as_float(sv[4 * t4 + 1]), __uint_as_float(zv[4 * t4 + 1])));
        sv[4 * t4 + 2] = __float_as_uint(fmaf(g4.z, __uint_as_float(sv[4 * t4 + 2]), __uint_as_float(zv[4 * t4 + 2])));
        sv[4 * t4 + 3] = __float_as_uint(fmaf(g4.w, __uint_as_float(sv[4 * t4 + 3]), __uint_as_float(zv[4 * t4 + 3])));
      }
      tmem_st32(tb + lane_base + L_::st(st_b) + c, sv);
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8)
        *reinterpret_cast<uint4*>(sm + L_::S + st_b * K32 + sw128_chunk(row, c / 8 + q8, K16)) =
            pack8(reinterpret_cast<const float*>(sv) + 8 * q8);
    }
    tmem_st_wait();
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
    // ---- write the final / summary state (row-major [i][j], fp32)
    float* dst = nullptr;
    if (PC) {
      if (a.sT && seg == nseg - 1) dst = a.sT + (int64_t)pair * D * D;
    } else {
      const int64_t u = (int64_t)pair * (a.max_segs - 1) + seg;
      dst = (st_b == 0 ? a.mbuf : a.lbuf) + u * D * D;
    }
    if (dst != nullptr) {
      for (int c = st_lo; c < st_hi; c += 32) {
        uint32_t v[32];
        tmem_ld32(tb + lane_base + L_::st(st_b) + c, v);
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
// (sequence, head, 16-column slice). M_{j+1} streams into shared memory
// (cp.async, double-buffered) while step j is computed.
constexpr int kCombSlices = 8, kCombCols = D / kCombSlices, kMStride = D + 4;
constexpr int kCombSmem = (2 * D * kMStride + D * kCombCols) * 4;

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(256) kda_tc_combine(const __grid_constant__ TcArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* Ms = reinterpret_cast<float*>(smem_raw);  // [2][128][132]
  float* Ss = Ms + 2 * D * kMStride;               // [128][16]
  const int pair = blockIdx.x / kCombSlices, j0 = (blockIdx.x % kCombSlices) * kCombCols;
  const int s = pair / a.H;
  int64_t t0, t1;
  if (!tc_seq_bounds(a, s, t0, t1)) return;
  const int64_t len = t1 - t0;
  const int nseg = len > 0 ? (int)((len + a.seg_tokens - 1) / a.seg_tokens) : 1;
  if (nseg <= 1 || nseg > a.max_segs) return;
  const int tid = threadIdx.x;
  float* st0 = a.sstart + (int64_t)pair * a.max_segs * D * D;
  auto load_m = [&](int sg, int buf) {
    const float* M = a.mbuf + ((int64_t)pair * (a.max_segs - 1) + sg) * D * D;
    float* dst = Ms + buf * D * kMStride;
    for (int e = tid; e < D * D / 4; e += 256) {
      const int r = e >> 5, c = (e & 31) * 4;
      cp_async16(dst + r * kMStride + c, M + r * D + c);
    }
    cp_async_commit();
  };
  load_m(0, 0);
  for (int e = tid; e < D * kCombCols; e += 256) {
    const int i = e / kCombCols, c = e % kCombCols;
    const float x = a.s0 ? a.s0[(int64_t)pair * D * D + i * D + j0 + c] : 0.f;
    Ss[i * kCombCols + c] = x;
    st0[i * D + j0 + c] = x;
  }
  const int i = tid >> 1, ch = (tid & 1) * 8;
  for (int sg = 0; sg < nseg - 1; ++sg) {
    const int buf = sg & 1;
    cp_async_wait_all();
    __syncthreads();  // M_sg landed; S of the previous step is visible; other buffer free
    if (sg + 1 < nseg - 1) load_m(sg + 1, buf ^ 1);
    const float* Lm = a.lbuf + ((int64_t)pair * (a.max_segs - 1) + sg) * D * D + i * D + j0 + ch;
    const float4 l0 = *reinterpret_cast<const float4*>(Lm);
    const float4 l1 = *reinterpret_cast<const float4*>(Lm + 4);
    float acc[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
    const float* Mrow = Ms + buf * D * kMStride + i * kMStride;
#pragma unroll 8
    for (int k = 0; k < D; ++k) {
      const float m = Mrow[k];
      const float4 s0 = *reinterpret_cast<const float4*>(Ss + k * kCombCols + ch);
      const float4 s1 = *reinterpret_cast<const float4*>(Ss + k * kCombCols + ch + 4);
      acc[0] = fmaf(m, s0.x, acc[0]);
      acc[1] = fmaf(m, s0.y, acc[1]);
      acc[2] = fmaf(m, s0.z, acc[2]);
      acc[3] = fmaf(m, s0.w, acc[3]);
      acc[4] = fmaf(m, s1.x, acc[4]);
      acc[5] = fmaf(m, s1.y, acc[5]);
      acc[6] = fmaf(m, s1.z, acc[6]);
      acc[7] = fmaf(m, s1.w, acc[7]);
    }
    __syncthreads();  // every read of S done
    float* dst = st0 + (int64_t)(sg + 1) * D * D + i * D + j0 + ch;
    *reinterpret_cast<float4*>(Ss + i * kCombCols + ch) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4*>(Ss + i * kCombCols + ch + 4) =
        make_float4(acc[4], acc[5], acc[6], acc[7]);
    *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  cp_async_wait_all();
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
                             kCombSmem);
  if (e != cudaSuccess) return e;

  if (plan.max_segs > 1) {
    kda_tc_pass<false><<<static_cast<unsigned>(plan.pairs * (plan.max_segs - 1)), NT,
                         Sm<false>::BYTES + 1024, st>>>(a);
    kda_tc_combine<<<static_cast<unsigned>(plan.pairs * kCombSlices), 256, kCombSmem, st>>>(a);
  }
  kda_tc_pass<true><<<static_cast<unsigned>(plan.pairs * plan.max_segs), NT,
                      Sm<true>::BYTES + 1024, st>>>(a);
  return cudaGetLastError();
}

}  // namespace kda
