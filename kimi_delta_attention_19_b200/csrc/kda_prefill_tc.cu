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
//   W  = T K~,  U0 = T V                         (the chunk's WY factors)
//   U  = U0 - W S                                O = scale (Q~ S + P U)
//   S <- Diag(gl) S + Kb^T U
// Everything above the last two lines depends on the chunk alone. An intra-chunk
// kernel computes it for every (chunk, head) at once and leaves -W^T, U0^T, Kb^T,
// Q~^T, P and gl in the workspace. The walk over the chunks of a sequence, which
// carries S, is then four tensor-core products per chunk in the transposed frame
// (M = 128, the d_v index of S):
//   U^T = U0^T + S^T (-W)^T,  (Q~ S)^T = S^T Q~^T,  O^T += U^T P^T,  S^T += U^T Kb
// with S fp32 in tensor memory for the whole walk and a bf16 copy as the operand.
//
// Long sequences are split into segments that are walked in parallel:
//   summary walk: per segment, the affine map S_end = M S_start + L, found by
//                 walking the segment with the 256-column state [M | L] started
//                 at [I | 0] (the M half sees V = 0, i.e. U0 = 0);
//   combine:      S_start of every segment, sequentially per (sequence, head), fp32;
//   output walk:  per segment, the walk from its true S_start, writing outputs.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "kda_internal.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = kChunk;  // 64
constexpr int D = 128;     // d_k = d_v on this path
constexpr uint32_t K8 = 8192, K16 = 16384, K32 = 32768;

// Workspace tiles per (chunk slot, head), every one a row-major array of 64-element
// (128-byte) bf16 rows, the layout the walk's products take as operands:
//   wt:  [128][64] -W^T  (row i = key channel, column r = token of the chunk)
//   qt:  [128][64] Q~^T  (row i, column r)
//   u0:  [128][64] U0^T  (row j = value channel, column r)
//   kbt: [128][64] Kb^T  (row i, column s)
//   p:   [64][64]  P     (row r, column s)
//   gl:  [128]     fp32
// Written by TMA stores from 128-byte-swizzled staging tiles, read by TMA.
constexpr size_t kTileBig = size_t(C) * D * 2;
constexpr size_t kTilePt = size_t(C) * C * 2;
constexpr size_t kTileGl = size_t(D) * 4;
constexpr size_t kTileBytes = 4 * kTileBig + kTilePt + kTileGl;

// Sequence boundaries as both kernels see them.
struct SeqTable {
  const int32_t* cu;  // [n_seqs + 1] or null (then sequence s is [s T, (s + 1) T))
  int32_t* status;
  int64_t T, T_total;
  int n_seqs;
};

__device__ __forceinline__ int64_t seq_start(const SeqTable& q, int s) {
  return q.cu ? static_cast<int64_t>(q.cu[s]) : static_cast<int64_t>(s) * q.T;
}

__device__ __forceinline__ bool seq_bounds_tc(const SeqTable& q, int s, int64_t& t0, int64_t& t1) {
  if (q.cu == nullptr) {
    t0 = (int64_t)s * q.T;
    t1 = t0 + q.T;
    return true;
  }
  const int64_t c0 = q.cu[s], c1 = q.cu[s + 1];
  const bool ok = (c0 >= 0) && (c1 >= c0) && (c1 <= q.T_total) && (s != 0 || c0 == 0) &&
                  (s + 1 != q.n_seqs || c1 == q.T_total);
  if (!ok) {
    atomicExch(q.status, kDevBadSeqlens);
    return false;
  }
  t0 = c0;
  t1 = c1;
  return true;
}

// Workspace slot of chunk 0 of the sequence starting at token t0; chunk c uses slot
// base + c. A sequence of n tokens has ceil(n/64) <= floor(n/64) + 1 chunks, so the
// slots of consecutive sequences never collide and all stay below
// ceil(T_total/64) + n_seqs.
__device__ __forceinline__ int64_t slot_base(int64_t t0, int s) { return t0 / C + s; }

// Segments of a sequence: segment 0 holds first_tokens tokens, segment j >= 1
// seg_tokens - (j - 1) seg_dec (all multiples of the chunk length; a sequence's last
// segment may be shorter). Segment j starts at token seg_offset(j) of the sequence.
__host__ __device__ __forceinline__ int64_t seg_offset(int seg, int first_tokens, int seg_tokens,
                                                       int seg_dec) {
  if (seg == 0) return 0;
  const int64_t j = seg - 1;
  return first_tokens + j * seg_tokens - static_cast<int64_t>(seg_dec) * (j * (j - 1) / 2);
}
// Segments that hold len tokens, counted up to max_segs + 1 (a sequence longer than the
// plan covers).
__host__ __device__ __forceinline__ int seg_count(int64_t len, int first_tokens, int seg_tokens,
                                                  int seg_dec, int max_segs) {
  int k = 1;
  while (k <= max_segs && seg_offset(k, first_tokens, seg_tokens, seg_dec) < len) ++k;
  return k;
}

// Sequence owning chunk slot u: the last one whose first slot is <= u.
__device__ __forceinline__ int owner_seq(const SeqTable& q, int64_t u) {
  int lo = 0, hi = q.n_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (slot_base(seq_start(q, mid), mid) <= u) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

struct IntraArgs {
  CUtensorMap tm_q, tm_k, tm_g;  // [T_total][H*128] bf16, 64x128 boxes, no swizzle
  CUtensorMap tm_v;              // the same shape, 64x64 boxes, 128-byte swizzle (an MMA operand as loaded)
  // workspace tiles (layouts above), stored from 128-byte-swizzled staging tiles:
  CUtensorMap tm_wt, tm_qt, tm_u0, tm_kbt;  // [tiles*128][64] bf16, 128x64 boxes
  CUtensorMap tm_p;                         // [tiles*64][64], 64x64 boxes
  SeqTable seq;
  const __nv_bfloat16* beta;
  float* gl;
  int* flags;  // the walk kernel's hand-off flags, zeroed here (block 0)
  int n_flags;
  int* queue;      // tile counter (zero at the call's start): CTAs take tiles gridDim.x + *queue++
  int64_t n_tiles; // chunk slots x heads
  int* tile_ready; // streamed schedule: per tile, set to 1 once its workspace tiles are written; else null
  int H;
  float lb;
};

struct WalkArgs {
  CUtensorMap tm_wt, tm_qt, tm_u0, tm_kbt;  // [tiles*128][64] bf16, 128x64 boxes, 128-byte swizzle
  CUtensorMap tm_p;                         // [tiles*64][64], 64x64 boxes
  SeqTable seq;
  const float* gl;
  __nv_bfloat16* out;
  const float* s0;
  float* sT;
  float* sstart;  // [pairs, max_segs, D, D]  start state of segment j >= 2 (and of 1 when j = 2 exists)
  int* flags;     // [pairs, max_segs]  sstart of segment j written (1) or never coming (2); zeroed per call
  const int* tile_ready;  // streamed schedule: per tile, 1 once the intra-chunk kernel wrote it; else null
  float* snap;    // [floor(T_total / (snap_every C)), H, D, D] or null: prefix-cache snapshots
  int snap_every; // chunks between snapshots
  int H;
  int first_tokens, seg_tokens, seg_dec;  // segment 0; segment j >= 1: seg_tokens - (j - 1) seg_dec
  int max_segs;
  int64_t max_len;  // the caller's bound on a sequence's length
  float scale;
};

__device__ __forceinline__ unsigned char* align1024(unsigned char* p) {
  return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 1023) &
                                          ~static_cast<uintptr_t>(1023));
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  __nv_bfloat162 t = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(t);
}
// (x, y) as bf16 pairs hi + lo: hi = bf16(x), lo = bf16(x - hi), so hi + lo carries
// about 16 bits of x; products of split factors keep fp32 accuracy on the tensor cores.
__device__ __forceinline__ void split_bf16(float x, float y, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  const float2 hf = __bfloat1622float2(h);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = pack_bf16(x - hf.x, y - hf.y);
}
// 2^x by the hardware approximation (ex2.approx.ftz.f32: relative error ~2^-22).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 1/x by the hardware approximation (rcp.approx.ftz.f32: relative error ~2^-23).
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint4 pack8(const float* f) {
  return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                    pack_bf16(f[6], f[7]));
}
// Two fp32 values as one 64-bit register pair (first value in the low half), and the
// packed fused multiply-add of sm_100 (two independent round-to-nearest fp32 FMAs).
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f32x2_split(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// bf16 pair (lower half first) -> fp32 pair
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t u) {
  return f32x2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
__device__ __forceinline__ uint32_t pack_bf16x2(uint64_t v) {
  const float2 f = f32x2_split(v);
  return pack_bf16(f.x, f.y);
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// Limit, in SM clocks, of the first wait on the inputs of the intra-chunk kernel (its TMA
// loads) and of each walk (its first stage). A test-only build of the library sets it to a
// few clocks and, with KDA_FIRST_WAIT_STUCK, points that wait at a spare mbarrier that
// nothing arrives at (inputs that never land), so that it always runs out and each
// kernel's bail-out path (record the error, tell the CTAs waiting for a state hand-off that
// it is not coming, let the copies and products in flight finish, free tensor memory,
// return) runs on the GPU; every other wait keeps its own limit.
#ifndef KDA_FIRST_WAIT_LIMIT
#define KDA_FIRST_WAIT_LIMIT 4000000000LL
#endif
#ifndef KDA_FIRST_WAIT_STUCK
#define KDA_FIRST_WAIT_STUCK 0
#endif

// Bounded wait by thread 0 alone (the others sleep in the barrier instead of polling),
// then a uniform decision: true when it timed out. The other threads then observe the
// completed phase themselves, which orders the data it guards before their reads.
__device__ __forceinline__ bool cta_wait_failed(uint64_t* bar, uint32_t parity,
                                                long long limit = 4000000000LL) {
  const bool ok = threadIdx.x != 0 || mbar_wait(bar, parity, limit);
  if (__syncthreads_or(!ok)) return true;
  if (threadIdx.x != 0) mbar_try_wait(bar, parity);
  return false;
}


// gpu-scope acquire load and release store of a flag another CTA (or kernel) reads
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Wait, bounded, for a flag another CTA sets (a state hand-off, a tile): true when it says published, false when
// it says the state is not coming or the wait ran out.
__device__ __forceinline__ bool flag_wait(const int* p, long long limit_cycles = 4000000000LL) {
  const long long t0 = clock64();
  int f;
  while ((f = ld_acquire_gpu(p)) == 0)  // one thread per CTA polls: a load per L2 round trip
    if (clock64() - t0 > limit_cycles) return false;
  return f == 1;
}

// Orders this thread's bulk-copy (async proxy) memory accesses with its plain ones, in
// every state space: a completed bulk store before a release, an acquire before a bulk load.
__device__ __forceinline__ void fence_proxy_async_all() {
  asm volatile("fence.proxy.async;" ::: "memory");
}

// ------------------------------------------------------------------ intra-chunk kernel
// Persistent CTAs of 8 warps, two per SM, each taking (chunk slot, head) tiles from a
// queue: its first tile is blockIdx.x, every next one gridDim.x + an atomic counter, drawn
// while the current tile is worked (so tiles start in about launch order, and no CTA is
// left with a long static share). Tensor memory and barriers are set up once per CTA,
// which also removes the gap between one CTA's end and the next one's start on an SM
// slot. Everything of a chunk
// that does not depend on the state: decay tiles, the Gram products on the tensor
// cores, the two 32x32 diagonal blocks of (I + A)^{-1} on the CUDA cores, and the WY
// factors W = T K~, U0 = T V on the tensor cores, blocked on the two token halves so
// that the off-diagonal block of the inverse is never formed.
constexpr int kIntraThreads = 256;
constexpr size_t kIntraQueueOffset = 128;  // the tile queue's counter, in the workspace header
constexpr int kPStoreThread = 64;   // warp 2, lane 0: issues (and waits for) the P store
struct IntraSm {
  // Raw inputs as loaded by TMA; each region is reused once its contents are read.
  static constexpr uint32_t SV = 0;        // V, swizzled: [64 s][64 j] boxes (U0's A operand)
  static constexpr uint32_t KQ = K16;      // [K~ a0 | Q~ a0 | K~ a1 | Q~ a1], 8 KB each
  static constexpr uint32_t SK = 3 * K16;  // raw k, then K^, then T
  static constexpr uint32_t SG = 4 * K16;  // raw g, then the inverse's fp32 scratch
  static constexpr uint32_t SQ = 5 * K16;
  static constexpr uint32_t KH = SK, T = SK;
  // 128-byte-swizzled staging tiles of the TMA stores to the workspace: Q~^T and Kb^T
  // (phase 2, over the raw g and q), P (phase 4, after K^), -W^T and U0^T (phases 8-9;
  // their token columns 0..31 are also the A operands of the second WY product)
  static constexpr uint32_t QTS = SG, KBS = SQ, PS = SK + K8, WTS = SG, U0S = SQ;
  // phase 4 scratch (fp32, free until the staging of -W^T and U0^T): the diagonal
  // blocks' rows of A and the solves' transposition (rows of 36 floats), A_21 (rows of
  // 32 floats)
  static constexpr uint32_t NLO = SG, A22 = SG + 4608, NHT = SG + 9216, A21 = SQ;
  // G = N_hi A_21 and -G, bf16 B operands of the second WY product, over the dead Q~ half
  static constexpr uint32_t GP = KQ + K8, GN = KQ + K8 + 4096;
  // float[2][64]: 1/|k row|, 1/|q row| (prologue)
  static constexpr uint32_t RN = SQ + K16;
  static constexpr uint32_t TOT = RN + 512;       // float[4][128] partial decay sums
  static constexpr uint32_t BET = TOT + 2048;     // float[64]
  static constexpr uint32_t BARS = BET + 256;
  static constexpr uint32_t TPTR = BARS + 64;
  static constexpr uint32_t BYTES = TPTR + 16;
  // tensor-memory columns: [K~;Q~] K^^T (G), W^T, U0^T
  static constexpr uint32_t G = 0, W = 64, U = 128, COLS = 256;
};
static_assert(2 * (IntraSm::BYTES + 1024 + 1024) <= 233472, "two intra-chunk CTAs per SM");

// PRO: the raw-input prologue flags (KDA_PROLOGUE_*), a template parameter so the plain
// instance carries no trace of it.
template <int PRO>
__global__ void __launch_bounds__(kIntraThreads, 2) kda_tc_intra(const __grid_constant__ IntraArgs a) {
  using L_ = IntraSm;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = align1024(smem_raw);
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // The next kernel of the stream may be scheduled once every CTA of this grid has started
  // (it waits for this grid's completion itself before reading its results).
  griddep_launch_dependents();
  if (blockIdx.x == 0)  // the walk kernel's hand-off flags start cleared on every call
    for (int i = tid; i < a.n_flags; i += kIntraThreads) a.flags[i] = 0;

  float* tot = reinterpret_cast<float*>(sm + L_::TOT);
  float* bet = reinterpret_cast<float*>(sm + L_::BET);
  float* rn = reinterpret_cast<float*>(sm + L_::RN);
  uint64_t* bar_in = reinterpret_cast<uint64_t*>(sm + L_::BARS);  // g, k, q
  uint64_t* bar_v = bar_in + 1;
  uint64_t* bar_mma = bar_in + 2;
  uint64_t* bar_none = bar_in + 3;  // nothing arrives (the test-only stuck first wait)
  uint32_t* tptr = reinterpret_cast<uint32_t*>(sm + L_::TPTR);
  int64_t* next_tile = reinterpret_cast<int64_t*>(sm + L_::TPTR + 8);

  if (warp == 0) {
    tmem_alloc(tptr, L_::COLS);
    tmem_relinquish();
  } else if (tid == 32) {
    mbar_init(bar_in, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_none, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = *tptr;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  // phases: bar_in and bar_v complete once per live tile, bar_mma three times
  int tiles_done = 0, mma_issued = 0, mma_done = 0;
  bool in_done = true, v_done = true, failed = false;

  int64_t tile = blockIdx.x;
  while (tile < a.n_tiles) {
  const int64_t u = tile / a.H;
  const int h = static_cast<int>(tile % a.H);
  // ---- the (sequence, chunk) that owns slot u: the last sequence whose base is <= u
  const int s = owner_seq(a.seq, u);
  int64_t t0 = 0, t1 = 0, c = -1;
  if (seq_bounds_tc(a.seq, s, t0, t1)) c = u - slot_base(t0, s);
  if (c < 0 || c * C >= t1 - t0) {  // a slot between two sequences (or a malformed table)
    if (tid == 0) *next_tile = gridDim.x + static_cast<int64_t>(atomicAdd(a.queue, 1));
    __syncthreads();
    tile = *next_tile;
    __syncthreads();
    continue;
  }
  const int64_t r0 = t0 + c * C;
  const int L = (t1 - r0) < C ? static_cast<int>(t1 - r0) : C;
  const uint32_t par = tiles_done & 1;  // this tile's phase of bar_in and bar_v

  if (tid == 32) {
    // v is needed last (by the WY products): its own barrier
    mbar_arrive_expect_tx(bar_in, 3 * K16);
    mbar_arrive_expect_tx(bar_v, K16);
    // k, g, q: one [64 rows][128] box each (256-byte rows, half the row requests of two
    // 64-column boxes); v: two swizzled 64-column boxes (the MMA operand layout)
    tma_load_2d(sm + L_::SG, &a.tm_g, bar_in, h * D, static_cast<int>(r0));
    tma_load_2d(sm + L_::SK, &a.tm_k, bar_in, h * D, static_cast<int>(r0));
    tma_load_2d(sm + L_::SQ, &a.tm_q, bar_in, h * D, static_cast<int>(r0));
    for (int bx = 0; bx < 2; ++bx)
      tma_load_2d(sm + L_::SV + bx * K8, &a.tm_v, bar_v, h * D + 64 * bx, static_cast<int>(r0));
  }
  in_done = v_done = false;
  // the CTA's next tile, drawn now and used once this one is done
  int64_t nxt = 0;
  if (tid == 0) nxt = gridDim.x + static_cast<int64_t>(atomicAdd(a.queue, 1));
  // beta of this thread's row, kept in a register until phase 1 is done (its load then
  // overlaps the TMA wait and phase 1 instead of delaying them)
  const float beta_r = tid < L ? __bfloat162float(a.beta[(r0 + tid) * a.H + h]) : 0.f;

  do {
    if (cta_wait_failed(KDA_FIRST_WAIT_STUCK ? bar_none : bar_in, par, KDA_FIRST_WAIT_LIMIT)) {
      failed = true;
      break;
    }
    in_done = true;
    if (L < C) {
      // a sequence's ragged last chunk: rows past L (the next sequence's tokens, or the
      // zero fill past the end) become k = q = 0 and g = 0, so no later step masks rows
      for (int e = tid; e < (C - L) * 32; e += kIntraThreads) {
        const int r = L + (e >> 5), w = e & 31;  // 16 16-byte words per 256-byte row
        const uint32_t off = r * 256 + (w & 15) * 16;
        const int which = w >> 4;  // 0: k and g, 1: q
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        if (which == 0) {
          *reinterpret_cast<uint4*>(sm + L_::SK + off) = z;
          *reinterpret_cast<uint4*>(sm + L_::SG + off) = z;
        } else {
          *reinterpret_cast<uint4*>(sm + L_::SQ + off) = z;
        }
      }
      __syncthreads();
    }
    if (PRO & KDA_PROLOGUE_QK_L2NORM) {
      // raw k and q rows -> 1 / max(|row|, 1e-12): two threads per row, 64 columns each,
      // the 16-byte words visited in a lane-rotated order (conflict-free)
      const int which = tid >> 7, r = (tid & 127) >> 1, hf = tid & 1;
      const unsigned char* src = sm + (which ? L_::SQ : L_::SK) + r * 256 + hf * 128;
      float ss = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const uint4 x4 = *reinterpret_cast<const uint4*>(src + 16 * ((w + lane) & 7));
        const uint32_t xs[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack_bf16(xs[e]);
          ss = fmaf(f.x, f.x, ss);
          ss = fmaf(f.y, f.y, ss);
        }
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      if (hf == 0) rn[which * 64 + r] = inv_l2(ss);
      __syncthreads();
    }
    // ---- 1. raw k, q into registers; the per-token decay factors e_i = exp(max(g_i, lb))
    //         (one exponential each) and their product over this thread's rows.
    //         Thread = (channel pair p, quarter qr of 16 rows).
    const int p = tid & 63, qr = tid >> 6;
    const int ch = 2 * p, bx = p >> 5;
    constexpr float kLog2e = 1.4426950408889634f;
    const float lb2 = a.lb * kLog2e;
    // per-channel-pair arithmetic in packed fp32 pairs (mul.rn.f32x2: the same products)
    uint32_t kraw[16], qraw[16];
    uint64_t E2[16];
    {
      uint64_t pr = f32x2(1.f, 1.f);
      const uint32_t off0 = 16 * qr * 256 + 4 * p;  // raw rows are 256 bytes
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t off = off0 + i * 256;
        kraw[i] = *reinterpret_cast<const uint32_t*>(sm + L_::SK + off);
        qraw[i] = *reinterpret_cast<const uint32_t*>(sm + L_::SQ + off);
        float2 gg = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm + L_::SG + off));
        if (PRO & KDA_PROLOGUE_GATE_SIGMOID) {
          // rows past a ragged chunk's end hold a zero fill, which is a log decay of 0 as
          // given but not as a pre-activation: they must stay decay-free
          const bool live = 16 * qr + i < L;
          gg.x = live ? gate_from_preact(gg.x, a.lb) : 0.f;
          gg.y = live ? gate_from_preact(gg.y, a.lb) : 0.f;
        }
        const float2 gl2 = f32x2_split(mul_f32x2(f32x2(gg.x, gg.y), f32x2(kLog2e, kLog2e)));
        E2[i] = f32x2(ex2_approx(fmaxf(gl2.x, lb2)), ex2_approx(fmaxf(gl2.y, lb2)));
        pr = mul_f32x2(pr, E2[i]);
      }
      *reinterpret_cast<float2*>(tot + qr * 128 + ch) = f32x2_split(pr);
    }
    if (tid < C) bet[tid] = beta_r;
    __syncthreads();  // every raw read is done: SK, SG and SQ may be overwritten
    // ---- 2. decay tiles: K~, Q~, K^ (MMA operands); Q~^T and Kb^T rows 2p, 2p + 1 (this
    //         thread's 16 tokens, 32 contiguous bytes each) and gl to the workspace.
    //         With gamma_i = exp(Gamma_i) the running product of the e's: gamma_i is the
    //         product of the earlier quarters' totals and this quarter's e's up to i;
    //         1 / gamma_i and gl / gamma_i are the product of this quarter's e's after i
    //         times 1 / (product up to this quarter's end) or the later quarters' totals.
    //         No reciprocal of a small number is taken per element, and each factor stays
    //         within [exp(64 lb), exp(-64 lb)] (finite: lb * 64 >= -80).
    //         Rows 16 qr + i: the swizzle term depends on i % 8 only.
    {
      uint32_t qt0[8], qt1[8], kb0[8], kb1[8];  // bf16 pairs along the token index
      uint64_t tq[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 t2 = *reinterpret_cast<const float2*>(tot + q * 128 + ch);
        tq[q] = f32x2(t2.x, t2.y);
      }
      uint64_t pre = f32x2(1.f, 1.f), suf = f32x2(1.f, 1.f);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (q < qr) pre = mul_f32x2(pre, tq[q]);
        else if (q > qr) suf = mul_f32x2(suf, tq[q]);
      }
      const uint64_t glp = mul_f32x2(mul_f32x2(mul_f32x2(tq[0], tq[1]), tq[2]), tq[3]);
      if (qr == 3) *reinterpret_cast<float2*>(a.gl + tile * D + ch) = f32x2_split(glp);
      const float2 pq = f32x2_split(mul_f32x2(pre, qr == 0 ? tq[0] : qr == 1 ? tq[1] : qr == 2 ? tq[2] : tq[3]));
      const uint64_t inv = f32x2(rcp_approx(pq.x), rcp_approx(pq.y));
      const int c3 = (ch & 63) >> 3;
      const uint32_t row0 = 2 * qr * 1024 + (ch & 7) * 2;
      const uint32_t kq0 = L_::KQ + bx * K16 + row0, kh0b = L_::KH + bx * K8 + row0;
      auto row_off = [&](int i) -> uint32_t {
        return (i >> 3) * 1024 + (i & 7) * 128 + ((c3 ^ (i & 7)) << 4);
      };
      auto kq_in = [&](int i, uint64_t& kk, uint64_t& qq) {
        kk = bf16x2_to_f32x2(kraw[i]);
        qq = bf16x2_to_f32x2(qraw[i]);
        if (PRO & KDA_PROLOGUE_QK_L2NORM) {
          const float rk = rn[16 * qr + i], rq = rn[64 + 16 * qr + i];
          kk = mul_f32x2(kk, f32x2(rk, rk));
          qq = mul_f32x2(qq, f32x2(rq, rq));
        }
      };
      // forward over the rows: K~ = k gamma, Q~ = q gamma
      uint64_t gm = pre;
      float qprev0 = 0.f, qprev1 = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        gm = mul_f32x2(gm, E2[i]);
        uint64_t kk, qq;
        kq_in(i, kk, qq);
        const uint64_t qtv = mul_f32x2(qq, gm);
        const float2 qtf = f32x2_split(qtv);
        const float qt0f = qtf.x, qt1f = qtf.y;
        *reinterpret_cast<uint32_t*>(sm + kq0 + row_off(i)) = pack_bf16x2(mul_f32x2(kk, gm));
        *reinterpret_cast<uint32_t*>(sm + kq0 + K8 + row_off(i)) = pack_bf16(qt0f, qt1f);
        if (i & 1) {
          qt0[i >> 1] = pack_bf16(qprev0, qt0f);
          qt1[i >> 1] = pack_bf16(qprev1, qt1f);
        } else {
          qprev0 = qt0f;
          qprev1 = qt1f;
        }
      }
      // rows ch, ch + 1 of the Q~^T staging tile (raw g is dead): tokens 16 qr .. + 15
      auto stage2 = [&](uint32_t base, const uint32_t* r0w, const uint32_t* r1w) {
        *reinterpret_cast<uint4*>(sm + base + sw128_chunk(ch, 2 * qr, 0)) =
            make_uint4(r0w[0], r0w[1], r0w[2], r0w[3]);
        *reinterpret_cast<uint4*>(sm + base + sw128_chunk(ch, 2 * qr + 1, 0)) =
            make_uint4(r0w[4], r0w[5], r0w[6], r0w[7]);
        *reinterpret_cast<uint4*>(sm + base + sw128_chunk(ch + 1, 2 * qr, 0)) =
            make_uint4(r1w[0], r1w[1], r1w[2], r1w[3]);
        *reinterpret_cast<uint4*>(sm + base + sw128_chunk(ch + 1, 2 * qr + 1, 0)) =
            make_uint4(r1w[4], r1w[5], r1w[6], r1w[7]);
      };
      stage2(L_::QTS, qt0, qt1);
      // backward over the rows: K^ = k / gamma, Kb = k gl / gamma
      uint64_t rs = f32x2(1.f, 1.f);
      float kprev0 = 0.f, kprev1 = 0.f;
#pragma unroll
      for (int i = 15; i >= 0; --i) {
        uint64_t kk, qq;
        kq_in(i, kk, qq);
        *reinterpret_cast<uint32_t*>(sm + kh0b + row_off(i)) = pack_bf16x2(mul_f32x2(kk, mul_f32x2(rs, inv)));
        const float2 kbf = f32x2_split(mul_f32x2(kk, mul_f32x2(rs, suf)));
        const float kb0f = kbf.x, kb1f = kbf.y;
        if (!(i & 1)) {
          kb0[i >> 1] = pack_bf16(kb0f, kprev0);
          kb1[i >> 1] = pack_bf16(kb1f, kprev1);
        } else {
          kprev0 = kb0f;
          kprev1 = kb1f;
        }
        rs = mul_f32x2(rs, E2[i]);
      }
      stage2(L_::KBS, kb0, kb1);
    }
    fence_async_smem();
    __syncthreads();
    // ---- 3. MMA-g: [K~; Q~] K^^T, M = 128 (64 rows of K~, then 64 of Q~), N = 64;
    //         Q~^T and Kb^T to the workspace by TMA
    if (tid == 32) {
      tma_store_2d(&a.tm_qt, sm + L_::QTS, 0, static_cast<int>(tile * D));
      tma_store_2d(&a.tm_kbt, sm + L_::KBS, 0, static_cast<int>(tile * D));
      bulk_commit();
    }
    if (tid == 0) {
      // the CTA's next tile (drawn at this tile's start): its inputs into L2 now, so that its
      // loads find them there
      if (nxt < a.n_tiles) {
        const int64_t un = nxt / a.H;
        const int hn = static_cast<int>(nxt % a.H);
        const int sn = owner_seq(a.seq, un);
        const int64_t tn0 = seq_start(a.seq, sn);
        const int64_t cn = un - slot_base(tn0, sn);
        if (cn >= 0) {
          const int yn = static_cast<int>(tn0 + cn * C);
          if (yn < a.seq.T_total) {
            tma_prefetch_2d(&a.tm_g, hn * D, yn);
            tma_prefetch_2d(&a.tm_k, hn * D, yn);
            tma_prefetch_2d(&a.tm_q, hn * D, yn);
            tma_prefetch_2d(&a.tm_v, hn * D, yn);
            tma_prefetch_2d(&a.tm_v, hn * D + 64, yn);
          }
        }
      }
      tc_fence_after();
      const uint32_t ig = idesc_bf16(128, 64, 0, 0);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t ko = (k >> 2) * K16 + (k & 3) * 32;
        const uint32_t kho = (k >> 2) * K8 + (k & 3) * 32;
        umma_bf16(tb + L_::G, sdesc_sw128(sb + L_::KQ + ko, 16, 1024),
                  sdesc_sw128(sb + L_::KH + kho, 16, 1024), ig, k > 0);
      }
      umma_commit(bar_mma);
    }
    ++mma_issued;
    if (tid == 32) bulk_wait_read();  // the staging tiles are rewritten from phase 4 on
    if (cta_wait_failed(bar_mma, mma_done & 1)) { failed = true; break; }
    ++mma_done;
    tc_fence_after();
    // ---- 4-6. T = (I + A)^{-1} Diag(beta), blocked on the two 32-token halves:
    //   (I + A)^{-1} = [[N_lo, 0], [N_21, N_hi]], N_bb = (I + A_bb)^{-1},
    //   N_21 = -N_hi A_21 N_lo. For X = T B (B = K~ or V: the WY factors W, U0) that is
    //     X_lo = T_lo B_lo,   X_hi = T_hi B_hi - G X_lo,   G = N_hi A_21,
    //   T_bb = N_bb Diag(beta_b): one product with the block-diagonal T, then a short
    //   one that subtracts G X_lo from the upper half (N_21 is never formed).
    //   Rows r < 64 of the Gram accumulator (tensor-memory lanes 0..63) hold K~_r K^^T:
    //   warps 0, 1, 4, 5 take one row each and a half hh of its 64 columns, so the
    //   diagonal block of rows 0..31 is in the half of warp 0, that of rows 32..63 in the
    //   half of warp 5, and A_21 in warp 1's. Warps 2 and 3 write P from lanes 64..127.
    //   Forward substitution on the CUDA cores, a right-hand-side column per lane, columns
    //   of the block broadcast from shared memory: warp 0 solves (I + A_11) N_lo = I,
    //   warp 5 (I + A_22) N_hi = I and, beside it, warp 6 (I + A_22) G = A_21 (so G costs
    //   no extra step on the chain; the three solvers sit on three different SM
    //   sub-partitions, warp % 4).
    const bool rowt = (warp & 3) < 2;                       // rows r < 64 of A
    const int hh = warp >> 2;                               // column half 32 hh ..
    const int rr = (warp & 3) * 32 + lane;                  // row (when rowt)
    // x = (I + A_bb)^{-1} rhs for this lane's column: x_r = rhs_r - sum_{s<r} A_rs x_s,
    // column by column: once x_s is final, every later row takes its term -A_rs x_s, so
    // the dependent chain is one fused multiply-add per column (the loads of column s do
    // not depend on x and run ahead). `ncols` holds -A^T as rows of 36 floats (row s =
    // -column s of A; entries r <= s are zero, so the pair that holds x_s itself is
    // updated by zero). Packed fp32 pairs (fma.rn.f32x2: two independent fp32 FMAs per
    // instruction), x held as pairs (x_2m, x_2m+1).
    auto fsub = [&](const float* ncols, auto rhs, float (&x)[32]) {
      uint64_t x2[16];
#pragma unroll
      for (int m = 0; m < 16; ++m) x2[m] = f32x2(rhs(2 * m), rhs(2 * m + 1));
#pragma unroll
      for (int c = 0; c < 31; ++c) {
        const float2 pc = f32x2_split(x2[c >> 1]);
        const float xc = (c & 1) ? pc.y : pc.x;
        const uint64_t xx = f32x2(xc, xc);
#pragma unroll
        for (int q = c >> 2; q < 8; ++q) {
          const float4 a4 = *reinterpret_cast<const float4*>(ncols + c * 36 + 4 * q);
          if (2 * q + 1 >= (c >> 1)) x2[2 * q + 1] = fma_f32x2(f32x2(a4.z, a4.w), xx, x2[2 * q + 1]);
          if (2 * q >= (c >> 1)) x2[2 * q] = fma_f32x2(f32x2(a4.x, a4.y), xx, x2[2 * q]);
        }
      }
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        const float2 v2 = f32x2_split(x2[m]);
        x[2 * m] = v2.x;
        x[2 * m + 1] = v2.y;
      }
    };
    // this lane's row r of A (in v) as column r of -A^T in dst (rows of 36 floats)
    float* const a22 = reinterpret_cast<float*>(sm + L_::A22);
    float* const a21 = reinterpret_cast<float*>(sm + L_::A21);
    auto put_cols = [&](float* dst, const uint32_t (&v)[32]) {
#pragma unroll
      for (int c = 0; c < 32; ++c) dst[c * 36 + lane] = -__uint_as_float(v[c]);
    };
    {
      uint32_t v[32];
      if (rowt || hh == 0) {  // warps 6 and 7 read no Gram row (P is warps 2 and 3's)
        tmem_ld32(tb + lane_base + L_::G + 32 * hh, v);
        tmem_ld_wait(v);
      }
      if (rowt) {
        // A = Diag(beta) strict_lower(K~ K^^T), row rr, columns 32 hh ..
        const float br = bet[rr];
        float f[32];  // this row of the block-diagonal T (zero off the blocks)
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const int c = 32 * hh + t;
          v[t] = __float_as_uint(c < rr ? br * __uint_as_float(v[t]) : 0.f);
          f[t] = 0.f;
        }
        if (warp == 1) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(a21 + lane * 32 + 4 * q) =
                make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                            __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
          group_sync(1, 96);  // warps 1, 5, 6: A_21's rows and A_22's columns are in place
        } else if (warp == 4) {
          // the upper-right block of T is zero
        } else {
          // warps 0 and 5: N_bb column `lane`, back through a transposition scratch so
          // that lane l ends with row l of N_bb; T_bb = N_bb Diag(beta_b)
          float* const scr = reinterpret_cast<float*>(sm + (warp == 0 ? L_::NLO : L_::NHT));
          const float* ncols;
          if (warp == 0) {
            put_cols(scr, v);
            __syncwarp();
            ncols = scr;
          } else {
            put_cols(a22, v);
            group_sync(1, 96);
            ncols = a22;
          }
          float x[32];
          fsub(ncols, [&](int r) { return r == lane ? 1.f : 0.f; }, x);
          __syncwarp();
#pragma unroll
          for (int r = 0; r < 32; ++r) scr[r * 36 + lane] = x[r];
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 n4 = *reinterpret_cast<const float4*>(scr + lane * 36 + 4 * q);
            const float nq[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) f[4 * q + e] = nq[e] * bet[32 * hh + 4 * q + e];
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(sm + L_::T + sw128_chunk(rr, 4 * hh + q, K8)) = pack8(f + 8 * q);
      } else if (hh == 0) {
        // P = lower_incl(Q~ K^^T): row r, both column halves (warps 2 and 3, so that warp 6
        // goes straight to G)
        const int r = (warp & 3) * 32 + lane - 64;
        auto stage_p = [&](const uint32_t (&pv)[32], int half) {
          float f[32];
#pragma unroll
          for (int t = 0; t < 32; ++t) f[t] = 32 * half + t <= r ? __uint_as_float(pv[t]) : 0.f;
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8)
            *reinterpret_cast<uint4*>(sm + L_::PS + sw128_chunk(r, 4 * half + q8, 0)) = pack8(f + 8 * q8);
        };
        stage_p(v, 0);
        tmem_ld32(tb + lane_base + L_::G + 32, v);
        tmem_ld_wait(v);
        stage_p(v, 1);
        fence_async_smem();
        group_sync(2, 64);  // warps 2, 3: P is staged
        if (tid == kPStoreThread) {  // P to the workspace
          tma_store_2d(&a.tm_p, sm + L_::PS, 0, static_cast<int>(tile * C));
          bulk_commit();
        }
      } else if (warp == 6) {
        // G = N_hi A_21, column `lane`, as +G and -G rows (bf16, K-major B operands): lane
        // pairs trade values, even lanes write a +G pair of columns and odd lanes the -G pair
        group_sync(1, 96);
        float y[32];
        fsub(a22, [&](int r) { return a21[r * 32 + lane]; }, y);
        const int odd = lane & 1;
#pragma unroll
        for (int r = 0; r < 32; ++r) {
          const float other = __shfl_xor_sync(0xffffffffu, y[r], 1);
          const uint32_t off = sw128_chunk(r, lane >> 3, 0) + (lane & 6) * 2;
          const uint32_t pr = odd ? pack_bf16(-other, -y[r]) : pack_bf16(y[r], other);
          *reinterpret_cast<uint32_t*>(sm + (odd ? L_::GN : L_::GP) + off) = pr;
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    if (cta_wait_failed(bar_v, par)) { failed = true; break; }  // also the barrier for T, P, +-G
    v_done = true;
    // ---- 7. W^T = K~^T T^T and U0^T = V^T T^T with the block-diagonal T: the lower token
    //         half is final, the upper one still lacks -G X_lo. K~ (in the Gram operand)
    //         and V (as loaded) serve as MN-major A operands: 64-element column groups LBO
    //         apart, 8-row groups 1024 bytes apart, 16 rows of K per instruction.
    if (tid == 0) {
      tc_fence_after();
      const uint32_t iw = idesc_bf16(128, 64, 1, 0);
#pragma unroll
      for (int k = 0; k < C / 16; ++k) {
        const uint64_t tdesc = sdesc_sw128(sb + L_::T + k * 32, 16, 1024);
        umma_bf16(tb + L_::W, sdesc_sw128(sb + L_::KQ + k * 2048, K16, 1024), tdesc, iw, k > 0);
        umma_bf16(tb + L_::U, sdesc_sw128(sb + L_::SV + k * 2048, K8, 1024), tdesc, iw, k > 0);
      }
      umma_commit(bar_mma);
    }
    ++mma_issued;
    if (cta_wait_failed(bar_mma, mma_done & 1)) { failed = true; break; }
    ++mma_done;
    tc_fence_after();
    // ---- 8. token columns 0..31 of -W^T (warps 0..3) and U0^T (warps 4..7) to the staging
    //         tiles: tensor-memory lane i holds row i
    const int i = (warp & 3) * 32 + lane;
    const uint32_t xcol = hh ? L_::U : L_::W;
    const uint32_t xst = hh ? L_::U0S : L_::WTS;
    const uint32_t xsign = hh ? 0u : 0x80000000u;
    {
      uint32_t v[32];
      tmem_ld32(tb + lane_base + xcol, v);
      tmem_ld_wait(v);
#pragma unroll
      for (int t = 0; t < 32; ++t) v[t] ^= xsign;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(sm + xst + sw128_chunk(i, q, 0)) =
            pack8(reinterpret_cast<const float*>(v) + 8 * q);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- 9. the upper token half: W_hi^T += (-W_lo^T) G^T, U0_hi^T += U0_lo^T (-G)^T,
    //         the staged lower halves as K-major A operands (K = 32 tokens)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ib = idesc_bf16(128, 32, 0, 0);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        umma_bf16(tb + L_::W + 32, sdesc_sw128(sb + L_::WTS + k * 32, 16, 1024),
                  sdesc_sw128(sb + L_::GP + k * 32, 16, 1024), ib, 1);
        umma_bf16(tb + L_::U + 32, sdesc_sw128(sb + L_::U0S + k * 32, 16, 1024),
                  sdesc_sw128(sb + L_::GN + k * 32, 16, 1024), ib, 1);
      }
      umma_commit(bar_mma);
    }
    ++mma_issued;
    if (cta_wait_failed(bar_mma, mma_done & 1)) { failed = true; break; }
    ++mma_done;
    tc_fence_after();
    {
      uint32_t v[32];
      tmem_ld32(tb + lane_base + xcol + 32, v);
      tmem_ld_wait(v);
#pragma unroll
      for (int t = 0; t < 32; ++t) v[t] ^= xsign;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(sm + xst + sw128_chunk(i, 4 + q, 0)) =
            pack8(reinterpret_cast<const float*>(v) + 8 * q);
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 32) {
      tma_store_2d(&a.tm_wt, sm + L_::WTS, 0, static_cast<int>(tile * D));
      tma_store_2d(&a.tm_u0, sm + L_::U0S, 0, static_cast<int>(tile * D));
      bulk_commit();
    }
  } while (0);
  // the workspace stores have read their staging tiles before the next tile's loads (or
  // the CTA's exit) reuse that shared memory (their writes are visible to the next kernel
  // once this grid completes)
  if (tid == 32 || tid == kPStoreThread) {
    if (a.tile_ready) {
      // streamed schedule: this tile's stores complete and ordered before the release below
      bulk_wait_all();
      fence_proxy_async_all();
    } else {
      bulk_wait_read();
    }
  }
  if (failed) break;
  ++tiles_done;
  if (tid == 0) *next_tile = nxt;
  fence_async_smem();  // this tile's shared-memory writes before the next tile's TMA loads
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // streamed schedule: the tile (stores, and gl by plain stores) is published to the walk,
  // a gpu-scope release after the CTA barrier
  if (a.tile_ready && tid == 0) st_release_gpu(a.tile_ready + tile, 1);
  tile = *next_tile;
  }  // tiles
  if (failed && tid == 0) {
    atomicExch(a.seq.status, kDevWaitTimeout);
    // copies and products in flight finish before the CTA releases its memory
    const uint32_t par = tiles_done & 1;
    if (!in_done) mbar_wait(bar_in, par, 400000000LL);
    if (!v_done) mbar_wait(bar_v, par, 400000000LL);
    for (int m = mma_done; m < mma_issued; ++m) mbar_wait(bar_mma, m & 1, 400000000LL);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tb, L_::COLS);
  }
  // streamed schedule: this grid runs as the walk kernel's dependent; it completes only
  // after the walk does, so later work on the stream still sees both finished
  if (a.tile_ready) griddep_wait();
}

// ------------------------------------------------------------------ walk over chunks
// One kernel walks every segment: per (sequence, head) pair, CTA 0 walks segments 0 and 1
// with outputs, and CTA r >= 1 walks segment r's summary, combines its start state and
// then walks segment r + 1 with outputs (the kernel itself is at the end of this part).
// Each CTA is warp-specialized:
//   warps 0..15 conversion: warps w, w + 4, w + 8, w + 12 share the tensor-memory lanes
//               32 (w % 4)..+31 (state columns j) and split their columns four ways;
//               warps 0..7 own K half 0 of the products' operands, warps 8..15 K half 1.
//               They rescale the fp32 state, add U0 and pack U^T and S^T into bf16 MMA
//               operands kept in tensor memory, and write the outputs;
//   warp 16     issues the MMAs (one thread);
//   warp 17     streams each chunk's workspace tiles into three stages by TMA (one thread).
// Hand-offs are mbarriers: full/empty per stage, m1/m2 (MMA groups done), and per K half
// s_ready/y_ready (that half of the bf16 S^T or U^T operand is in tensor memory), so the
// first half of a product starts while the second half is still being packed.
constexpr int kWalkConvThreads = 512, kWalkThreads = 576;
constexpr int kWalkMmaWarp = 16, kWalkLoadWarp = 17;
constexpr int kConvBar = 1;   // named barrier of all the conversion warps
constexpr int kHalfBar0 = 2;  // named barriers of the two K halves' warps: 2, 3
template <bool PC>
struct WalkSm {
  static constexpr int NB = PC ? 1 : 2;  // 128-column state blocks: [S] or [M | L]
  // One input stage of 128-byte-swizzled tiles as TMA lands them (rows of 64 elements):
  //   output walk, even stage: WQ = [-W^T | Q~^T] (128 rows each), PK = [P (64 rows) | Kb^T]
  //   output walk, odd stage:  WQ = [Q~^T | -W^T],                  PK = [Kb^T | P]
  //   summary walk: WQ = -W^T, PK = Kb^T.
  // WQ is MMA-1's B operand, MN-major (rows = the state row i, 64 tokens each; the two
  // 64-token groups 16 KB apart); PK is MMA-2's, K-major (rows = output columns, 64
  // tokens each). The order follows the tensor-memory order of the accumulators.
  static constexpr uint32_t WQ = 0;
  static constexpr uint32_t U0 = PC ? K32 : K16;
  static constexpr uint32_t PK = U0 + K16;
  static constexpr uint32_t STAGE = PK + (PC ? K16 + K8 : K16);
  static constexpr int NSTAGE = 3;  // chunk n in stage n % 3: two chunks' loads in flight
  static constexpr uint32_t GL = NSTAGE * STAGE;  // float[3][128]: each stage's gl, own barrier
  static constexpr uint32_t END = GL + NSTAGE * 512;
  // Tensor-memory columns. Output walk, by chunk parity p: p = 0: [U | O] at 0..127,
  // S at 128..255 (so MMA-2's accumulator [O | S] is 64..255); p = 1: S at 128..255,
  // [O | U] at 256..383 (MMA-2's [S | O] is 128..319). Summary walk: S per block at
  // 128 b, U per block at 256 + 64 b. The bf16 S^T operand (64 columns of pairs) per
  // block at 384 + 64 b; the bf16 U^T operand is packed in place over U: K step k (16
  // columns of U) is packed into the first 8 of them, at U + uk(k).
  __device__ static constexpr uint32_t st(int b) { return PC ? 128 : 128 * b; }
  __device__ static constexpr uint32_t uc(int b, int p) { return PC ? (p ? 320 : 0) : 256 + 64 * b; }
  __device__ static constexpr uint32_t yo(int p) { return p ? 256 : 64; }
  __device__ static constexpr uint32_t sbf(int b) { return 384 + 64 * b; }
  __device__ static constexpr uint32_t uk(int k) { return 16 * k; }
};
// mbarriers of one walk: full, empty and gl per stage; m1, m2; s_ready and y_ready per K
// half (then a spare one that nothing arrives at, for the test-only stuck first wait)
constexpr int kWalkBars = 3 * WalkSm<true>::NSTAGE + 6;
// Shared memory of the walk kernel: the output walk's stages and gl (the summary walk's
// smaller ones overlap them); the combine's M operand tiles, inside the output walk's
// third stage, which is not loaded before the combine's products have read them; one
// mbarrier set per walk and the combine's; the tensor-memory address.
struct WalkKSm {
  static constexpr uint32_t MT = 146 * 1024;           // M: bf16 hi tile | lo tile (2 x 32 KB)
  static constexpr uint32_t BARS = WalkSm<true>::END;  // two sets of 16, then the combine's
  static constexpr uint32_t TPTR = BARS + 2 * 16 * 8 + 16;
  static constexpr uint32_t BYTES = TPTR + 16;
  static constexpr uint32_t COLS = 512;                // tensor memory, allocated once
};
static_assert(kWalkBars + 1 <= 16, "walk barrier set");
static_assert(WalkKSm::MT % 1024 == 0 && WalkKSm::MT >= WalkSm<false>::END &&
                  WalkKSm::MT >= 2 * WalkSm<true>::STAGE && WalkKSm::MT + 2 * K32 <= WalkSm<true>::GL,
              "M tiles: past the summary walk's buffers and the output walk's first two stages");
static_assert(WalkKSm::BYTES + 1024 <= 232448, "walk shared memory");

// Segment `seg` of the sequence [t0, t1), head h: its tokens [c_begin, c_end) and the
// workspace tile of its first chunk (chunk n of the segment: tile0 + n H).
struct Seg {
  int64_t t0, len, off, c_begin, c_end, tile0;
  int n_chunks, h;
};
__device__ __forceinline__ Seg seg_geom(const WalkArgs& a, int s, int h, int64_t t0, int64_t t1,
                                        int seg) {
  Seg g;
  g.t0 = t0;
  g.len = t1 - t0;
  g.h = h;
  g.off = seg_offset(seg, a.first_tokens, a.seg_tokens, a.seg_dec);
  g.c_begin = t0 + g.off;
  const int64_t c_next = t0 + seg_offset(seg + 1, a.first_tokens, a.seg_tokens, a.seg_dec);
  g.c_end = c_next < t1 ? c_next : t1;
  g.n_chunks = g.c_end > g.c_begin ? static_cast<int>((g.c_end - g.c_begin + C - 1) / C) : 0;
  g.tile0 = (slot_base(t0, s) + g.off / C) * a.H + h;
  return g;
}

// The loads of chunk n of a walk (barrier set `bars`) into stage n % 3, which the caller
// knows to be free: gl first, on its own barrier (the conversion warps need only it to
// rescale), then the tiles.
template <bool PC>
__device__ __forceinline__ void issue_chunk(const WalkArgs& a, unsigned char* sm, uint64_t* bars,
                                            int64_t tile0, int n) {
  using L_ = WalkSm<PC>;
  constexpr int NS = L_::NSTAGE;
  const int st = n & 1, sg = n % NS;  // layout parity, stage
  uint64_t* const full = bars + sg;
  uint64_t* const glb = bars + 2 * NS + sg;
  unsigned char* dst = sm + sg * L_::STAGE;
  const int64_t tile = tile0 + static_cast<int64_t>(n) * a.H;
  const int y = static_cast<int>(tile * D);  // row of the [tiles * 128][64] arrays
  mbar_arrive_expect_tx(glb, 512);
  bulk_load(reinterpret_cast<float*>(sm + L_::GL) + sg * D, a.gl + tile * D, 512, glb);
  mbar_arrive_expect_tx(full, L_::STAGE);
  if (PC) {
    // even stages: [-W^T | Q~^T], [P | Kb^T]; odd stages: [Q~^T | -W^T], [Kb^T | P]
    tma_load_2d(dst + L_::WQ + st * K16, &a.tm_wt, full, 0, y);
    tma_load_2d(dst + L_::WQ + (st ^ 1) * K16, &a.tm_qt, full, 0, y);
    tma_load_2d(dst + L_::PK + (st ? 0 : K8), &a.tm_kbt, full, 0, y);
    tma_load_2d(dst + L_::PK + (st ? K16 : 0), &a.tm_p, full, 0, static_cast<int>(tile * C));
  } else {
    tma_load_2d(dst + L_::WQ, &a.tm_wt, full, 0, y);
    tma_load_2d(dst + L_::PK, &a.tm_kbt, full, 0, y);
  }
  tma_load_2d(dst + L_::U0, &a.tm_u0, full, 0, y);
}

// One walk over segment `seg` (geometry g) of the (sequence, head) pair with the barrier
// set `bars`. The output walk (PC) starts from the segment's start state (already in
// tensor memory when `from_tmem`, else the initial state or zero), writes the outputs,
// the final state when `last` and its end state, as the next segment's start, when
// `put_next`. The summary walk leaves M as the combine's bf16 hi/lo operand tiles in
// shared memory and L in tensor memory (columns 128..255). The caller has issued the
// loads of the first `pre` chunks. Ends with a CTA barrier; returns false (in every
// thread) when a wait ran out.
template <bool PC, bool SNAP>
__device__ __forceinline__ bool walk_segment(const WalkArgs& a, unsigned char* sm, uint32_t tb,
                                             uint64_t* bars, const Seg& g, int pair, int seg,
                                             bool from_tmem, int pre, bool last, bool put_next) {
  using L_ = WalkSm<PC>;
  constexpr int NB = L_::NB;
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = g.h;
  const int64_t t0 = g.t0, len = g.len, off = g.off, c_begin = g.c_begin, c_end = g.c_end;
  const int n_chunks = g.n_chunks;
  const int64_t tile0 = g.tile0;
  bool good = true;  // this thread's waits all completed

  float* gls = reinterpret_cast<float*>(sm + L_::GL);
  constexpr int NS = L_::NSTAGE;
  uint64_t* bar_full = bars;        // per stage: the tiles have landed
  uint64_t* bar_empty = bars + NS;  // per stage: the products have read it
  uint64_t* bar_gl = bars + 2 * NS; // per stage: the stage's gl has landed
  uint64_t* bar_m1 = bars + 3 * NS;
  uint64_t* bar_m2 = bars + 3 * NS + 1;
  uint64_t* bar_sready = bars + 3 * NS + 2;  // two column halves
  uint64_t* bar_yready = bars + 3 * NS + 4;  // two column halves
  tc_fence_after();  // after the caller's barrier: tensor memory as the previous step left it

  if (warp == kWalkLoadWarp) {
    // ============================================================ stage loads
    if (lane == 0 && n_chunks > 0) {
      tma_prefetch_desc(&a.tm_wt);
      tma_prefetch_desc(&a.tm_u0);
      tma_prefetch_desc(&a.tm_kbt);
      if (PC) {
        tma_prefetch_desc(&a.tm_qt);
        tma_prefetch_desc(&a.tm_p);
      }
      int issued = pre;
      bool ok = true;
      for (int n = pre; n < n_chunks; ++n) {
        const int sg = n % NS;
        if (n >= NS && !(ok = mbar_wait(bar_empty + sg, ((n - NS) / NS) & 1))) break;
        if (a.tile_ready) {
          // streamed schedule: the intra-chunk kernel, running beside this one, publishes
          // each tile once its stores are complete
          if (!(ok = flag_wait(a.tile_ready + tile0 + static_cast<int64_t>(n) * a.H))) break;
          fence_proxy_async_all();
        }
        issue_chunk<PC>(a, sm, bars, tile0, n);
        ++issued;
      }
      if (!ok) {
        atomicExch(a.seq.status, kDevWaitTimeout);
        good = false;
      }
      // the copies in flight land before the CTA can exit
      for (int n = issued >= NS ? issued - NS : 0; n < issued; ++n) {
        mbar_wait(bar_gl + n % NS, (n / NS) & 1, 400000000LL);
        mbar_wait(bar_full + n % NS, (n / NS) & 1, 400000000LL);
      }
    }
  } else if (warp == kWalkMmaWarp) {
    // ============================================================ MMA issue
    if (lane == 0) {
      int m_issued = 0;
      bool ok = true;
      for (int n = 0; n < n_chunks && ok; ++n) {
        const int st = n & 1, sg = n % NS;  // layout parity, stage
        const uint32_t stg = sb + sg * L_::STAGE;
        if (!(ok = mbar_wait(bar_full + sg, (n / NS) & 1))) break;
        // MMA-1: U^T = S^T (-W)^T and (output walk) (Q~ S)^T = S^T Q~^T, K = the 128 state
        // rows in two halves, each started once its half of S^T is packed; B MN-major: 16
        // rows of the stage tiles per K step. The output walk takes both in one N = 128
        // product (B = the stage's two 64-token tiles, 16 KB apart): an M = 128, K = 16
        // tcgen05.mma costs about the same for N = 64 and N = 128, so one product per K step
        // is half the tensor-pipe time of two.
        const uint32_t i1 = idesc_bf16(128, PC ? 128 : 64, 0, 1);
        const uint32_t d1 = PC ? (st ? L_::yo(1) : L_::uc(0, 0)) : 0;  // [U | O] or [O | U]
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (!(ok = mbar_wait(bar_sready + half, n & 1))) break;
          tc_fence_after();
#pragma unroll
          for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const int k = 4 * half + kk;
              umma_bf16_tmem_a(tb + (PC ? d1 : L_::uc(b, st)), tb + L_::sbf(b) + 8 * k,
                               sdesc_sw128(stg + L_::WQ + k * 2048, K16, 1024), i1, k > 0);
            }
        }
        if (!ok) break;
        umma_commit(bar_m1);
        ++m_issued;
        // MMA-2: output walk: [O^T | S^T] (or [S^T | O^T]) += U^T [P^T | Kb] in one N = 192
        // product; summary walk: S^T += U^T Kb per block (B operands K-major: the stage's
        // rows of P and Kb^T, 16 tokens = 32 bytes per K step)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (!(ok = mbar_wait(bar_yready + half, n & 1))) break;
          tc_fence_after();
          if (PC) {
            const uint32_t i2 = idesc_bf16(128, 192, 0, 0);
            const uint32_t d2 = st ? L_::st(0) : L_::yo(0);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              const int k = 2 * half + kk;
              umma_bf16_tmem_a(tb + d2, tb + L_::uc(0, st) + L_::uk(k),
                               sdesc_sw128(stg + L_::PK + k * 32, 16, 1024), i2, 1);
            }
          } else {
            const uint32_t i2 = idesc_bf16(128, 128, 0, 0);
#pragma unroll
            for (int b = 0; b < NB; ++b)
#pragma unroll
              for (int kk = 0; kk < 2; ++kk) {
                const int k = 2 * half + kk;
                umma_bf16_tmem_a(tb + L_::st(b), tb + L_::uc(b, 0) + L_::uk(k),
                                 sdesc_sw128(stg + L_::PK + k * 32, 16, 1024), i2, 1);
              }
          }
        }
        if (!ok) break;
        umma_commit(bar_m2);
        umma_commit(bar_empty + sg);
        ++m_issued;
      }
      if (!ok) {
        atomicExch(a.seq.status, kDevWaitTimeout);
        good = false;
        // every product issued so far (committed or not) finishes before tensor memory
        // is released: one more commit on m1, whose phase count is (m_issued + 1) / 2
        umma_commit(bar_m1);
        mbar_wait(bar_m1, ((m_issued + 1) / 2) & 1, 400000000LL);
      }
    }
  } else {
    // ============================================================ conversion warps
    // Warp w holds tensor-memory lanes 32 (w % 4) .. + 31 (state columns j) and part
    // pt = w / 4 of the columns: state rows i = 32 pt .. + 31, U^T and O^T columns (the
    // chunk's tokens) 16 pt .. + 15. Warps 0..7 (parts 0, 1) own K half 0 of both MMA
    // operands (state rows 0..63, tokens 0..31), warps 8..15 K half 1; each half has its
    // own named barrier and releases its half of each product as soon as it is packed.
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int row = (warp & 3) * 32 + lane;  // tensor-memory lane = state column j
    const int pt = warp >> 2;                // column part
    const int kh = pt >> 1;                  // the K half this warp's columns belong to
    const int half_bar = kHalfBar0 + kh;     // named barrier of this half's 256 threads
    const bool half_lead = (warp & 7) == 0 && lane == 0;
    // S <- Diag(gl) S on this thread's 32 fp32 state rows of block b (held in v), written
    // back to tensor memory: the decay of the chunk about to be walked. Not waited for
    // here: the next U^T pack's store wait covers it, before MMA-2 accumulates onto it.
    auto rescale = [&](int b, int sg, uint32_t (&v)[32]) {
      const float* gl = gls + sg * D + 32 * pt;
#pragma unroll
      for (int t4 = 0; t4 < 8; ++t4) {
        const float4 g = *reinterpret_cast<const float4*>(gl + 4 * t4);
        const float2 a0 = f32x2_split(mul_f32x2(f32x2(g.x, g.y),
                                                f32x2(__uint_as_float(v[4 * t4]), __uint_as_float(v[4 * t4 + 1]))));
        const float2 a1 = f32x2_split(mul_f32x2(f32x2(g.z, g.w),
                                                f32x2(__uint_as_float(v[4 * t4 + 2]), __uint_as_float(v[4 * t4 + 3]))));
        v[4 * t4 + 0] = __float_as_uint(a0.x);
        v[4 * t4 + 1] = __float_as_uint(a0.y);
        v[4 * t4 + 2] = __float_as_uint(a1.x);
        v[4 * t4 + 3] = __float_as_uint(a1.y);
      }
      tmem_st32(tb + lane_base + L_::st(b) + 32 * pt, v);
    };
    // this thread's 32 state rows of block b (in v) into the bf16 S^T operand
    auto pack_state = [&](int b, const uint32_t (&v)[32]) {
      uint32_t pk[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) pk[t] = pack_bf16(__uint_as_float(v[2 * t]), __uint_as_float(v[2 * t + 1]));
      tmem_st16(tb + lane_base + L_::sbf(b) + 16 * pt, pk);
    };
    bool failed = false;
    // U0^T[j][r] of the next chunk for this thread's tokens r = 16 pt .. + 15 (16-byte
    // chunks 2 pt, 2 pt + 1 of row j of the swizzled [128 j][64 r] tile of stage sg),
    // read as soon as the stage has landed, a chunk before the U^T pack that adds it
    float u0v[16];
    auto load_u0 = [&](int sg) {
      const unsigned char* u0r = sm + sg * L_::STAGE + L_::U0;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const uint4 w4 = *reinterpret_cast<const uint4*>(u0r + sw128_chunk(row, 2 * pt + q, 0));
        const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack_bf16(w[e]);
          u0v[8 * q + 2 * e] = f.x;
          u0v[8 * q + 2 * e + 1] = f.y;
        }
      }
    };
    // initial state: fp32 into tensor memory (unless it is there already), bf16 copy as
    // the MMA operand; then the first chunk's decay on the fp32 copy
    {
      const float* src = (PC && a.s0) ? a.s0 + static_cast<int64_t>(pair) * D * D : nullptr;
      uint32_t v[32];  // the last block's values (the only one in the output walk)
#pragma unroll 1
      for (int b = 0; b < NB; ++b) {
        if (PC && from_tmem) {
          tmem_ld32(tb + lane_base + L_::st(b) + 32 * pt, v);
          tmem_ld_wait(v);
        } else {
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const int c = 32 * pt + t;
            float x;
            if (PC) x = src ? src[static_cast<int64_t>(c) * D + row] : 0.f;
            else x = (b == 0 && c == row) ? 1.f : 0.f;
            v[t] = __float_as_uint(x);
          }
        }
        pack_state(b, v);
        if (NB > 1 || (n_chunks == 0 && !from_tmem))  // the unscaled fp32 state (reloaded below / final)
          tmem_st32(tb + lane_base + L_::st(b) + 32 * pt, v);
      }
      tmem_st_wait();
      tc_fence_before();
      group_sync(half_bar, 256);
      if (half_lead && n_chunks > 0) mbar_arrive(bar_sready + kh);
      if (n_chunks > 0) {
        const bool ok = mbar_wait(KDA_FIRST_WAIT_STUCK ? bars + kWalkBars : bar_gl, 0, KDA_FIRST_WAIT_LIMIT) &&
                        mbar_wait(bar_full, 0);
        if (group_any(kConvBar, kWalkConvThreads, !ok)) {
          failed = true;
        } else {
          if (NB == 1) {
            rescale(0, 0, v);
          } else {
#pragma unroll 1
            for (int b = 0; b < NB; ++b) {
              tmem_ld32(tb + lane_base + L_::st(b) + 32 * pt, v);
              tmem_ld_wait(v);
              rescale(b, 0, v);
            }
          }
          load_u0(0);
        }
      }
    }

    // O of chunk n (tensor-memory buffer yo(n & 1)) straight to global memory: lane pairs
    // (j, j + 1) trade values so that each lane writes two adjacent columns of one token
    // (even lanes the tokens 16 pt + 2 t, odd lanes 16 pt + 2 t + 1); a sequence's ragged
    // last chunk stops at its length (rows past it belong to the next sequence)
    auto emit_out = [&](int n) {
      const int64_t c0 = c_begin + static_cast<int64_t>(n) * C;
      const int L = (c_end - c0) < C ? static_cast<int>(c_end - c0) : C;
      uint32_t v[16];
      tmem_ld16(tb + lane_base + L_::yo(n & 1) + 16 * pt, v);
      tmem_ld_wait(v);
      const int odd = lane & 1;
      const int64_t ostride = static_cast<int64_t>(a.H) * D;
      __nv_bfloat16* o = a.out + ((c0 + 16 * pt + odd) * a.H + h) * D + (row & ~1);
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const float2 xs = f32x2_split(mul_f32x2(f32x2(a.scale, a.scale),
                                                f32x2(__uint_as_float(v[2 * t]), __uint_as_float(v[2 * t + 1]))));
        const float x0 = xs.x, x1 = xs.y;
        const float recv = __shfl_xor_sync(0xffffffffu, odd ? x0 : x1, 1);
        const uint32_t pr = odd ? pack_bf16(recv, x1) : pack_bf16(x0, recv);
        if (16 * pt + 2 * t + odd < L) *reinterpret_cast<uint32_t*>(o + 2 * t * ostride) = pr;
      }
    };

    // The fp32 state after chunk n (this thread's 32 state rows of column `row`, in v)
    // when that chunk is full and closes a snapshot interval of the sequence
    auto store_snapshot = [&](int n, const uint32_t (&v)[32]) {
      const int64_t done = off / C + n + 1;  // chunks of the sequence walked so far
      if (done % a.snap_every != 0 || done * C > len) return;
      const int64_t idx = t0 / (static_cast<int64_t>(C) * a.snap_every) + done / a.snap_every - 1;
      float* dst = a.snap + (idx * a.H + h) * D * D + static_cast<int64_t>(32 * pt) * D + row;
#pragma unroll
      for (int t = 0; t < 32; ++t) dst[t * D] = __uint_as_float(v[t]);
    };

    // Per chunk n (stage n % 3 has landed): MMA-1(n) runs -> U^T (+ U0^T) packed ->
    // MMA-2(n) runs while the previous chunk's outputs are written -> S^T packed for
    // MMA-1(n + 1), then the fp32 state rescaled by the next chunk's decay.
    for (int n = 0; n < n_chunks && !failed; ++n) {
      const int st = n & 1;
      if (group_any(kConvBar, kWalkConvThreads, !mbar_wait(bar_m1, n & 1))) {
        failed = true;
        break;
      }
      tc_fence_after();
      // ---- U^T (+ U0^T) -> bf16 operand, packed in place: this thread's 16 columns are
      //      K step pt, packed into their first 8
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        uint32_t v[16], pk[8];
        const uint32_t col = L_::uc(b, st) + 16 * pt;
        tmem_ld16(tb + lane_base + col, v);
        tmem_ld_wait(v);
        const bool with_u0 = PC || b == 1;  // the M block of the summary walk has V = 0
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          uint64_t x = f32x2(__uint_as_float(v[2 * t]), __uint_as_float(v[2 * t + 1]));
          if (with_u0) x = add_f32x2(x, f32x2(u0v[2 * t], u0v[2 * t + 1]));
          pk[t] = pack_bf16x2(x);
        }
        tmem_st8(tb + lane_base + col, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      group_sync(half_bar, 256);
      if (half_lead) mbar_arrive(bar_yready + kh);
      // ---- while MMA-2(n) runs: the previous chunk's outputs
      if (PC && n > 0) emit_out(n - 1);
      // MMA-2(n) done; the next chunk's gl and tiles (issued two chunks ahead) have landed
      const bool more = n + 1 < n_chunks;
      const int sg1 = (n + 1) % NS;
      const uint32_t ph1 = ((n + 1) / NS) & 1;
      {
        bool ok = mbar_wait(bar_m2, n & 1);
        if (more) ok = ok && mbar_wait(bar_gl + sg1, ph1) && mbar_wait(bar_full + sg1, ph1);
        if (group_any(kConvBar, kWalkConvThreads, !ok)) {
          failed = true;
          break;
        }
      }
      tc_fence_after();
      // ---- bf16 S^T operand for MMA-1(n + 1) (each half released when packed), then the
      //      next chunk's decay on the fp32 state and its U0^T, while MMA-1(n + 1) runs
      uint32_t v[32];
#pragma unroll 1
      for (int b = 0; b < NB; ++b) {
        tmem_ld32(tb + lane_base + L_::st(b) + 32 * pt, v);
        tmem_ld_wait(v);
        pack_state(b, v);
      }
      tmem_st_wait();
      tc_fence_before();
      group_sync(half_bar, 256);
      if (half_lead && more) mbar_arrive(bar_sready + kh);
      if (PC && SNAP) store_snapshot(n, v);  // while MMA-1(n + 1) runs
      if (more) {
        if (NB == 1) {
          rescale(0, sg1, v);
        } else {
#pragma unroll 1
          for (int b = 0; b < NB; ++b) {
            tmem_ld32(tb + lane_base + L_::st(b) + 32 * pt, v);
            tmem_ld_wait(v);
            rescale(b, sg1, v);
          }
        }
        load_u0(sg1);
      }
    }
    if (PC && !failed && n_chunks > 0) {
      tc_fence_after();
      emit_out(n_chunks - 1);  // the last chunk's outputs
    }
    tmem_st_wait();  // a decay store left in flight by a wait that ran out
    if (failed) {
      if (tid == 0) atomicExch(a.seq.status, kDevWaitTimeout);
      good = false;
    } else if (!PC) {
      // ---- summary: M[i][j] (i = 32 pt + t, j = row) as the combine's B operand, already
      //      split: two 128x128 bf16 tiles hi = bf16(M), lo = bf16(M - hi), each two
      //      64-column atoms of 128-byte-swizzled rows i (K-major: row i holds M[i][:])
      uint32_t v[32];
      tmem_ld32(tb + lane_base + L_::st(0) + 32 * pt, v);
      tmem_ld_wait(v);
      unsigned char* mb = sm + WalkKSm::MT;
      const uint32_t cofs = (row >> 6) * K16 + (row & 7) * 2;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const float x = __uint_as_float(v[t]);
        const __nv_bfloat16 hi = __float2bfloat16_rn(x);
        const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
        const uint32_t o = cofs + sw128_chunk(32 * pt + t, (row & 63) >> 3, 0);
        *reinterpret_cast<__nv_bfloat16*>(mb + o) = hi;
        *reinterpret_cast<__nv_bfloat16*>(mb + K32 + o) = lo;
      }
      fence_async_smem();  // read by the tensor cores next
    } else if (last || put_next) {
      // ---- final state, or the next segment's start state (row-major [i][j], fp32)
      float* dst = last ? a.sT : a.sstart + static_cast<int64_t>(pair) * a.max_segs * D * D;
      if (dst != nullptr) {
        dst += last ? static_cast<int64_t>(pair) * D * D : static_cast<int64_t>(seg + 1) * D * D;
        uint32_t v[32];
        tmem_ld32(tb + lane_base + L_::st(0) + 32 * pt, v);
        tmem_ld_wait(v);
#pragma unroll
        for (int t = 0; t < 32; ++t) __stcg(dst + static_cast<int64_t>(32 * pt + t) * D + row, __uint_as_float(v[t]));
      }
    }
  }
  tc_fence_before();
  const bool bad = __syncthreads_or(!good);
  tc_fence_after();
  return !bad;
}

// ------------------------------------------------------------------ combine
// Start state of segment r + 1 from that of segment r, S_{r+1} = M_r S_r + L_r, by the CTA
// that has just walked segment r's summary. One 128x128x128 product on the tensor cores in
// the transposed frame, S_{r+1}^T = S_r^T M_r^T + L_r^T, at fp32 accuracy through a bf16
// split of both factors, x = hi + lo with hi = bf16(x), lo = bf16(x - hi):
//   S^T M^T ~= S_hi^T M_hi^T + S_hi^T M_lo^T + S_lo^T M_hi^T
// (the dropped lo x lo term is ~2^-16 of the product). L_r^T is the accumulator already:
// the summary walk's second state block, in the tensor-memory columns where the output
// walk keeps its state, so S_{r+1} stays there as the next output walk's start state. M_r
// is the B operand the summary walk left in shared memory; S_r^T, published by the CTA of
// segment r - 1, is split into the A operand.
struct CombTm {
  static constexpr uint32_t D = 128, AH = 256, AL = 320;
};
// The whole CTA calls it; `publish`: segment r + 2 has a summary walk, whose CTA waits for
// S_{r+1}. `prefetch()`, called by the load warp's thread, issues the next walk's first
// loads: before the wait when S_r is at least a hop away (r >= 2, flag not yet set), else
// at the end, once S_{r+1} is published: with the walks streaming from HBM an SM takes
// its 144 KB in ~4 us, and copies still landing slow every step of the combine down
// (S_1, for r = 1, is planned to arrive with the summary's end).
// Returns false (in every thread) when S_r never came or a wait ran out.
template <typename F>
__device__ __forceinline__ bool combine_step(const WalkArgs& a, unsigned char* sm, uint32_t tb,
                                             uint64_t* bar, int pair, int r, bool publish,
                                             F&& prefetch) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int* const flags = a.flags + static_cast<int64_t>(pair) * a.max_segs;
  float* const sst = a.sstart + static_cast<int64_t>(pair) * a.max_segs * D * D;
  const bool loader = tid == kWalkLoadWarp * 32;
  bool fetched = false;
  if (loader && r >= 2 && ld_acquire_gpu(flags + r) == 0) {
    prefetch();
    fetched = true;
  }
  const bool ok_in = tid != 0 || flag_wait(flags + r);
  if (__syncthreads_or(!ok_in)) {
    if (loader && !fetched) prefetch();  // the caller drains what it asked for
    return false;
  }
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const int row = (warp & 3) * 32 + lane;  // tensor-memory lane = state column j
  const int pt = warp >> 2;                // K part: state rows k = 32 pt .. + 31
  if (warp < kWalkMmaWarp) {
    // S_r^T[j][k] = S_r[k][j] -> hi/lo bf16 pairs, tensor-memory column k / 2 of each half
    // (read from L2: another SM wrote it)
    const float* src = sst + static_cast<int64_t>(r) * D * D + static_cast<int64_t>(32 * pt) * D + row;
    uint32_t hi[16], lo[16];
#pragma unroll
    for (int t = 0; t < 16; ++t)
      split_bf16(__ldcg(src + (2 * t) * D), __ldcg(src + (2 * t + 1) * D), hi[t], lo[t]);
    tmem_st16(tb + lane_base + CombTm::AH + 16 * pt, hi);
    tmem_st16(tb + lane_base + CombTm::AL + 16 * pt, lo);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  if (tid == kWalkMmaWarp * 32) {
    tc_fence_after();
    const uint32_t id = idesc_bf16(128, 128, 0, 0);
    const uint32_t mb = smem_u32(sm + WalkKSm::MT);
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
      const uint32_t ko = (k >> 2) * K16 + (k & 3) * 32;  // K step k: atom k / 4, 32 bytes each
      const uint64_t bh = sdesc_sw128(mb + ko, 16, 1024), bl = sdesc_sw128(mb + K32 + ko, 16, 1024);
      umma_bf16_tmem_a(tb + CombTm::D, tb + CombTm::AH + 8 * k, bh, id, 1);
      umma_bf16_tmem_a(tb + CombTm::D, tb + CombTm::AH + 8 * k, bl, id, 1);
      umma_bf16_tmem_a(tb + CombTm::D, tb + CombTm::AL + 8 * k, bh, id, 1);
    }
    umma_commit(bar);
  }
  if (cta_wait_failed(bar, 0)) {
    if (loader && !fetched) prefetch();  // the caller drains what it asked for
    // the products finish before tensor memory can be released
    if (tid == 0) mbar_wait(bar, 0, 400000000LL);
    return false;
  }
  tc_fence_after();
  if (publish) {
    if (warp < kWalkMmaWarp) {
      uint32_t v[32];
      tmem_ld32(tb + lane_base + CombTm::D + 32 * pt, v);
      tmem_ld_wait(v);
      float* dst = sst + static_cast<int64_t>(r + 1) * D * D + static_cast<int64_t>(32 * pt) * D + row;
#pragma unroll
      for (int t = 0; t < 32; ++t) __stcg(dst + t * D, __uint_as_float(v[t]));
    }
    // every thread's stores, then the flag by a gpu-scope release, which the CTA barrier
    // makes cumulative over the other threads' stores
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) st_release_gpu(flags + r + 1, 1);
  }
  if (loader && !fetched) prefetch();
  return true;
}

// ------------------------------------------------------------------ walk kernel
// CTA r of the `per` CTAs of a (sequence, head) pair:
//   r = 0:  the output walk of segment 0, whose end state S_1 it publishes (when segment 1
//           has a summary walk), then the output walk of segment 1 from S_1 in tensor memory;
//   r >= 1: the summary walk of segment r (in parallel with segment 0's walk), the
//           combine step S_{r+1} = M_r S_r + L_r as soon as CTA r - 1 has published S_r
//           (publishing S_{r+1} in turn), then the output walk of segment r + 1 from S_{r+1}
//           in tensor memory.
// The grid (pairs x per <= the SM count, one CTA per SM) is resident at once, which the
// hand-off waits rely on; each is bounded, and a CTA whose walk failed publishes "not
// coming" so that the later ones stop waiting. The first two chunks of a CTA's second
// walk are loaded while the combine waits. SNAP: the output walks also write
// chunk-boundary snapshots (a separate instance, so the plain walk carries no trace of
// them).
template <bool SNAP>
__global__ void __launch_bounds__(kWalkThreads, 1) kda_tc_walk(const __grid_constant__ WalkArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = align1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int per = a.max_segs > 2 ? a.max_segs - 1 : 1;
  const int r = blockIdx.x % per, pair = blockIdx.x / per;
  const int s = pair / a.H, h = pair % a.H;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + WalkKSm::BARS);  // first walk
  uint64_t* bars2 = bars + 16;                                         // second walk
  uint64_t* bar_comb = bars + 32;
  uint32_t* tptr = reinterpret_cast<uint32_t*>(sm + WalkKSm::TPTR);
  // tensor memory once for the CTA's lifetime (an allocation after the relinquish is not
  // allowed)
  if (warp == 0) {
    tmem_alloc(tptr, WalkKSm::COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i <= kWalkBars; ++i) {
      mbar_init(bars + i, 1);
      mbar_init(bars2 + i, 1);
    }
    mbar_init(bar_comb, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = *tptr;
  if (a.tile_ready) {
    // streamed schedule: the intra-chunk kernel runs as this grid's dependent, beside it;
    // let it be scheduled now (the tiles are waited for one by one)
    griddep_launch_dependents();
  } else {
    griddep_wait();  // the workspace tiles and the cleared flags come from the intra-chunk kernel
  }

  int64_t t0 = 0, t1 = 0;
  int nseg = 0;
  if (seq_bounds_tc(a.seq, s, t0, t1)) {
    nseg = seg_count(t1 - t0, a.first_tokens, a.seg_tokens, a.seg_dec, a.max_segs);
    if (t1 - t0 > a.max_len || nseg > a.max_segs) {  // the caller's max_seqlen bound was too small
      if (r == 0 && tid == 0) atomicExch(a.seq.status, kDevBadSeqlens);
      nseg = 0;
    }
  }
  int* const flags = a.flags + static_cast<int64_t>(pair) * a.max_segs;
  const bool loader = tid == kWalkLoadWarp * 32;
  if (nseg > 0 && r == 0) {
    const bool ok = walk_segment<true, SNAP>(a, sm, tb, bars, seg_geom(a, s, h, t0, t1, 0), pair, 0,
                                             false, 0, nseg == 1, nseg > 2);
    // after the walk's closing barrier, so the release covers S_1's stores by every thread
    if (nseg > 2 && tid == 0) st_release_gpu(flags + 1, ok ? 1 : 2);
    if (ok && nseg > 1) {
      const Seg g1 = seg_geom(a, s, h, t0, t1, 1);
      const int pre = g1.n_chunks < 2 ? g1.n_chunks : 2;
      if (loader)
        for (int n = 0; n < pre; ++n) issue_chunk<true>(a, sm, bars2, g1.tile0, n);
      walk_segment<true, SNAP>(a, sm, tb, bars2, g1, pair, 1, true, pre, nseg == 2, false);
    }
  } else if (nseg > 0 && r <= nseg - 2) {
    bool ok = walk_segment<false, false>(a, sm, tb, bars, seg_geom(a, s, h, t0, t1, r), pair, r,
                                         false, 0, false, false);
    const Seg g2 = seg_geom(a, s, h, t0, t1, r + 1);
    // the next walk's first two chunks into stages 0 and 1 (the summary walk is done with
    // them; the M tiles sit in stage 2), issued during the combine step
    const int pre = !ok ? 0 : g2.n_chunks < 2 ? g2.n_chunks : 2;
    const bool publish = r + 1 <= nseg - 2;
    if (ok)
      ok = combine_step(a, sm, tb, bar_comb, pair, r, publish, [&] {
        for (int n = 0; n < pre; ++n) issue_chunk<true>(a, sm, bars2, g2.tile0, n);
      });
    if (!ok && publish && tid == 0) st_release_gpu(flags + r + 1, 2);
    if (ok) {
      walk_segment<true, SNAP>(a, sm, tb, bars2, g2, pair, r + 1, true, pre, r + 1 == nseg - 1, false);
    } else if (loader) {
      // the loads issued for the walk that will not run land before the CTA exits
      for (int n = 0; n < pre; ++n) {
        mbar_wait(bars2 + 2 * WalkSm<true>::NSTAGE + n, 0, 400000000LL);
        mbar_wait(bars2 + n, 0, 400000000LL);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tb, WalkKSm::COLS);
  }
  griddep_launch_dependents();
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

// 2-D bf16 tensor map over `rows` rows of `cols` elements, `pitch` bytes apart,
// moved in boxes of `box_rows` rows x `box_cols`; with `swizzle` (64 columns) a box
// lands in the 128-byte-swizzled operand layout.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t pitch,
              bool swizzle, uint32_t box_cols = 64, uint32_t box_rows = 64) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(pitch)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t align_to(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

bool tc_path_applies(const kda_shape& s, int64_t T_total) {
  return s.dtype == KDA_BF16 && s.dk == D && s.dv == D && T_total > 0;
}

TcPlan tc_plan(int64_t T_total, int n_seqs, int H, int64_t max_len) {
  TcPlan p{};
  p.n_slots = (T_total + C - 1) / C + n_seqs;
  p.pairs = static_cast<int64_t>(n_seqs) * H;
  if (max_len < 1) max_len = 1;
  // Segments: the walk kernel runs one CTA per SM and a chunk costs about the same in
  // every CTA, so a sequence of Lc chunks is cut into segment 0 plus m later segments with
  // m = SMs / pairs, walked by m CTAs: CTA 0 walks segments 0 and 1 with outputs, CTA
  // r >= 1 the summary of segment r beside segment 0's walk, then (after the combine
  // steps of CTAs 1 .. r, one after another) segment r + 1 with outputs. Segment 0 is
  // 1.2 n chunks, as the summary walk's chunk step is ~1.2x the output walk's, so S_1 is
  // ready when the summaries are; segment j >= 1 is n - (j - 1) delta chunks, delta = 2
  // chunks (about one combine hop of output walk), so that the later segments, whose
  // output walks start a hop later each, finish together. delta drops to 1, then 0, where
  // it would take the last planned segment below max(4, n / 2) chunks.
  const int64_t Lc = (max_len + C - 1) / C;
  const int64_t m = p.pairs > 0 ? 148 / p.pairs : 1;
  p.seg_dec = 0;
  // Streamed schedule: one output walk per (sequence, head) from the start, beside the
  // intra-chunk kernel on the other SMs, each tile taken as soon as it is written (from L2).
  // Chosen when a model of the two schedules (per-tile and per-chunk costs measured on the
  // 8K x 32-head workload) favours it: the streamed time is the longer of one walk over the
  // longest sequence (~1.9 us a chunk) and the tiles on 2 x (SMs - pairs) CTA slots; the
  // segmented time is the tiles on all 296 slots, then the segmented walks.
  const double tiles_us = 12.6 * static_cast<double>(p.n_slots * H);
  const double walk_seg = (m >= 2 && Lc >= 16) ? 5.1 * static_cast<double>(Lc) / (static_cast<double>(m) + 1.26)
                                               : 1.9 * static_cast<double>(Lc);
  const double t_seg = tiles_us / 296.0 + walk_seg;
  double t_str = 1e300;
  if (p.pairs >= 1 && p.pairs <= 100) {
    const double intra = tiles_us / (2.0 * static_cast<double>(148 - p.pairs));
    t_str = (1.9 * static_cast<double>(Lc) > intra ? 1.9 * static_cast<double>(Lc) : intra) + 10.0;
  }
  p.streamed = t_str < 0.97 * t_seg;
  // KDA_PREFILL_SCHEDULE=segmented|streamed overrides the model (a tool that runs kernels one
  // at a time, a profiler say, needs the segmented one: the streamed walk waits for tiles a
  // kernel launched after it writes)
  if (const char* env = std::getenv("KDA_PREFILL_SCHEDULE")) {
    if (std::strcmp(env, "segmented") == 0) p.streamed = false;
    else if (std::strcmp(env, "streamed") == 0) p.streamed = p.pairs >= 1 && p.pairs <= 100;
  }
  if (p.streamed || m < 2 || Lc < 16) {
    p.first_tokens = p.seg_tokens = 1 << 30;  // one segment per sequence
    p.max_segs = 1;
  } else {
    int64_t n = 4, delta = 2;
    for (; delta >= 0; --delta) {
      // n = ceil((Lc + delta m (m - 1) / 2) / (1.2 + m)): the segments cover Lc chunks
      n = (5 * (Lc + delta * (m * (m - 1) / 2)) + 5 * m + 6 - 1) / (5 * m + 6);
      if (n < 4) n = 4;
      const int64_t lo = n / 2 > 4 ? (n + 1) / 2 : 4;
      if (n - (m - 1) * delta >= lo) break;
    }
    if (delta < 0) delta = 0;
    const int64_t n0 = (6 * n + 4) / 5;  // ceil(1.2 n)
    p.first_tokens = static_cast<int>(n0 * C);
    p.seg_tokens = static_cast<int>(n * C);
    p.seg_dec = static_cast<int>(delta * C);
    p.max_segs = seg_count(max_len, p.first_tokens, p.seg_tokens, p.seg_dec, static_cast<int>(m) + 1);
  }
  const size_t state = sizeof(float) * D * D;
  size_t off = kWorkspaceHeader;
  p.ready_off = off;  // per-tile ready flags of the streamed schedule
  off += align_to(sizeof(int) * static_cast<size_t>(p.n_slots) * static_cast<size_t>(H), 256);
  if (p.max_segs > 2)  // the start state of every segment and its hand-off flag
    off += (state + sizeof(int)) * static_cast<size_t>(p.pairs) * static_cast<size_t>(p.max_segs);
  p.tiles_off = align_to(off, 1024);
  p.ws_bytes = p.tiles_off + kTileBytes * static_cast<size_t>(p.n_slots) * static_cast<size_t>(H);
  return p;
}

cudaError_t launch_prefill_tc(const PrefillArgs& pa, cudaStream_t st) {
  const TcPlan plan = tc_plan(pa.T_total, pa.n_seqs, pa.H, pa.max_len);
  if (pa.ws_bytes < plan.ws_bytes) return cudaErrorInvalidValue;
  const int64_t tiles = plan.n_slots * pa.H;
  const SeqTable seq{pa.cu, pa.status, pa.T, pa.T_total, pa.n_seqs};
  // workspace: header | M, L, S_start (segmented walks only) | per-chunk tiles
  unsigned char* tp = pa.ws + plan.tiles_off;
  auto* wt = reinterpret_cast<__nv_bfloat16*>(tp);
  __nv_bfloat16* qt = wt + tiles * C * D;
  __nv_bfloat16* u0 = qt + tiles * C * D;
  __nv_bfloat16* kbt = u0 + tiles * C * D;
  __nv_bfloat16* pm = kbt + tiles * C * D;
  auto* gl = reinterpret_cast<float*>(pm + tiles * C * C);
  const uint64_t in_cols = static_cast<uint64_t>(pa.H) * D, in_pitch = in_cols * 2;
  const uint64_t rows_big = static_cast<uint64_t>(tiles) * D;  // [tiles * 128][64] arrays
  const uint64_t rows_p = static_cast<uint64_t>(tiles) * C;    // [tiles * 64][64]

  IntraArgs ia;
  memset(&ia, 0, sizeof ia);
  WalkArgs wa;
  memset(&wa, 0, sizeof wa);
  if (!make_map(&ia.tm_q, pa.q, in_cols, pa.T_total, in_pitch, false, D) ||
      !make_map(&ia.tm_k, pa.k, in_cols, pa.T_total, in_pitch, false, D) ||
      !make_map(&ia.tm_g, pa.g, in_cols, pa.T_total, in_pitch, false, D) ||
      !make_map(&ia.tm_v, pa.v, in_cols, pa.T_total, in_pitch, true) ||
      !make_map(&ia.tm_wt, wt, C, rows_big, C * 2, true, C, D) ||
      !make_map(&ia.tm_qt, qt, C, rows_big, C * 2, true, C, D) ||
      !make_map(&ia.tm_u0, u0, C, rows_big, C * 2, true, C, D) ||
      !make_map(&ia.tm_kbt, kbt, C, rows_big, C * 2, true, C, D) ||
      !make_map(&ia.tm_p, pm, C, rows_p, C * 2, true) ||

      !make_map(&wa.tm_wt, wt, C, rows_big, C * 2, true, C, D) ||
      !make_map(&wa.tm_qt, qt, C, rows_big, C * 2, true, C, D) ||
      !make_map(&wa.tm_u0, u0, C, rows_big, C * 2, true, C, D) ||
      !make_map(&wa.tm_kbt, kbt, C, rows_big, C * 2, true, C, D) ||
      !make_map(&wa.tm_p, pm, C, rows_p, C * 2, true))
    return cudaErrorInvalidValue;
  ia.seq = seq;
  ia.beta = static_cast<const __nv_bfloat16*>(pa.beta);
  ia.gl = gl;
  ia.queue = reinterpret_cast<int*>(pa.ws + kIntraQueueOffset);
  if (plan.streamed) {
    ia.tile_ready = reinterpret_cast<int*>(pa.ws + plan.ready_off);
    wa.tile_ready = ia.tile_ready;
  }
  ia.n_tiles = tiles;
  ia.H = pa.H;
  ia.lb = pa.lb;

  wa.seq = seq;
  wa.gl = gl;
  wa.out = static_cast<__nv_bfloat16*>(pa.out);
  wa.s0 = pa.s0;
  wa.sT = pa.sT;
  wa.snap = pa.snap;
  wa.snap_every = pa.snap_every;
  if (plan.max_segs > 2) {
    const size_t units = static_cast<size_t>(plan.pairs) * plan.max_segs;
    wa.sstart = reinterpret_cast<float*>(pa.ws + plan.ready_off +
                                         align_to(sizeof(int) * static_cast<size_t>(tiles), 256));
    wa.flags = reinterpret_cast<int*>(wa.sstart + units * D * D);
    ia.flags = wa.flags;
    ia.n_flags = static_cast<int>(units);
  }
  wa.H = pa.H;
  wa.first_tokens = plan.first_tokens;
  wa.max_len = pa.max_len;
  wa.seg_tokens = plan.seg_tokens;
  wa.seg_dec = plan.seg_dec;
  wa.max_segs = plan.max_segs;
  wa.scale = pa.scale;

  void (*intra)(IntraArgs) = pa.prologue == 0 ? kda_tc_intra<0>
                            : pa.prologue == 1 ? kda_tc_intra<1>
                            : pa.prologue == 2 ? kda_tc_intra<2>
                                               : kda_tc_intra<3>;
  // dynamic shared memory limits are per function and per device: set them every call
  cudaError_t e = cudaFuncSetAttribute(intra, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       IntraSm::BYTES + 1024);
  const bool snap = pa.snap != nullptr;
  void (*walk)(WalkArgs) = snap ? kda_tc_walk<true> : kda_tc_walk<false>;
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(walk, cudaFuncAttributeMaxDynamicSharedMemorySize, WalkKSm::BYTES + 1024);
  if (e != cudaSuccess) return e;

  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // a launch with programmatic stream serialization: it may be scheduled once every CTA of
  // the kernel before it on the stream has triggered (griddepcontrol.launch_dependents)
  auto launch_dep = [&](const void* fn, int64_t grid, int threads, uint32_t smem, void* arg) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {arg};
    return cudaLaunchKernelExC(&cfg, fn, args);
  };
  if (plan.streamed) {
    // The walk first, one CTA per (sequence, head) (pairs < SMs), then the intra-chunk
    // kernel as its dependent on the remaining SMs, two persistent CTAs per SM: the walk's
    // CTAs are all resident before it starts, so the two share the GPU; the walk waits for
    // each tile's ready flag (cleared here), the intra-chunk kernel never waits for the walk
    // until its own end.
    e = cudaMemsetAsync(ia.tile_ready, 0, sizeof(int) * static_cast<size_t>(tiles), st);
    if (e == cudaSuccess) {
      walk<<<static_cast<unsigned>(plan.pairs), kWalkThreads, WalkKSm::BYTES + 1024, st>>>(wa);
      e = cudaGetLastError();
    }
    const int64_t slots = 2 * (static_cast<int64_t>(sms) - plan.pairs);
    if (e == cudaSuccess)
      e = launch_dep(reinterpret_cast<const void*>(intra), tiles < slots ? tiles : slots,
                     kIntraThreads, IntraSm::BYTES + 1024, &ia);
  } else {
    // two resident CTAs per SM, taking tiles from the queue; then the walk kernel, whose
    // CTAs set up while the intra-chunk kernel drains and then wait for it
    const int64_t intra_grid = tiles < 2 * static_cast<int64_t>(sms) ? tiles : 2 * static_cast<int64_t>(sms);
    intra<<<static_cast<unsigned>(intra_grid), kIntraThreads, IntraSm::BYTES + 1024, st>>>(ia);
    e = cudaGetLastError();
    const int64_t per = plan.max_segs > 2 ? plan.max_segs - 1 : 1;
    if (e == cudaSuccess)
      e = launch_dep(reinterpret_cast<const void*>(walk), plan.pairs * per, kWalkThreads,
                     WalkKSm::BYTES + 1024, &wa);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace kda
