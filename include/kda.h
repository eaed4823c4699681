/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention library.
 *
 * Kimi Delta Attention (KDA) is a gated delta-rule linear attention with a
 * fixed-size state per head. Sources (web pages about the Kimi K3 report):
 *   - "Kimi K3 深度拆解" (chenxutan.com), section 4.2 "线性注意力与 Delta Rule":
 *     the delta-rule state update, the fixed [d_k, d_v] state, the per-token
 *     write strength beta in (0,1), q/k L2-normalised (by the caller, or by the
 *     optional prologue below), read-out from the updated state, and the
 *     chunk-parallel / inter-chunk-recurrent form.
 *   - "Kimi K3 技術報告：三個架構改動" (akiraxclaw.com), section "長度":
 *     channel-wise gating (each key channel has its own forget rate).
 *   - "3 分钟看懂 Kimi K3" (landx.limxdynamics.com), "第一条主线", Figure 3:
 *     the log decay is bounded below so every causal chunk is a dense matmul.
 *
 * Per head, with S in R^{d_k x d_v} (rows = key channels), each token t does
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp max(g_t, lb)) S_{t-1} + beta_t k_t v_t^T
 *     o_t = scale * S_t^T q_t
 * where g_t in R^{d_k} is the per-channel log decay and lb = g_lower_bound.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller. The library
 *     never frees or retains them and never allocates device memory per call
 *     (scratch is the caller's `workspace`).
 *   - Layouts are token-major and contiguous: q, k, g [tokens, H, d_k];
 *     v, out [tokens, H, d_v]; beta [tokens, H]; states [n, H, d_k, d_v] fp32
 *     row-major. Every tensor pointer must be 16-byte aligned.
 *   - q, k, v, g, beta and out share `dtype`; states are always fp32.
 *   - Work is enqueued on `stream`; no call synchronises the stream.
 *   - Argument errors are reported before anything is launched. A launch
 *     failure returns KDA_ERR_CUDA; the library does not clear sticky errors.
 *   - Malformed cu_seqlens contents (only visible on the device) are not
 *     trapped: the kernels skip the bad sequences and record KDA_ERR_DEVICE in
 *     the workspace, readable with kda_workspace_status().
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kda_stream_t; /* same type as cudaStream_t */

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad shape, workspace too small */
    KDA_ERR_UNSUPPORTED = 2, /* valid but not implemented: head dims, chunk, lb*chunk range */
    KDA_ERR_CUDA = 3,        /* a CUDA launch or query failed */
    KDA_ERR_DEVICE = 4       /* a device-side check failed (see kda_workspace_status) */
} kda_status;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

typedef struct {
    int64_t T;          /* tokens per sequence when cu_seqlens == NULL (then B sequences
                           of T tokens each); total packed tokens when cu_seqlens != NULL */
    int32_t B;          /* batch; must be 1 when cu_seqlens != NULL */
    int32_t H;          /* heads */
    int32_t dk, dv;     /* head dims: each 64 or 128 */
    int32_t n_seqs;     /* with cu_seqlens: number of sequences (len(cu_seqlens) - 1, >= 1);
                           without cu_seqlens: must be 0 (the library uses B) */
    int64_t max_seqlen; /* with cu_seqlens: an upper bound on every sequence's length
                           (0 = unknown, taken as T). It sizes the workspace and the
                           schedule; a sequence longer than it is skipped and reported
                           as KDA_ERR_DEVICE. Ignored without cu_seqlens. */
    kda_dtype dtype;    /* dtype of q, k, v, g, beta and out */
    float scale;        /* read-out scale; 0 selects 1/sqrt(dk) */
    float g_lower_bound;/* lb: g is clamped to >= lb inside the library. Must satisfy
                           lb < 0 and lb * chunk >= -80 so exp(-cumsum) stays finite */
    int32_t chunk;      /* chunk length; 64 is the supported value */
    int32_t prologue;   /* 0, or KDA_PROLOGUE_* flags: inputs are raw and the library
                           applies the prologue inside its kernels (see below) */
} kda_shape;

/*
 * Optional input prologue, fused into every entry point's kernels (prefill, snapshots,
 * no-alloc prefill, decode, backward). With 0 the inputs are used as given.
 *  KDA_PROLOGUE_QK_L2NORM   q and k are raw: each (token, head) row is divided by
 *                           max(||row||_2, 1e-12) in fp32 before use ("Kimi K3 深度拆解",
 *                           section 4.2: the delta rule takes L2-normalised q and k).
 *  KDA_PROLOGUE_GATE_SIGMOID g holds gate pre-activations a; the log decay is
 *                           lb * sigmoid(a), inside (lb, 0), so the lower bound holds by
 *                           construction ("3 分钟看懂 Kimi K3", 第一条主线 / Figure 3: the
 *                           log decay is bounded below). The clamp max(., lb) still applies.
 * Other bits are rejected with KDA_ERR_INVALID_ARG.
 */
#define KDA_PROLOGUE_QK_L2NORM 1
#define KDA_PROLOGUE_GATE_SIGMOID 2

/*
 * Bytes of device scratch kda_chunk_fwd needs for this shape (a pure function
 * of the shape fields). Returns 0 for an invalid shape.
 */
size_t kda_chunk_fwd_workspace_size(const kda_shape *shape);

/*
 * Chunked prefill ("Kimi K3 深度拆解", section 4.2: chunk-parallel with an
 * inter-chunk recurrence; "3 分钟看懂 Kimi K3", Figure 3: bounded log decay).
 *
 *  q, k, g      [B*T, H, dk] (or [T, H, dk] packed)     dtype
 *  v            [B*T, H, dv]                            dtype
 *  beta         [B*T, H]                                dtype
 *  initial_state[n, H, dk, dv] fp32, or NULL for zeros (n = B, or n_seqs)
 *  cu_seqlens   int32 [n_seqs + 1] or NULL: 0 = c_0 <= c_1 <= ... <= c_n = T.
 *               Sequences may be empty (their final state is their initial state).
 *  out          [B*T, H, dv] dtype (written)
 *  final_state  [n, H, dk, dv] fp32, or NULL to skip. May alias initial_state
 *               (resume in place).
 *  workspace    device scratch of >= kda_chunk_fwd_workspace_size(shape) bytes,
 *               256-byte aligned, used only for the duration of the enqueued work.
 *               Calls that share a workspace must be ordered on one stream.
 *
 * Schedule (bf16 with dk = dv = 128): an intra-chunk kernel and a walk kernel. Where a
 * built-in model of the two schedules favours it, the walk runs first, one CTA per
 * (sequence, head), and the intra-chunk kernel runs beside it as its programmatic
 * dependent on the other SMs; the walk takes each chunk's tiles as soon as they are
 * written (a bounded wait on a per-tile flag). Otherwise the walk runs after it, long
 * sequences split into segments walked in parallel. KDA_PREFILL_SCHEDULE=segmented or
 * =streamed in the environment overrides the model; a tool that runs kernels one at a time
 * (a profiler) needs `segmented`. The workspace size depends on the schedule: keep the
 * variable unchanged between kda_chunk_fwd_workspace_size and the call.
 */
kda_status kda_chunk_fwd(const void *q, const void *k, const void *v, const void *g,
                         const void *beta, const float *initial_state,
                         const int32_t *cu_seqlens, void *out, float *final_state,
                         const kda_shape *shape, void *workspace, size_t workspace_bytes,
                         kda_stream_t stream);

/*
 * kda_chunk_fwd that also keeps the state at regular chunk boundaries of each
 * sequence, for a prefix cache: a later request that shares the first m
 * intervals of a sequence resumes from snapshot m by passing it as
 * initial_state, instead of recomputing the prefix ("3 分钟看懂 Kimi K3",
 * 第一条主线: KDA state and prefix-cache scheduling for long requests; the state
 * after any prefix is the recurrence's own S_t, "Kimi K3 深度拆解", section 4.2).
 *
 *  snapshot_chunks  k >= 1: one snapshot every k chunks (k * chunk tokens).
 *  snapshots        fp32 [n_snapshots, H, dk, dv], device, written. For sequence n,
 *                   whose first token is c_n in the packed layout (c_n = n * T
 *                   without cu_seqlens), and for m = 1 .. floor(len_n / (k * chunk)),
 *                   the state after the sequence's first m * k * chunk tokens (seeded
 *                   by its initial state) is written at index
 *                   floor(c_n / (k * chunk)) + m - 1. The sequences' index ranges never
 *                   overlap; an index no sequence reaches is left as it was. Must not
 *                   overlap any other argument.
 *  n_snapshots      capacity of `snapshots`; must be >= kda_snapshot_count(shape, k).
 *                   `snapshots` may be NULL only when that count is 0.
 * Every other argument, every result and the workspace size are those of
 * kda_chunk_fwd; out and final_state hold exactly the values kda_chunk_fwd writes.
 * Returns KDA_ERR_INVALID_ARG for snapshot_chunks < 1, a short or misaligned
 * `snapshots`, or any argument kda_chunk_fwd rejects.
 */
kda_status kda_chunk_fwd_snapshots(const void *q, const void *k, const void *v, const void *g,
                                   const void *beta, const float *initial_state,
                                   const int32_t *cu_seqlens, void *out, float *final_state,
                                   int32_t snapshot_chunks, float *snapshots,
                                   int64_t n_snapshots, const kda_shape *shape,
                                   void *workspace, size_t workspace_bytes,
                                   kda_stream_t stream);

/*
 * Snapshot slots kda_chunk_fwd_snapshots needs: floor(T_total / (snapshot_chunks *
 * chunk)), T_total = B * T without cu_seqlens, T with them. Returns -1 for an
 * invalid shape or snapshot_chunks < 1.
 */
int64_t kda_snapshot_count(const kda_shape *shape, int32_t snapshot_chunks);

/*
 * Bytes of device scratch kda_chunk_bwd needs for this shape (a pure function of the
 * shape fields). Returns 0 for an invalid shape.
 */
size_t kda_chunk_bwd_workspace_size(const kda_shape *shape);

/*
 * Gradients of kda_chunk_fwd for training: given dL/dout and dL/dfinal_state of a scalar
 * loss L, writes dL/dq, dL/dk, dL/dv, dL/dg, dL/dbeta and dL/dinitial_state. It is the
 * reverse of the chunk-parallel form with its inter-chunk recurrence ("Kimi K3 深度拆解",
 * section 4.2), walked from the last chunk back; the state at every chunk start comes
 * from a forward pass with per-chunk snapshots that this call runs first.
 *
 *  q, k, v, g, beta, initial_state, cu_seqlens, shape: as in kda_chunk_fwd (the same
 *               forward inputs). With shape->prologue set the inputs are raw and dq, dk,
 *               dg are the gradients of the raw q, k and gate pre-activations.
 *  d_out        [B*T, H, dv] dtype, or NULL for zeros
 *  d_final_state[n, H, dk, dv] fp32, or NULL for zeros
 *  dq, dk, dg   [B*T, H, dk] dtype (written)     dv [B*T, H, dv] dtype (written)
 *  dbeta        [B*T, H] dtype (written)
 *  d_initial_state [n, H, dk, dv] fp32 (written), or NULL to skip
 *  workspace    >= kda_chunk_bwd_workspace_size(shape) bytes, 256-byte aligned.
 * g enters through max(g, lb): where g < lb its gradient is 0 (at g == lb it passes).
 * Computed in fp32 on CUDA cores (one CTA per sequence, head and 32- or 16-column slice of dv);
 * dq, dk, dg and dbeta sum the slices' contributions with fp32 atomics, so their last
 * bits may differ between runs. Errors as in kda_chunk_fwd; when its forward pass skips a
 * sequence (malformed cu_seqlens, or longer than max_seqlen) KDA_ERR_DEVICE is recorded and
 * that sequence's gradients are unspecified.
 */
kda_status kda_chunk_bwd(const void *q, const void *k, const void *v, const void *g,
                         const void *beta, const float *initial_state,
                         const int32_t *cu_seqlens, const void *d_out,
                         const float *d_final_state, void *dq, void *dk, void *dv, void *dg,
                         void *dbeta, float *d_initial_state, const kda_shape *shape,
                         void *workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_chunk_fwd without a workspace argument, for callers that cannot call
 * cudaMalloc: code running while a CUDA graph is being captured (allocation is
 * not capturable), plugin hosts that hand a library no scratch buffer, and
 * serving loops where an allocation would synchronise the device. The pages
 * describe no such entry point; it exists only for these callers.
 *
 * Arguments and results are those of kda_chunk_fwd; the caller still passes
 * every input and output. The scratch comes from one fixed device array of
 * KDA_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits. It allocates nothing.
 *  - Returns KDA_ERR_UNSUPPORTED when kda_chunk_fwd_workspace_size(shape)
 *    exceeds KDA_NOALLOC_SCRATCH_BYTES (use kda_chunk_fwd with a workspace).
 *  - The first call on a device looks up that device's copy of the array
 *    (cudaGetSymbolAddress, once per device, for the current device); make
 *    that first call before any stream capture. The current device must be the
 *    device of `stream`.
 *  - All calls on a device share the array and it keeps the previous call's
 *    contents (the prefill clears what must start at zero). Calls whose work
 *    overlaps on the GPU, e.g. on unordered streams, race on the array.
 *  - The array's address is looked up per CUDA context: after a device reset, or
 *    with another context current, the next call looks it up again (again a call
 *    to make before any stream capture in that context).
 *  - Device-side errors (malformed cu_seqlens, a sequence longer than
 *    max_seqlen) are recorded in the array's status word: read it with
 *    kda_workspace_status(NULL, 0, stream, &code) on the same device.
 */
#define KDA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

kda_status kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *g,
                                 const void *beta, const float *initial_state,
                                 const int32_t *cu_seqlens, void *out, float *final_state,
                                 const kda_shape *shape, kda_stream_t stream);

/*
 * One decode step for N = shape->B sequences (one token each), updating the
 * fp32 state in place ("Kimi K3 深度拆解", section 4.2: constant cost per token,
 * O(d_k d_v) read-out independent of the position).
 *
 *  q, k, g     [N, H, dk] dtype      v [N, H, dv] dtype      beta [N, H] dtype
 *  state       fp32 [n_slots, H, dk, dv], updated in place
 *  state_slots int32 [N] indices into state (serving), or NULL for slot = n.
 *              Slots must be distinct within one call and < n_slots; the
 *              library does not check distinctness (duplicate slots race).
 *  n_slots     number of state slots (>= N when state_slots is NULL)
 *  out         [N, H, dv] dtype (written)
 *  shape       B = N, T = 1; n_seqs, max_seqlen and chunk are ignored.
 *  status      int32 device word, or NULL. A state_slots entry outside [0, n_slots)
 *              (only visible on the device) is not trapped: that sequence's state is
 *              left untouched, its out rows are set to NaN, and, when status is not
 *              NULL, 3 is written to *status. The library never clears *status (zero it
 *              before the steps it should cover); kda_workspace_status(status, 4, ...)
 *              reads it back.
 * Allocates nothing; safe to capture in a CUDA graph.
 */
kda_status kda_decode_step(const void *q, const void *k, const void *v, const void *g,
                           const void *beta, float *state, const int32_t *state_slots,
                           int64_t n_slots, void *out, const kda_shape *shape,
                           int32_t *status, kda_stream_t stream);

/*
 * Synchronises `stream` and reads the device-side status word a previous
 * kda_chunk_fwd (or kda_chunk_bwd) left in `workspace`: KDA_OK, or KDA_ERR_DEVICE
 * when a malformed cu_seqlens, a sequence longer than max_seqlen or an expired
 * bounded wait was detected (*device_code: 1 cu_seqlens or max_seqlen, 2 wait,
 * 3 decode slot). The word is cleared by the next kda_chunk_fwd on that workspace.
 * workspace == NULL reads the word of kda_chunk_fwd_noalloc's fixed array on the
 * current device (workspace_bytes is then ignored). A decode status word (see
 * kda_decode_step) is read the same way, with workspace_bytes = 4. Diagnostic only:
 * the compute path never calls it.
 */
kda_status kda_workspace_status(const void *workspace, size_t workspace_bytes,
                                kda_stream_t stream, int32_t *device_code);

/* Static description of a status code. Never NULL. */
const char *kda_status_string(kda_status status);

/* Library version, e.g. "0.1.0". */
const char *kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
