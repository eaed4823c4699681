"""Thin Python binding of the KDA C ABI (include/kda.h).

Argument marshalling only: every step of the computation runs in libkda.so's
CUDA kernels. PyTorch supplies device memory and the current stream. There is
no CPU or PyTorch fallback: if libkda.so is missing, importing this module
raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_DEVICE = range(5)
KDA_F32, KDA_BF16 = 0, 1
CHUNK = 64
PROLOGUE_QK_L2NORM = 1     # raw q, k: rows divided by max(||row||_2, 1e-12) in the kernels
PROLOGUE_GATE_SIGMOID = 2  # g holds gate pre-activations a: log decay = lb * sigmoid(a)


class KdaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib.kda_status_string(status).decode()}")


class Shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("B", ctypes.c_int32), ("H", ctypes.c_int32),
                ("dk", ctypes.c_int32), ("dv", ctypes.c_int32), ("n_seqs", ctypes.c_int32),
                ("max_seqlen", ctypes.c_int64), ("dtype", ctypes.c_int),
                ("scale", ctypes.c_float), ("g_lower_bound", ctypes.c_float),
                ("chunk", ctypes.c_int32), ("prologue", ctypes.c_int32)]


def _load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m kimi_delta_attention_19_b200.build` (no fallback exists)")
    L = ctypes.CDLL(path)
    p, sz, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    L.kda_chunk_fwd_workspace_size.restype = sz
    L.kda_chunk_fwd_workspace_size.argtypes = [ctypes.POINTER(Shape)]
    L.kda_chunk_fwd.restype = st
    L.kda_chunk_fwd.argtypes = [p, p, p, p, p, p, p, p, p, ctypes.POINTER(Shape), p, sz, p]
    L.kda_chunk_fwd_snapshots.restype = st
    L.kda_chunk_fwd_snapshots.argtypes = [p, p, p, p, p, p, p, p, p, ctypes.c_int32, p,
                                          ctypes.c_int64, ctypes.POINTER(Shape), p, sz, p]
    L.kda_chunk_bwd_workspace_size.restype = sz
    L.kda_chunk_bwd_workspace_size.argtypes = [ctypes.POINTER(Shape)]
    L.kda_chunk_bwd.restype = st
    L.kda_chunk_bwd.argtypes = [p, p, p, p, p, p, p, p, p, p, p, p, p, p, p,
                                ctypes.POINTER(Shape), p, sz, p]
    L.kda_snapshot_count.restype = ctypes.c_int64
    L.kda_snapshot_count.argtypes = [ctypes.POINTER(Shape), ctypes.c_int32]
    L.kda_chunk_fwd_noalloc.restype = st
    L.kda_chunk_fwd_noalloc.argtypes = [p, p, p, p, p, p, p, p, p, ctypes.POINTER(Shape), p]
    L.kda_decode_step.restype = st
    L.kda_decode_step.argtypes = [p, p, p, p, p, p, p, ctypes.c_int64, p,
                                  ctypes.POINTER(Shape), p, p]
    L.kda_workspace_status.restype = st
    L.kda_workspace_status.argtypes = [p, sz, p, ctypes.POINTER(ctypes.c_int32)]
    L.kda_status_string.restype = ctypes.c_char_p
    L.kda_status_string.argtypes = [st]
    L.kda_version.restype = ctypes.c_char_p
    L.kda_version.argtypes = []
    return L


lib = _load()


def load_library(path: str) -> ctypes.CDLL:
    """Another build of the same C ABI (e.g. the test-only short-wait variant), with the
    argument types declared as for `lib`."""
    return _load(path)

EXPORTED = ("kda_chunk_fwd_workspace_size", "kda_chunk_fwd", "kda_chunk_fwd_noalloc",
            "kda_chunk_fwd_snapshots", "kda_snapshot_count", "kda_chunk_bwd_workspace_size",
            "kda_chunk_bwd", "kda_decode_step",
            "kda_workspace_status", "kda_status_string", "kda_version")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KDA_F32
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; KDA takes float32 or bfloat16")


def _ptr(t: torch.Tensor | None):
    """Device address of a tensor argument; the C ABI takes contiguous token-major tensors."""
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError(f"KDA tensors must be contiguous (got strides {tuple(t.stride())} "
                         f"for shape {tuple(t.shape)})")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_shape(T: int, H: int, dk: int, dv: int, dtype: torch.dtype, *, B: int = 1,
               n_seqs: int = 0, max_seqlen: int = 0, scale: float | None = None,
               lb: float = -1.0, chunk: int = CHUNK, prologue: int = 0) -> Shape:
    code = KDA_F32 if dtype == torch.float32 else KDA_BF16
    return Shape(T=T, B=B, H=H, dk=dk, dv=dv, n_seqs=n_seqs, max_seqlen=max_seqlen, dtype=code,
                 scale=0.0 if scale is None else float(scale), g_lower_bound=float(lb),
                 chunk=chunk, prologue=int(prologue))


def workspace_size(shape: Shape) -> int:
    return int(lib.kda_chunk_fwd_workspace_size(ctypes.byref(shape)))


def alloc_workspace(shape: Shape, device) -> torch.Tensor:
    n = workspace_size(shape)
    if n == 0:
        raise KdaError(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_workspace_size")
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(n, dtype=torch.uint8, device=device)


def _prefill_shape(q, v, cu_seqlens, max_seqlen, scale, lb, prologue=0):
    batched = q.dim() == 4
    if batched:
        B, T, H, dk = q.shape
    else:
        B = 1
        T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is not None:
        assert not batched, "cu_seqlens takes packed [T, H, d] inputs"
        n = cu_seqlens.numel() - 1
    else:
        n = B
    shape = make_shape(T, H, dk, dv, q.dtype, B=B, n_seqs=n if cu_seqlens is not None else 0,
                       max_seqlen=max_seqlen, scale=scale, lb=lb, prologue=prologue)
    return shape, n


def chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
              beta: torch.Tensor, *, initial_state: torch.Tensor | None = None,
              cu_seqlens: torch.Tensor | None = None, max_seqlen: int = 0,
              scale: float | None = None, lb: float = -1.0, out: torch.Tensor | None = None,
              final_state: torch.Tensor | None = None, output_final_state: bool = True,
              workspace: torch.Tensor | None = None, prologue: int = 0, stream=None):
    """Chunked prefill. q, k, g: [T, H, dk] (or [B, T, H, dk]); v: [..., dv]; beta: [..., H].

    prologue: 0 or PROLOGUE_* flags (raw q/k and/or gate pre-activations in g).
    Returns (out, final_state). final_state is fp32 [n, H, dk, dv] (None if not requested).
    """
    shape, n = _prefill_shape(q, v, cu_seqlens, max_seqlen, scale, lb, prologue)
    H, dk, dv = shape.H, shape.dk, shape.dv
    if out is None:
        out = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty(n, H, dk, dv, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(shape, q.device)
    rc = lib.kda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state),
                           _ptr(cu_seqlens), _ptr(out), _ptr(final_state), ctypes.byref(shape),
                           _ptr(workspace), workspace.numel(), _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd")
    return out, final_state


def snapshot_count(shape: Shape, snapshot_chunks: int) -> int:
    """Snapshot slots kda_chunk_fwd_snapshots writes into for this shape (-1: invalid)."""
    return int(lib.kda_snapshot_count(ctypes.byref(shape), int(snapshot_chunks)))


def chunk_fwd_snapshots(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                        beta: torch.Tensor, *, snapshot_chunks: int,
                        snapshots: torch.Tensor | None = None,
                        initial_state: torch.Tensor | None = None,
                        cu_seqlens: torch.Tensor | None = None, max_seqlen: int = 0,
                        scale: float | None = None, lb: float = -1.0,
                        out: torch.Tensor | None = None, final_state: torch.Tensor | None = None,
                        output_final_state: bool = True, workspace: torch.Tensor | None = None,
                        prologue: int = 0, stream=None):
    """Prefill that also keeps the state every `snapshot_chunks` chunks (prefix cache).

    Returns (out, final_state, snapshots); snapshots is fp32 [snapshot_count, H, dk, dv].
    Sequence n (first packed token c_n) stores the state after its first m * snapshot_chunks
    * 64 tokens at index c_n // (snapshot_chunks * 64) + m - 1, m = 1, 2, ...; indices no
    sequence reaches keep their previous contents (zeros when this call allocates).
    """
    shape, n = _prefill_shape(q, v, cu_seqlens, max_seqlen, scale, lb, prologue)
    H, dk, dv = shape.H, shape.dk, shape.dv
    count = snapshot_count(shape, snapshot_chunks)
    if count < 0:
        raise KdaError(KDA_ERR_INVALID_ARG, "kda_snapshot_count")
    if snapshots is None:
        snapshots = torch.zeros(count, H, dk, dv, dtype=torch.float32, device=q.device)
    if out is None:
        out = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty(n, H, dk, dv, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(shape, q.device)
    rc = lib.kda_chunk_fwd_snapshots(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                     _ptr(initial_state), _ptr(cu_seqlens), _ptr(out),
                                     _ptr(final_state), int(snapshot_chunks),
                                     _ptr(snapshots) if snapshots.numel() else None,
                                     snapshots.shape[0], ctypes.byref(shape), _ptr(workspace),
                                     workspace.numel(), _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd_snapshots")
    return out, final_state, snapshots


def chunk_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
              beta: torch.Tensor, d_out: torch.Tensor | None, *,
              d_final_state: torch.Tensor | None = None,
              initial_state: torch.Tensor | None = None,
              cu_seqlens: torch.Tensor | None = None, max_seqlen: int = 0,
              scale: float | None = None, lb: float = -1.0, want_d_initial: bool = True,
              workspace: torch.Tensor | None = None, prologue: int = 0, stream=None):
    """Gradients of chunk_fwd: (dq, dk, dv, dg, dbeta, d_initial_state).

    Same layouts as chunk_fwd; d_out like out, d_final_state like final_state (fp32).
    d_initial_state is fp32 [n, H, dk, dv] (None unless want_d_initial). With prologue
    flags the inputs are raw and dq, dk, dg are the raw inputs' gradients.
    """
    shape, n = _prefill_shape(q, v, cu_seqlens, max_seqlen, scale, lb, prologue)
    H, dk, dv_ = shape.H, shape.dk, shape.dv
    dq, dkk, dg = (torch.empty_like(q) for _ in range(3))
    dvv = torch.empty_like(v)
    dbeta = torch.empty_like(beta)
    ds0 = (torch.empty(n, H, dk, dv_, dtype=torch.float32, device=q.device)
           if want_d_initial else None)
    if workspace is None:
        nbytes = int(lib.kda_chunk_bwd_workspace_size(ctypes.byref(shape)))
        if nbytes == 0:
            raise KdaError(KDA_ERR_INVALID_ARG, "kda_chunk_bwd_workspace_size")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    rc = lib.kda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                           _ptr(initial_state), _ptr(cu_seqlens), _ptr(d_out),
                           _ptr(d_final_state), _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dg),
                           _ptr(dbeta), _ptr(ds0), ctypes.byref(shape), _ptr(workspace),
                           workspace.numel(), _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_bwd")
    return dq, dkk, dvv, dg, dbeta, ds0


class _ChunkKDA(torch.autograd.Function):
    """chunk_fwd with chunk_bwd as its backward (both in the library's kernels)."""

    @staticmethod
    def forward(ctx, q, k, v, g, beta, initial_state, cu_seqlens, max_seqlen, scale, lb,
                prologue):
        out, fin = chunk_fwd(q, k, v, g, beta, initial_state=initial_state,
                             cu_seqlens=cu_seqlens, max_seqlen=max_seqlen, scale=scale, lb=lb,
                             prologue=prologue)
        ctx.save_for_backward(q, k, v, g, beta, initial_state, cu_seqlens)
        ctx.opts = (max_seqlen, scale, lb, prologue)
        return out, fin

    @staticmethod
    def backward(ctx, d_out, d_fin):
        q, k, v, g, beta, s0, cu = ctx.saved_tensors
        max_seqlen, scale, lb, prologue = ctx.opts
        dq, dk, dv, dg, dbeta, ds0 = chunk_bwd(
            q, k, v, g, beta, None if d_out is None else d_out.contiguous(),
            d_final_state=None if d_fin is None else d_fin.contiguous(), initial_state=s0,
            cu_seqlens=cu, max_seqlen=max_seqlen, scale=scale, lb=lb,
            want_d_initial=s0 is not None and ctx.needs_input_grad[5], prologue=prologue)
        return dq, dk, dv, dg, dbeta, ds0, None, None, None, None, None


def kda_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                  beta: torch.Tensor, *, initial_state: torch.Tensor | None = None,
                  cu_seqlens: torch.Tensor | None = None, max_seqlen: int = 0,
                  scale: float | None = None, lb: float = -1.0, prologue: int = 0):
    """Differentiable chunked prefill: (out, final_state) as chunk_fwd returns them, with
    gradients for q, k, v, g, beta and initial_state from kda_chunk_bwd (for training).
    Same layouts and options as chunk_fwd."""
    return _ChunkKDA.apply(q, k, v, g, beta, initial_state, cu_seqlens, max_seqlen, scale, lb,
                           prologue)


NOALLOC_SCRATCH_BYTES = 64 << 20


def chunk_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                      beta: torch.Tensor, *, out: torch.Tensor, final_state: torch.Tensor | None,
                      initial_state: torch.Tensor | None = None,
                      cu_seqlens: torch.Tensor | None = None, max_seqlen: int = 0,
                      scale: float | None = None, lb: float = -1.0, prologue: int = 0,
                      stream=None):
    """kda_chunk_fwd_noalloc: the prefill with the library's fixed scratch array.

    For callers that cannot allocate device memory, so `out` (and `final_state`,
    if wanted) must be passed in. Same layouts as chunk_fwd.
    """
    batched = q.dim() == 4
    if batched:
        B, T, H, dk = q.shape
    else:
        B = 1
        T, H, dk = q.shape
    dv = v.shape[-1]
    n = cu_seqlens.numel() - 1 if cu_seqlens is not None else 0
    shape = make_shape(T, H, dk, dv, q.dtype, B=B, n_seqs=n, max_seqlen=max_seqlen,
                       scale=scale, lb=lb, prologue=prologue)
    rc = lib.kda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                   _ptr(initial_state), _ptr(cu_seqlens), _ptr(out),
                                   _ptr(final_state), ctypes.byref(shape), _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd_noalloc")
    return out, final_state


def decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                beta: torch.Tensor, state: torch.Tensor, *, state_slots: torch.Tensor | None = None,
                scale: float | None = None, lb: float = -1.0, out: torch.Tensor | None = None,
                prologue: int = 0, status: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """One token per sequence: q, k, g [N, H, dk]; v [N, H, dv]; beta [N, H].

    Updates fp32 `state` [n_slots, H, dk, dv] in place; returns out [N, H, dv].
    `status` (int32 device tensor, optional) receives 3 when a state_slots entry is
    out of range (that sequence's out rows are NaN and its state is untouched).
    """
    N, H, dk = q.shape
    dv = v.shape[-1]
    shape = make_shape(1, H, dk, dv, q.dtype, B=N, scale=scale, lb=lb, prologue=prologue)
    if out is None:
        out = torch.empty(N, H, dv, dtype=q.dtype, device=q.device)
    rc = lib.kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state),
                             _ptr(state_slots), state.shape[0], _ptr(out), ctypes.byref(shape),
                             _ptr(status), _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_decode_step")
    return out


def workspace_status(workspace: torch.Tensor | None, stream=None) -> tuple[int, int]:
    """(status, device code) left in `workspace` by the last kda_chunk_fwd (synchronises).
    None reads the status word of chunk_fwd_noalloc's fixed array on the current device;
    a decode status tensor is read the same way as a workspace."""
    code = ctypes.c_int32(0)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.kda_workspace_status(_ptr(workspace), nbytes, _stream(stream), ctypes.byref(code))
    return rc, code.value


def default_scale(dk: int) -> float:
    return 1.0 / math.sqrt(dk)
