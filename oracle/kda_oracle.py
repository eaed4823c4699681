"""Python face of the KDA oracle (fp64, CPU).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers. Nothing in the CUDA library imports this
module, and this module imports nothing from the library.

Two independent fp64 implementations live here:

* ``recurrent`` -- the token-by-token definition (C, ``kda_oracle.c``):
  S_t = (I - b_t k_t k_t^T) Diag(exp max(g_t, lb)) S_{t-1} + b_t k_t v_t^T,
  o_t = scale * S_t^T q_t.  Sources: "Kimi K3 深度拆解" (chenxutan.com) section 4.2
  (delta rule, toy single-head loop), "Kimi K3 技術報告：三個架構改動" (akiraxclaw.com)
  section "長度" (channel-wise gating), "3 分钟看懂 Kimi K3" (landx.limxdynamics.com)
  "第一条主线" / Figure 3 (log decay bounded below).

  ``backward`` is the reverse-mode gradient of that loop (C), differentiating each
  step of it in reverse order with recomputed states.

  Options of the same C loop: ``recurrent_snapshots`` also records the state after
  every P tokens of each sequence (prefix-cache snapshots), and ``prologue`` takes raw
  inputs: q, k rows L2-normalised per token (QK_L2NORM) and/or gate pre-activations a
  with log decay lb * sigmoid(a) (GATE_SIGMOID).

* ``chunked`` -- the closed form of the same recurrence over chunks of C
  tokens, derived independently (numpy, plain matrix products, one chunk at a
  time). Used only to pin ``recurrent``; it is the chunk-parallel form the
  pages name in "Kimi K3 深度拆解" section 4.2 ("chunk 并行、块间递推").
  Within a chunk with inclusive per-channel log-decay sums G_r:
      K~ = K*exp(G), K^ = K*exp(-G), Q~ = Q*exp(G)
      A  = Diag(beta) * strict_lower(K~ K^^T)
      U  = (I + A)^{-1} Diag(beta) (V - K~ S0)
      O  = scale * (Q~ S0 + lower_incl(Q~ K^^T) U)
      S  = Diag(exp G_last) S0 + (K * exp(G_last - G))^T U
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lib = None
_lib_lock = threading.Lock()

F32 = 0
BF16 = 1
QK_L2NORM = 1       # prologue: q, k rows divided by max(||.||_2, 1e-12)
GATE_SIGMOID = 2    # prologue: g holds pre-activations a, log decay = lb * sigmoid(a)


def build(src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the C oracle into a shared library (plain gcc, no GPU)."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _bind(path: str):
    lib = ctypes.CDLL(path)
    f = lib.kda_oracle_recurrent
    f.restype = ctypes.c_int
    p = ctypes.c_void_p
    f.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  p, ctypes.c_int, p, p, p, p, p, p, ctypes.c_double, ctypes.c_double,
                  p, p, ctypes.c_int64, p, ctypes.c_int]
    f = lib.kda_oracle_recurrent_ex
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  p, ctypes.c_int, p, p, p, p, p, p, ctypes.c_double, ctypes.c_double,
                  p, p, ctypes.c_int64, p, ctypes.c_int64, p, p, ctypes.c_int, ctypes.c_int]
    f = lib.kda_oracle_backward
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  p, ctypes.c_int, p, p, p, p, p, p, ctypes.c_double, ctypes.c_double,
                  p, p, p, p, p, p, p, p, ctypes.c_int, ctypes.c_int]
    return lib


def load(path: str | None = None):
    """Load (building first if missing or older than the source) the oracle library."""
    global _lib
    if path is not None:
        return _bind(path)
    with _lib_lock:
        if _lib is None:
            stale = (not os.path.exists(_LIB_PATH)
                     or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
            if stale:
                build()
            _lib = _bind(_LIB_PATH)
    return _lib


def _as_input(x):
    """Return (contiguous numpy array, dtype code). Accepts torch (f32/bf16) or numpy f32."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach()
            if x.device.type != "cpu":
                x = x.cpu()
            x = x.contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), F32
            raise TypeError(f"oracle input dtype {x.dtype} not supported")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"oracle input dtype {x.dtype} not supported")


def recurrent(q, k, v, g, beta, *, cu_seqlens=None, initial_state=None,
              lb: float = -1.0, scale: float | None = None, out_rows=None,
              want_out: bool = True, prologue: int = 0, n_threads: int | None = None,
              lib=None):
    """Token-by-token fp64 recurrence.

    prologue: 0, or QK_L2NORM | GATE_SIGMOID (the raw-input prologue, see kda_oracle.c).

    q, k, g: [T, H, dk]; v: [T, H, dv]; beta: [T, H] (all the same dtype, f32 or bf16).
    cu_seqlens: None (one sequence) or int sequence [n+1].
    initial_state: None or fp64/f32 array [n, H, dk, dv].
    out_rows: None (all tokens) or sorted token indices; the output then has one
    row per listed token.
    Returns (out fp64 [rows, H, dv] or None, final_state fp64 [n, H, dk, dv]).
    """
    qa, dt = _as_input(q)
    ka, dt2 = _as_input(k)
    va, dt3 = _as_input(v)
    ga, dt4 = _as_input(g)
    ba, dt5 = _as_input(beta)
    if len({dt, dt2, dt3, dt4, dt5}) != 1:
        raise TypeError("all oracle inputs must share one dtype")
    T, H, dk = qa.shape
    dv = va.shape[2]
    assert ka.shape == (T, H, dk) and ga.shape == (T, H, dk)
    assert va.shape == (T, H, dv) and ba.shape == (T, H)
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    n = len(cu) - 1
    s0 = None
    if initial_state is not None:
        s0 = np.ascontiguousarray(np.asarray(_to_numpy(initial_state), dtype=np.float64))
        assert s0.shape == (n, H, dk, dv), s0.shape
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    rows = None
    if out_rows is not None:
        rows = np.ascontiguousarray(np.asarray(out_rows, dtype=np.int64))
        assert np.all(np.diff(rows) > 0), "out_rows must be strictly increasing"
    n_rows = T if rows is None else len(rows)
    out = np.zeros((n_rows, H, dv), dtype=np.float64) if want_out else None
    fin = np.zeros((n, H, dk, dv), dtype=np.float64)
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    lib = lib or load()

    def ptr(a):
        return None if a is None else a.ctypes.data_as(ctypes.c_void_p)

    if prologue:
        rc = lib.kda_oracle_recurrent_ex(T, H, dk, dv, n, ptr(cu), dt, ptr(qa), ptr(ka),
                                         ptr(va), ptr(ga), ptr(ba), ptr(s0), float(lb),
                                         float(scale), ptr(out), ptr(rows),
                                         0 if rows is None else len(rows), ptr(fin), 0, None,
                                         None, int(prologue), int(n_threads))
    else:
        rc = lib.kda_oracle_recurrent(T, H, dk, dv, n, ptr(cu), dt, ptr(qa), ptr(ka), ptr(va),
                                      ptr(ga), ptr(ba), ptr(s0), float(lb), float(scale),
                                      ptr(out), ptr(rows), 0 if rows is None else len(rows),
                                      ptr(fin), int(n_threads))
    if rc != 0:
        raise ValueError(f"kda_oracle_recurrent failed with code {rc}")
    return out, fin


def recurrent_snapshots(q, k, v, g, beta, *, snapshot_tokens: int, cu_seqlens=None,
                        initial_state=None, lb: float = -1.0, scale: float | None = None,
                        want_out: bool = False, prologue: int = 0,
                        n_threads: int | None = None, lib=None):
    """The token-by-token recurrence, also recording the state at regular points.

    For each sequence n and every m >= 1 with m * snapshot_tokens <= len_n, the
    state after the sequence's first m * snapshot_tokens tokens (seeded by its
    initial state). A prefix cache keeps such states ("3 分钟看懂 Kimi K3",
    第一条主线: KDA state and prefix-cache scheduling for long requests).

    Returns (out or None, final_state [n, H, dk, dv], snaps [sum_n count_n, H, dk, dv],
    first [n]): sequence n's snapshots are snaps[first[n] : first[n] + count_n] in order,
    count_n = len_n // snapshot_tokens (a compact layout, all fp64).
    """
    qa, dt = _as_input(q)
    ka, _ = _as_input(k)
    va, _ = _as_input(v)
    ga, _ = _as_input(g)
    ba, _ = _as_input(beta)
    T, H, dk = qa.shape
    dv = va.shape[2]
    if snapshot_tokens <= 0:
        raise ValueError("snapshot_tokens must be positive")
    cu = (np.array([0, T], dtype=np.int64) if cu_seqlens is None
          else np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64)))
    n = len(cu) - 1
    counts = np.diff(cu) // snapshot_tokens
    first = np.ascontiguousarray(np.concatenate([[0], np.cumsum(counts)[:-1]]).astype(np.int64))
    snaps = np.zeros((max(int(counts.sum()), 1), H, dk, dv), dtype=np.float64)
    s0 = None
    if initial_state is not None:
        s0 = np.ascontiguousarray(np.asarray(_to_numpy(initial_state), dtype=np.float64))
        assert s0.shape == (n, H, dk, dv), s0.shape
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    out = np.zeros((T, H, dv), dtype=np.float64) if want_out else None
    fin = np.zeros((n, H, dk, dv), dtype=np.float64)
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    lib = lib or load()

    def ptr(a):
        return None if a is None else a.ctypes.data_as(ctypes.c_void_p)

    rc = lib.kda_oracle_recurrent_ex(T, H, dk, dv, n, ptr(cu), dt, ptr(qa), ptr(ka),
                                     ptr(va), ptr(ga), ptr(ba), ptr(s0), float(lb),
                                     float(scale), ptr(out), None, 0, ptr(fin),
                                     int(snapshot_tokens), ptr(first), ptr(snaps),
                                     int(prologue), int(n_threads))
    if rc != 0:
        raise ValueError(f"kda_oracle_recurrent_snapshots failed with code {rc}")
    return out, fin, snaps[:int(counts.sum())], first


def backward(q, k, v, g, beta, *, d_out=None, d_final=None, cu_seqlens=None,
             initial_state=None, lb: float = -1.0, scale: float | None = None,
             prologue: int = 0, n_threads: int | None = None, lib=None) -> dict:
    """fp64 reverse-mode gradients of the token recurrence (kda_oracle.c, "backward").

    prologue: 0, or QK_L2NORM | GATE_SIGMOID: raw inputs; gradients of the raw q, k and
    gate pre-activations.

    d_out: dL/do [T, H, dv] (None = 0); d_final: dL/dS_final [n, H, dk, dv] (None = 0).
    Returns dict dq, dk, dg [T, H, dk], dv [T, H, dv], dbeta [T, H], ds0 [n, H, dk, dv],
    all fp64 numpy.
    """
    qa, dt = _as_input(q)
    ka, _ = _as_input(k)
    va, _ = _as_input(v)
    ga, _ = _as_input(g)
    ba, _ = _as_input(beta)
    T, H, dk = qa.shape
    dv = va.shape[2]
    cu = (np.array([0, T], dtype=np.int64) if cu_seqlens is None
          else np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64)))
    n = len(cu) - 1

    def f64(x, shape):
        if x is None:
            return None
        a = np.ascontiguousarray(np.asarray(_to_numpy(x), dtype=np.float64))
        assert a.shape == shape, (a.shape, shape)
        return a
    s0 = f64(initial_state, (n, H, dk, dv))
    do = f64(d_out, (T, H, dv))
    dS = f64(d_final, (n, H, dk, dv))
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    res = {"dq": np.zeros((T, H, dk)), "dk": np.zeros((T, H, dk)), "dv": np.zeros((T, H, dv)),
           "dg": np.zeros((T, H, dk)), "dbeta": np.zeros((T, H)),
           "ds0": np.zeros((n, H, dk, dv))}
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    lib = lib or load()

    def ptr(a):
        return None if a is None else a.ctypes.data_as(ctypes.c_void_p)

    rc = lib.kda_oracle_backward(T, H, dk, dv, n, ptr(cu), dt, ptr(qa), ptr(ka), ptr(va),
                                 ptr(ga), ptr(ba), ptr(s0), float(lb), float(scale), ptr(do),
                                 ptr(dS), ptr(res["dq"]), ptr(res["dk"]), ptr(res["dv"]),
                                 ptr(res["dg"]), ptr(res["dbeta"]), ptr(res["ds0"]),
                                 int(prologue), int(n_threads))
    if rc != 0:
        raise ValueError(f"kda_oracle_backward failed with code {rc}")
    return res


def _to_numpy(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().cpu().double().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x)


def _widen(x) -> np.ndarray:
    """Exact widening of an f32 / bf16 input to fp64 numpy (fp64 inputs pass through)."""
    if isinstance(x, np.ndarray) and x.dtype == np.float64:
        return x
    a, dt = _as_input(x)
    if dt == BF16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _forward_substitution(L: np.ndarray, B: np.ndarray) -> np.ndarray:
    """Solve (I + L) X = B for strictly lower-triangular L, row by row."""
    n = L.shape[0]
    X = np.zeros_like(B)
    for r in range(n):
        X[r] = B[r] - L[r, :r] @ X[:r]
    return X


def chunked(q, k, v, g, beta, *, chunk: int, cu_seqlens=None, initial_state=None,
            lb: float = -1.0, scale: float | None = None):
    """fp64 chunked closed form (see module docstring). Small inputs only."""
    Q, K, V, G, B = (_widen(x) for x in (q, k, v, g, beta))
    T, H, dk = Q.shape
    dv = V.shape[2]
    cu = [0, T] if cu_seqlens is None else [int(c) for c in cu_seqlens]
    n = len(cu) - 1
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    out = np.zeros((T, H, dv))
    fin = np.zeros((n, H, dk, dv))
    S0all = None if initial_state is None else np.asarray(_to_numpy(initial_state), dtype=np.float64)
    for s in range(n):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0all is None else S0all[s, h].copy()
            for c0 in range(cu[s], cu[s + 1], chunk):
                c1 = min(c0 + chunk, cu[s + 1])
                Kc, Qc, Vc = K[c0:c1, h], Q[c0:c1, h], V[c0:c1, h]
                bc = B[c0:c1, h]
                Gc = np.cumsum(np.maximum(G[c0:c1, h], lb), axis=0)
                Kt = Kc * np.exp(Gc)
                Kh = Kc * np.exp(-Gc)
                Qt = Qc * np.exp(Gc)
                A = np.tril(Kt @ Kh.T, -1) * bc[:, None]
                U = _forward_substitution(A, bc[:, None] * (Vc - Kt @ S))
                out[c0:c1, h] = scale * (Qt @ S + np.tril(Qt @ Kh.T) @ U)
                S = np.exp(Gc[-1])[:, None] * S + (Kc * np.exp(Gc[-1] - Gc)).T @ U
            fin[s, h] = S
    return out, fin
