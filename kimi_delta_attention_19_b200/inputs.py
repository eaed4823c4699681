"""Seeded synthetic KDA workloads.

This module only draws inputs; it holds none of the attention arithmetic, so
both the CUDA path and the fp64 oracle can consume exactly the same tensors.

Recipe (one torch generator, seeded, drawn in this fixed order):
  lengths (varlen only) -> q -> k -> v -> g_raw -> beta_raw -> initial state
  q, k  ~ N(0, 1), then L2-normalised over d_k per (token, head)
  v     ~ N(0, 1)
  beta  = sigmoid(N(0, 1))                       (write strength in (0, 1))
  g     = -g_scale * sigmoid(N(0, 1))            (per-channel log decay in [-g_scale, 0))
  S0    ~ state_std * N(0, 1), fp32              (or absent -> zeros)
Everything is drawn in fp32 and cast once to the input dtype, before any
consumer sees it. With raw=True (inputs for the library's prologue) the same
draws are returned untransformed: q, k ~ N(0, 1) not normalised, and g holds
the gate pre-activation g_scale * N(0, 1).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass
class Workload:
    """One named workload: shapes, dtype and distribution parameters."""
    name: str
    H: int
    dk: int
    dv: int
    dtype: torch.dtype
    T: int = 0                      # tokens per sequence (fixed-length) ...
    B: int = 1
    varlen: list[int] | None = None  # ... or explicit packed lengths
    n_varlen: int = 0               # draw this many lengths U[len_lo, len_hi]
    len_lo: int = 0
    len_hi: int = 0
    chunk: int = 64
    g_scale: float = 1.0
    state_std: float | None = 0.02
    lb: float = -1.0
    extra: dict = field(default_factory=dict)


# The five workloads the library is specified and measured on.
WORKLOADS = {
    "fp32_h2_t256_d64": Workload("fp32_h2_t256_d64", H=2, dk=64, dv=64, dtype=torch.float32,
                                 T=256, state_std=None),
    "bf16_h32_t8192_d128": Workload("bf16_h32_t8192_d128", H=32, dk=128, dv=128,
                                    dtype=torch.bfloat16, T=8192),
    "varlen8_h32_d128": Workload("varlen8_h32_d128", H=32, dk=128, dv=128, dtype=torch.bfloat16,
                                 n_varlen=8, len_lo=1024, len_hi=32768),
    "bf16_h16_t1m_d128": Workload("bf16_h16_t1m_d128", H=16, dk=128, dv=128,
                                  dtype=torch.bfloat16, T=1 << 20),
    "decode_n256_h32_d128": Workload("decode_n256_h32_d128", H=32, dk=128, dv=128,
                                     dtype=torch.bfloat16, B=256, T=1,
                                     extra={"steps": 1000}),
}


@dataclass
class Inputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    initial_state: torch.Tensor | None
    cu_seqlens: torch.Tensor | None   # int32 [n+1] or None
    lengths: list[int]


def draw_lengths(n: int, lo: int, hi: int, gen: torch.Generator) -> list[int]:
    """n sequence lengths uniform on the integers [lo, hi]."""
    x = torch.randint(lo, hi + 1, (n,), generator=gen, device=gen.device)
    return [int(v) for v in x.cpu().tolist()]


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_inputs(T: int | None = None, H: int = 2, dk: int = 64, dv: int = 64, *,
                dtype: torch.dtype = torch.float32, seed: int = 0, device: str = "cpu",
                lengths: list[int] | None = None, n_varlen: int = 0, len_lo: int = 0,
                len_hi: int = 0, g_scale: float = 1.0, state_std: float | None = 0.02,
                batch: int | None = None, raw: bool = False) -> Inputs:
    """Draw one workload's inputs.

    Token-major packed layout: q, k, g [T, H, dk]; v [T, H, dv]; beta [T, H].
    With `lengths` or `n_varlen`, tokens of several sequences are packed and
    cu_seqlens (int32) delimits them; `batch` B gives B sequences of T tokens
    each, also packed (T_total = B*T) with a cu_seqlens.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    if n_varlen:
        lengths = draw_lengths(n_varlen, len_lo, len_hi, gen)
    if batch is not None:
        lengths = [T] * batch
    if lengths is not None:
        T_total = int(sum(lengths))
    else:
        assert T is not None
        T_total = T
        lengths = [T]

    def randn(*shape):
        return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)

    unit = (lambda x: x) if raw else _l2n
    q = unit(randn(T_total, H, dk)).to(dtype)
    k = unit(randn(T_total, H, dk)).to(dtype)
    v = randn(T_total, H, dv).to(dtype)
    g_raw = randn(T_total, H, dk)
    g = (g_scale * g_raw if raw else -g_scale * torch.sigmoid(g_raw)).to(dtype)
    beta = torch.sigmoid(randn(T_total, H)).to(dtype)
    n = len(lengths)
    s0 = None
    if state_std is not None:
        s0 = (state_std * randn(n, H, dk, dv)).contiguous()
    cu = None
    if len(lengths) > 1 or n_varlen:
        c = [0]
        for L in lengths:
            c.append(c[-1] + int(L))
        cu = torch.tensor(c, dtype=torch.int32, device=device)
    return Inputs(q, k, v, g, beta, s0, cu, list(lengths))


def correlated_key_inputs(*, seed: int = 19, H: int = 4, lengths: list[int] | None = None,
                          noise: float = 0.8, g_scale: float = 0.05) -> Inputs:
    """bf16 inputs whose keys share one direction per head (unit rows of base + noise * N(0, 1):
    pairwise cosine ~0.6 at noise 0.8) with a weak decay (g = -g_scale * sigmoid(N(0, 1))) and
    beta = sigmoid(N(1, 1)): an ill-conditioned (I + A) with large off-diagonal inverse blocks.
    d_k = d_v = 128; q, v and the initial state as in make_inputs."""
    x = make_inputs(None, H=H, dk=128, dv=128, dtype=torch.float32, seed=seed,
                    lengths=lengths or [192, 77], state_std=0.02)
    gen = torch.Generator().manual_seed(seed + 1)
    base = torch.randn(1, H, 128, generator=gen)
    k = base + noise * torch.randn(x.k.shape, generator=gen)
    x.k = _l2n(k).to(torch.bfloat16)
    x.q = x.q.to(torch.bfloat16)
    x.v = x.v.to(torch.bfloat16)
    x.g = (-g_scale * torch.sigmoid(torch.randn(x.g.shape, generator=gen))).to(torch.bfloat16)
    x.beta = torch.sigmoid(torch.randn(x.beta.shape, generator=gen) + 1.0).to(torch.bfloat16)
    return x


def workload_inputs(w: Workload, *, seed: int = 0, device: str = "cpu") -> Inputs:
    """Inputs for a named prefill workload (decode draws per step, see decode_token)."""
    if w.n_varlen:
        return make_inputs(None, w.H, w.dk, w.dv, dtype=w.dtype, seed=seed, device=device,
                           n_varlen=w.n_varlen, len_lo=w.len_lo, len_hi=w.len_hi,
                           g_scale=w.g_scale, state_std=w.state_std)
    return make_inputs(w.T, w.H, w.dk, w.dv, dtype=w.dtype, seed=seed, device=device,
                       g_scale=w.g_scale, state_std=w.state_std,
                       batch=(w.B if w.B > 1 else None))


def decode_state(N: int, H: int, dk: int, dv: int, *, seed: int = 0, device: str = "cpu",
                 state_std: float = 0.02) -> torch.Tensor:
    """fp32 serving state [N, H, dk, dv] ~ state_std * N(0, 1)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return state_std * torch.randn(N, H, dk, dv, generator=gen, device=device,
                                   dtype=torch.float32)


def decode_tokens(steps: int, N: int, H: int, dk: int, dv: int, *, dtype=torch.bfloat16,
                  seed: int = 1, device: str = "cpu", g_scale: float = 1.0,
                  raw: bool = False) -> Inputs:
    """`steps` tokens for each of N sequences, step-major: q, k, g [steps, N, H, dk] etc.
    raw=True: untransformed draws, as in make_inputs."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)

    def randn(*shape):
        return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)

    unit = (lambda x: x) if raw else _l2n
    q = unit(randn(steps, N, H, dk)).to(dtype)
    k = unit(randn(steps, N, H, dk)).to(dtype)
    v = randn(steps, N, H, dv).to(dtype)
    g_raw = randn(steps, N, H, dk)
    g = (g_scale * g_raw if raw else -g_scale * torch.sigmoid(g_raw)).to(dtype)
    beta = torch.sigmoid(randn(steps, N, H)).to(dtype)
    return Inputs(q, k, v, g, beta, None, None, [steps] * N)
