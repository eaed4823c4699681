"""GPU parity of the backward pass (kda_chunk_bwd) against the fp64 reverse-mode oracle:
every gradient (dq, dk, dv, dg, dbeta, dS0) element by element, on the CUDA-core fp32
inputs and on bf16 inputs (whose chunk start states come from the tensor-core forward),
with varlen, empty and ragged sequences, the clamp active, and multi-segment forwards."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from kimi_delta_attention_19_b200.inputs import make_inputs
from oracle import kda_oracle as ko
from tests.parity import errors

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
# rel-L2 bounds per gradient: fp32 inputs are computed in fp32 throughout (observed
# <= 1.1e-6); bf16 inputs add the bf16 rounding of the stored gradients (2^-9 relative)
# and the tensor-core forward's chunk start states, the forward's own budget (observed
# <= 2.2e-3), so they take the forward's bf16 bound.
TOL = {torch.float32: 1e-5, torch.bfloat16: 5e-3}
# max-abs bounds per gradient, relative to the gradient's largest magnitude (at least 1),
# so that one bad element cannot hide behind the norm: bf16 takes the forward's max-abs
# bound of 3e-2 on O(1) values; fp32 is 1e-4 (observed max-abs <= ~1e-5 relative).
MAX_ABS = {torch.float32: 1e-4, torch.bfloat16: 3e-2}
NAMES = ("dq", "dk", "dv", "dg", "dbeta", "ds0")


@pytest.fixture(scope="module")
def kda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kimi_delta_attention_19_b200 import kda as k
    return k


def _check(kda, x, dtype, what, lb=-1.0, seed=0, with_final=True, prologue=0):
    rng = np.random.default_rng(seed)
    T, H, dv = x.v.shape
    n = len(x.lengths)
    d_out = torch.tensor(rng.standard_normal((T, H, dv)), dtype=torch.float32).to(dtype)
    d_fin = (torch.tensor(rng.standard_normal((n, H, x.q.shape[2], dv)), dtype=torch.float32)
             if with_final else None)
    cu = x.cu_seqlens
    got = kda.chunk_bwd(*(t.to(DEV) for t in (x.q, x.k, x.v, x.g, x.beta)), d_out.to(DEV),
                        d_final_state=None if d_fin is None else d_fin.to(DEV),
                        initial_state=x.initial_state.to(DEV),
                        cu_seqlens=None if cu is None else cu.to(DEV),
                        max_seqlen=max(x.lengths), lb=lb, prologue=prologue)
    torch.cuda.synchronize()
    ref = ko.backward(x.q, x.k, x.v, x.g, x.beta, d_out=d_out.double(), d_final=d_fin,
                      cu_seqlens=None if cu is None else cu.tolist(),
                      initial_state=x.initial_state, lb=lb, prologue=prologue)
    for name, gt in zip(NAMES, got):
        rel, mx = errors(gt, ref[name])
        assert rel <= TOL[dtype], f"{what} {name}: rel-L2 {rel:.3e} > {TOL[dtype]:.0e} (max-abs {mx:.3e})"
        bound = MAX_ABS[dtype] * max(1.0, float(np.max(np.abs(ref[name]))) if ref[name].size else 1.0)
        assert mx <= bound, f"{what} {name}: max-abs {mx:.3e} > {bound:.3e} (rel-L2 {rel:.3e})"


@pytest.mark.parametrize("d", [64, 128])
def test_backward_fp32(kda, d):
    x = make_inputs(None, H=2, dk=d, dv=d, dtype=torch.float32, seed=501 + d,
                    lengths=[130, 0, 64, 70, 1], state_std=0.02)
    _check(kda, x, torch.float32, f"fp32 d={d}")


def test_backward_fp32_clamp_active(kda):
    x = make_inputs(None, H=2, dk=64, dv=64, dtype=torch.float32, seed=503, lengths=[200],
                    state_std=0.02, g_scale=3.0)
    assert float(x.g.min()) < -1.0
    _check(kda, x, torch.float32, "clamp active")


def test_backward_mixed_dims(kda):
    x = make_inputs(None, H=2, dk=128, dv=64, dtype=torch.float32, seed=504, lengths=[100, 29],
                    state_std=0.02)
    _check(kda, x, torch.float32, "dk=128 dv=64")
    x = make_inputs(None, H=2, dk=64, dv=128, dtype=torch.bfloat16, seed=505, lengths=[77],
                    state_std=0.02)
    _check(kda, x, torch.bfloat16, "dk=64 dv=128 bf16")


def test_backward_bf16_tensor_core_forward(kda):
    """bf16 d=128: chunk start states from the tensor-core forward, several segments."""
    x = make_inputs(None, H=2, dk=128, dv=128, dtype=torch.bfloat16, seed=506,
                    lengths=[330, 0, 1300, 64], state_std=0.02)
    _check(kda, x, torch.bfloat16, "bf16 tc")


def test_backward_without_upstream_state_grad(kda):
    x = make_inputs(None, H=4, dk=128, dv=128, dtype=torch.bfloat16, seed=507,
                    lengths=[257, 3], state_std=0.02)
    _check(kda, x, torch.bfloat16, "no dS_final", with_final=False)


def test_full_bf16_h32_t8192_d128_backward(kda):
    """The 8K-token, 32-head workload: every gradient of every element."""
    from kimi_delta_attention_19_b200.inputs import WORKLOADS, workload_inputs
    x = workload_inputs(WORKLOADS["bf16_h32_t8192_d128"])
    _check(kda, x, torch.bfloat16, "8K x 32 heads", seed=7)


@pytest.mark.parametrize("dtype,d,prologue", [(torch.bfloat16, 128, 3), (torch.float32, 64, 3),
                                              (torch.float32, 128, 1), (torch.bfloat16, 64, 2)])
def test_backward_prologue(kda, dtype, d, prologue):
    """Raw inputs through the fused prologue: gradients of the raw q, k (L2 normalisation)
    and gate pre-activations (lb * sigmoid), against the oracle's chain rule."""
    raw = make_inputs(None, H=2, dk=d, dv=d, dtype=dtype, seed=508 + d, lengths=[140, 0, 64],
                      state_std=0.02, raw=True)
    ref = make_inputs(None, H=2, dk=d, dv=d, dtype=dtype, seed=508 + d, lengths=[140, 0, 64],
                      state_std=0.02)
    if not prologue & 1:
        raw.q, raw.k = ref.q, ref.k
    if not prologue & 2:
        raw.g = ref.g
    _check(kda, raw, dtype, f"prologue={prologue} {dtype} d={d}", lb=-0.9, prologue=prologue)


def test_backward_batched_layout_and_no_dout(kda):
    """[B, T, H, d] inputs without cu_seqlens, and d_out = None (only dS_final drives L)."""
    x = make_inputs(100, H=2, dk=128, dv=128, dtype=torch.bfloat16, seed=512, batch=3,
                    state_std=0.02)
    rng = np.random.default_rng(5)
    d_fin = torch.tensor(rng.standard_normal((3, 2, 128, 128)), dtype=torch.float32)
    args = [t.to(DEV).view(3, 100, *t.shape[1:]) for t in (x.q, x.k, x.v, x.g, x.beta)]
    got = kda.chunk_bwd(*args, None, d_final_state=d_fin.to(DEV),
                        initial_state=x.initial_state.to(DEV))
    torch.cuda.synchronize()
    ref = ko.backward(x.q, x.k, x.v, x.g, x.beta, d_out=None, d_final=d_fin,
                      cu_seqlens=x.cu_seqlens.tolist(), initial_state=x.initial_state)
    for name, gt in zip(NAMES, got):
        rel, mx = errors(gt.reshape(ref[name].shape), ref[name])
        assert rel <= TOL[torch.bfloat16], f"batched {name}: rel-L2 {rel:.3e}"


def test_backward_bad_cu_seqlens_reports_without_trap(kda):
    """A malformed cu_seqlens is skipped and reported in the workspace status word."""
    x = make_inputs(None, H=2, dk=64, dv=64, dtype=torch.float32, seed=513,
                    lengths=[100, 60], state_std=0.02)
    cu = torch.tensor([0, 120, 100], dtype=torch.int32, device=DEV)  # not monotone
    shape = kda.make_shape(160, 2, 64, 64, torch.float32, n_seqs=2, max_seqlen=120)
    ws = torch.empty(int(kda.lib.kda_chunk_bwd_workspace_size(kda.ctypes.byref(shape))),
                     dtype=torch.uint8, device=DEV)
    d_out = torch.ones_like(x.v).to(DEV)
    kda.chunk_bwd(*(t.to(DEV) for t in (x.q, x.k, x.v, x.g, x.beta)), d_out, cu_seqlens=cu,
                  max_seqlen=120, workspace=ws)
    rc, code = kda.workspace_status(ws)
    assert rc == kda.KDA_ERR_DEVICE and code != 0


def test_autograd_function_matches_oracle(kda):
    """kda_attention under torch autograd: loss.backward() gives the oracle's gradients."""
    x = make_inputs(None, H=2, dk=64, dv=64, dtype=torch.float32, seed=520,
                    lengths=[100, 40], state_std=0.02)
    q, k, v, g, b = (t.to(DEV).requires_grad_() for t in (x.q, x.k, x.v, x.g, x.beta))
    s0 = x.initial_state.to(DEV).requires_grad_()
    out, fin = kda.kda_attention(q, k, v, g, b, initial_state=s0,
                                 cu_seqlens=x.cu_seqlens.to(DEV), max_seqlen=100)
    rng = np.random.default_rng(9)
    w_out = torch.tensor(rng.standard_normal(tuple(out.shape)), dtype=torch.float32).to(DEV)
    w_fin = torch.tensor(rng.standard_normal(tuple(fin.shape)), dtype=torch.float32).to(DEV)
    loss = (out * w_out).sum() + (fin * w_fin).sum()
    loss.backward()
    torch.cuda.synchronize()
    ref = ko.backward(x.q, x.k, x.v, x.g, x.beta, d_out=w_out.cpu().double(),
                      d_final=w_fin.cpu(), cu_seqlens=x.cu_seqlens.tolist(),
                      initial_state=x.initial_state)
    for name, t in zip(NAMES, (q, k, v, g, b, s0)):
        rel, mx = errors(t.grad, ref[name])
        assert rel <= TOL[torch.float32], f"autograd {name}: rel-L2 {rel:.3e}"
