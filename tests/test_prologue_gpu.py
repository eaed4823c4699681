"""GPU parity of the fused raw-input prologue against the fp64 oracle running the same
prologue: q/k rows L2-normalised per (token, head) inside the kernels
(KDA_PROLOGUE_QK_L2NORM) and log decays lb * sigmoid(a) from gate pre-activations
(KDA_PROLOGUE_GATE_SIGMOID), on every path: the tensor-core prefill (all four flag
combinations), the CUDA-core prefill, the snapshots entry point and the decode step."""
from __future__ import annotations

import pytest
import torch

from kimi_delta_attention_19_b200.inputs import decode_state, decode_tokens, make_inputs
from oracle import kda_oracle as ko
from tests.parity import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
QK, GATE = ko.QK_L2NORM, ko.GATE_SIGMOID


@pytest.fixture(scope="module")
def kda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kimi_delta_attention_19_b200 import kda as k
    assert (k.PROLOGUE_QK_L2NORM, k.PROLOGUE_GATE_SIGMOID) == (QK, GATE)
    return k


def _inputs(lengths, H, d, dtype, seed, prologue):
    """Raw where the prologue transforms, the usual (normalised / -sigmoid) draws elsewhere."""
    raw = make_inputs(None, H=H, dk=d, dv=d, dtype=dtype, seed=seed, lengths=lengths,
                      state_std=0.02, raw=True)
    ref = make_inputs(None, H=H, dk=d, dv=d, dtype=dtype, seed=seed, lengths=lengths,
                      state_std=0.02)
    if not prologue & QK:
        raw.q, raw.k = ref.q, ref.k
    if not prologue & GATE:
        raw.g = ref.g
    return raw


def _check(kda, x, dtype, prologue, what, lb=-1.0):
    cu = x.cu_seqlens
    out, fin = kda.chunk_fwd(*(t.to(DEV) for t in (x.q, x.k, x.v, x.g, x.beta)),
                             initial_state=x.initial_state.to(DEV),
                             cu_seqlens=None if cu is None else cu.to(DEV),
                             max_seqlen=max(x.lengths), lb=lb, prologue=prologue)
    torch.cuda.synchronize()
    ro, rs = ko.recurrent(x.q, x.k, x.v, x.g, x.beta,
                          cu_seqlens=None if cu is None else cu.tolist(),
                          initial_state=x.initial_state, lb=lb, prologue=prologue)
    assert_close(out, ro, dtype, f"{what} out")
    assert_close(fin, rs, dtype, f"{what} final_state")


@pytest.mark.parametrize("prologue", [QK, GATE, QK | GATE])
def test_prologue_tensor_core(kda, prologue):
    """bf16 d=128: ragged chunks, an empty sequence and a multi-segment sequence."""
    x = _inputs([130, 0, 64, 2100, 1], 2, 128, torch.bfloat16, 401, prologue)
    _check(kda, x, torch.bfloat16, prologue, f"tc prologue={prologue}")


def test_prologue_tensor_core_many_heads_lb(kda):
    """Single-segment schedule, and a lower bound other than -1 (lb scales the gate)."""
    x = _inputs([700, 333], 16, 128, torch.bfloat16, 402, QK | GATE)
    _check(kda, x, torch.bfloat16, QK | GATE, "tc H=16 lb=-0.5", lb=-0.5)


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.float32, 128),
                                     (torch.bfloat16, 64)])
def test_prologue_cuda_core(kda, dtype, d):
    x = _inputs([200, 0, 65], 2, d, dtype, 403, QK | GATE)
    _check(kda, x, dtype, QK | GATE, f"simt {dtype} d={d}")


def test_prologue_zero_rows(kda):
    """All-zero q or k rows stay zero (the norm is floored at 1e-12), as in the oracle."""
    x = _inputs([150], 2, 128, torch.bfloat16, 404, QK | GATE)
    x.q[5:9] = 0
    x.k[70:72] = 0
    _check(kda, x, torch.bfloat16, QK | GATE, "zero rows")


def test_prologue_snapshots(kda):
    x = _inputs([600, 200], 2, 128, torch.bfloat16, 405, QK | GATE)
    P = 128
    _, fin, snaps = kda.chunk_fwd_snapshots(
        *(t.to(DEV) for t in (x.q, x.k, x.v, x.g, x.beta)), snapshot_chunks=2,
        initial_state=x.initial_state.to(DEV), cu_seqlens=x.cu_seqlens.to(DEV),
        max_seqlen=600, prologue=QK | GATE)
    torch.cuda.synchronize()
    cu = x.cu_seqlens.tolist()
    _, rs, rsnap, first = ko.recurrent_snapshots(
        x.q, x.k, x.v, x.g, x.beta, snapshot_tokens=P, cu_seqlens=cu,
        initial_state=x.initial_state, prologue=QK | GATE)
    assert_close(fin, rs, torch.bfloat16, "prologue snapshots final_state")
    lib_idx = [cu[n] // P + m for n in range(2) for m in range((cu[n + 1] - cu[n]) // P)]
    assert_close(snaps[lib_idx], rsnap, torch.bfloat16, "prologue snapshots")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_prologue_decode(kda, dtype):
    """Chained decode steps on raw tokens equal the oracle's prologue recurrence."""
    N, H, d, steps = 8, 4, 128, 12
    S0 = decode_state(N, H, d, d, seed=3, device=DEV)
    tok = decode_tokens(steps, N, H, d, d, dtype=dtype, seed=4, device=DEV, raw=True)
    state = S0.clone()
    outs = [kda.decode_step(tok.q[t], tok.k[t], tok.v[t], tok.g[t], tok.beta[t], state,
                            prologue=QK | GATE) for t in range(steps)]
    torch.cuda.synchronize()
    perm = torch.tensor([t * N + n for n in range(N) for t in range(steps)])

    def pack(a):
        return a.reshape(steps * N, *a.shape[2:])[perm.to(a.device)].cpu()
    ro, rs = ko.recurrent(pack(tok.q), pack(tok.k), pack(tok.v), pack(tok.g), pack(tok.beta),
                          cu_seqlens=[n * steps for n in range(N + 1)], initial_state=S0.cpu(),
                          prologue=QK | GATE)
    got = torch.stack(outs).reshape(steps * N, H, d)[perm.to(DEV)]
    assert_close(got, ro, dtype, "prologue decode out")
    assert_close(state, rs, dtype, "prologue decode state")
