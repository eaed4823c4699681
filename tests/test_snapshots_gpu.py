"""GPU parity of the chunk-boundary state snapshots (prefix cache) against the fp64
oracle, through kda_chunk_fwd_snapshots.

Snapshot m of sequence n is the state after its first m * k * 64 tokens; the library
stores it at index c_n // (k * 64) + m - 1 (c_n: the sequence's first packed token).
Checked here: the values (against the oracle's recorded states), the index layout
(unreached indices keep their sentinel), that recording changes neither the outputs
nor the final states, and that a prefill resumed from a snapshot continues the
sequence exactly as the full prefill does.
"""
from __future__ import annotations

import pytest
import torch

from kimi_delta_attention_19_b200.inputs import WORKLOADS, make_inputs, workload_inputs
from oracle import kda_oracle as ko
from tests.parity import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def kda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kimi_delta_attention_19_b200 import kda as k
    return k


def _cu(x):
    if x.cu_seqlens is not None:
        return [int(c) for c in x.cu_seqlens.tolist()]
    return [0, x.q.shape[0]]


def _check_snapshots(kda, x, dtype, kchunks, what, max_seqlen=0, batch=None):
    """Snapshots of one call against the oracle; returns the snapshot tensor."""
    P = 64 * kchunks
    cu = _cu(x)
    T_total = cu[-1]
    args = [t.to(DEV) for t in (x.q, x.k, x.v, x.g, x.beta)]
    kw = dict(initial_state=None if x.initial_state is None else x.initial_state.to(DEV))
    if batch is None:
        kw.update(cu_seqlens=None if x.cu_seqlens is None else x.cu_seqlens.to(DEV),
                  max_seqlen=max_seqlen)
    else:  # B equal sequences in the [B, T, H, d] layout, no cu_seqlens
        args = [a.view(batch, T_total // batch, *a.shape[1:]) for a in args]
    count = T_total // P
    snaps = torch.full((count, x.q.shape[1], x.q.shape[2], x.v.shape[2]), float("nan"),
                       device=DEV)
    out, fin, snaps = kda.chunk_fwd_snapshots(*args, snapshot_chunks=kchunks, snapshots=snaps,
                                              **kw)
    out0, fin0 = kda.chunk_fwd(*args, **kw)
    torch.cuda.synchronize()
    # recording the snapshots changes nothing else
    assert torch.equal(out, out0) and torch.equal(fin, fin0), what

    _, rs, rsnap, first = ko.recurrent_snapshots(
        x.q, x.k, x.v, x.g, x.beta, snapshot_tokens=P, cu_seqlens=cu,
        initial_state=x.initial_state)
    assert_close(fin, rs, dtype, f"{what} final_state")
    lib_idx, ref_idx = [], []
    for n in range(len(cu) - 1):
        for m in range(1, (cu[n + 1] - cu[n]) // P + 1):
            lib_idx.append(cu[n] // P + m - 1)
            ref_idx.append(int(first[n]) + m - 1)
    assert len(set(lib_idx)) == len(lib_idx) and all(0 <= i < count for i in lib_idx)
    if lib_idx:
        assert_close(snaps[lib_idx], rsnap[ref_idx], dtype, f"{what} snapshots")
    untouched = sorted(set(range(count)) - set(lib_idx))
    if untouched:
        assert torch.isnan(snaps[untouched]).all(), f"{what}: an unreached index was written"
    return snaps


@pytest.mark.parametrize("kchunks", [1, 3])
def test_snapshots_tensor_core_segments(kda, kchunks):
    """bf16 d=128 (tensor-core path) with 1, 2, 3 and many segments per sequence:
    snapshots come from every segment's output walk."""
    lengths = [320, 577, 0, 3000, 64, 130]
    x = make_inputs(None, H=2, dk=128, dv=128, dtype=torch.bfloat16, seed=301,
                    lengths=lengths, state_std=0.02)
    _check_snapshots(kda, x, torch.bfloat16, kchunks, f"tc k={kchunks}",
                     max_seqlen=max(lengths))


def test_snapshots_tensor_core_many_heads(kda):
    """Single-segment schedule (many heads) with ragged tails."""
    x = make_inputs(None, H=32, dk=128, dv=128, dtype=torch.bfloat16, seed=302,
                    lengths=[700, 129, 1024, 63], state_std=0.02)
    _check_snapshots(kda, x, torch.bfloat16, 2, "tc H=32", max_seqlen=1024)


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.float32, 128),
                                     (torch.bfloat16, 64)])
def test_snapshots_cuda_core(kda, dtype, d):
    """fp32 inputs and d=64 heads (CUDA-core path)."""
    x = make_inputs(None, H=2, dk=d, dv=d, dtype=dtype, seed=303 + d,
                    lengths=[200, 0, 64, 333], state_std=0.02)
    _check_snapshots(kda, x, dtype, 1, f"simt {dtype} d={d}", max_seqlen=333)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_snapshots_batched_layout(kda, dtype, d):
    """[B, T, H, d] inputs: sequence n starts at c_n = n T, so its first snapshot sits at
    n T // (k 64), with gaps when T is not a multiple of the interval."""
    x = make_inputs(200, H=2, dk=d, dv=d, dtype=dtype, seed=305, batch=3, state_std=0.02)
    _check_snapshots(kda, x, dtype, 1, f"batched {dtype}", batch=3)


def test_snapshot_interval_longer_than_sequences(kda):
    """No sequence reaches the interval: zero slots, nothing written, results unchanged."""
    x = make_inputs(None, H=2, dk=128, dv=128, dtype=torch.bfloat16, seed=306,
                    lengths=[100, 60], state_std=0.02)
    _check_snapshots(kda, x, torch.bfloat16, 4, "long interval", max_seqlen=100)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_resume_from_snapshot(kda, dtype, d):
    """Prefix-cache reuse: the suffix of a sequence prefilled from snapshot m gives the
    outputs and final state of the whole-sequence prefill (against the oracle)."""
    T, kchunks = 1500, 4
    x = make_inputs(T, H=2, dk=d, dv=d, dtype=dtype, seed=307, state_std=0.02)
    ro, rs = ko.recurrent(x.q, x.k, x.v, x.g, x.beta, initial_state=x.initial_state)
    dev = [t.to(DEV) for t in (x.q, x.k, x.v, x.g, x.beta)]
    _, _, snaps = kda.chunk_fwd_snapshots(*dev, snapshot_chunks=kchunks,
                                          initial_state=x.initial_state.to(DEV))
    P = 64 * kchunks
    assert snaps.shape[0] == T // P
    for m in (1, T // P):
        t0 = m * P
        sl = [t[t0:] for t in dev]
        out, fin = kda.chunk_fwd(*sl, initial_state=snaps[m - 1:m].contiguous())
        torch.cuda.synchronize()
        assert_close(out, ro[t0:], dtype, f"resume at {t0} out")
        assert_close(fin, rs, dtype, f"resume at {t0} final_state")


def test_full_bf16_h32_t8192_d128_snapshots(kda):
    """The 8K-token, 32-head workload with a snapshot every 1024 tokens."""
    x = workload_inputs(WORKLOADS["bf16_h32_t8192_d128"])
    _check_snapshots(kda, x, torch.bfloat16, 16, "8K snapshots")
