"""GPU test of kda_chunk_fwd_noalloc, the prefill entry point for callers that
cannot allocate device memory (graph capture, plugin hosts without a workspace,
serving loops that must not synchronise on an allocation).

It is checked against the regular kda_chunk_fwd (caller workspace) on the same
inputs, for two calls in a row, because the fixed scratch array keeps the
previous call's contents. The file name sorts last so that a run stopping at the
first failure has already run every other test.
"""
from __future__ import annotations

import pytest
import torch

from kimi_delta_attention_19_b200.inputs import make_inputs
from tests.parity import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def kda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kimi_delta_attention_19_b200 import kda as k
    return k


def _both(kda, x):
    args = [t.to(DEV) for t in (x.q, x.k, x.v, x.g, x.beta)]
    s0 = None if x.initial_state is None else x.initial_state.to(DEV)
    cu = None if x.cu_seqlens is None else x.cu_seqlens.to(DEV)
    n = len(x.lengths)
    ref_out, ref_fin = kda.chunk_fwd(*args, initial_state=s0, cu_seqlens=cu,
                                     max_seqlen=max(x.lengths))
    out = torch.full_like(ref_out, float("nan"))
    fin = torch.full((n, *ref_fin.shape[1:]), float("nan"), device=DEV)
    kda.chunk_fwd_noalloc(*args, out=out, final_state=fin, initial_state=s0, cu_seqlens=cu,
                          max_seqlen=max(x.lengths))
    torch.cuda.synchronize()
    return (out, fin), (ref_out, ref_fin)


def test_noalloc_matches_workspace_entry_point_twice(kda):
    calls = [
        make_inputs(None, H=4, dk=128, dv=128, dtype=torch.bfloat16, seed=91,
                    lengths=[700, 1, 0, 1500], state_std=0.02),
        make_inputs(None, H=2, dk=128, dv=128, dtype=torch.bfloat16, seed=92,
                    lengths=[65, 2100], state_std=0.02),
    ]
    for i, x in enumerate(calls):
        (out, fin), (ref_out, ref_fin) = _both(kda, x)
        assert_close(out, ref_out.float(), torch.bfloat16, f"call {i} out")
        assert_close(fin, ref_fin, torch.bfloat16, f"call {i} final_state")


def test_noalloc_fp32_inputs(kda):
    x = make_inputs(300, H=2, dk=64, dv=64, dtype=torch.float32, seed=93, state_std=0.02)
    (out, fin), (ref_out, ref_fin) = _both(kda, x)
    assert_close(out, ref_out, torch.float32, "fp32 out")
    assert_close(fin, ref_fin, torch.float32, "fp32 final_state")


def test_noalloc_rejects_shapes_beyond_its_scratch(kda):
    big = None
    # packed sequences without a max_seqlen bound: scratch is sized for the worst case
    for T, H, n in ((1 << 19, 32, 64), (1 << 20, 16, 1), (1 << 22, 64, 0)):
        sh = kda.make_shape(T, H, 128, 128, torch.bfloat16, n_seqs=n)
        if kda.workspace_size(sh) > kda.NOALLOC_SCRATCH_BYTES:
            big = (T, H, n)
            break
    if big is None:
        pytest.skip("no supported shape needs more scratch than the fixed array")
    T, H, n = big
    x = torch.empty(16, device=DEV)  # never read: the size check comes first
    with pytest.raises(kda.KdaError) as e:
        lib_shape = kda.make_shape(T, H, 128, 128, torch.bfloat16, n_seqs=n)
        import ctypes
        rc = kda.lib.kda_chunk_fwd_noalloc(*([ctypes.c_void_p(x.data_ptr())] * 5), None, None,
                                           ctypes.c_void_p(x.data_ptr()), None,
                                           ctypes.byref(lib_shape), None)
        if rc != kda.KDA_OK:
            raise kda.KdaError(rc, "kda_chunk_fwd_noalloc")
    assert e.value.status == kda.KDA_ERR_UNSUPPORTED
