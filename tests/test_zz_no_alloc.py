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
        # the same kernels on the same inputs, only the scratch differs: bit for bit
        assert torch.equal(out, ref_out), f"call {i} out differs from kda_chunk_fwd"
        assert torch.equal(fin, ref_fin), f"call {i} final_state differs from kda_chunk_fwd"
        assert kda.workspace_status(None) == (kda.KDA_OK, 0)


def test_noalloc_fp32_inputs(kda):
    x = make_inputs(300, H=2, dk=64, dv=64, dtype=torch.float32, seed=93, state_std=0.02)
    (out, fin), (ref_out, ref_fin) = _both(kda, x)
    assert_close(out, ref_out, torch.float32, "fp32 out")
    assert_close(fin, ref_fin, torch.float32, "fp32 final_state")
    assert torch.equal(out, ref_out) and torch.equal(fin, ref_fin)


def test_noalloc_reports_device_errors_in_its_status_word(kda):
    """A malformed cu_seqlens (only visible on the device) is recorded in the fixed
    array's status word, which workspace_status(None) reads; the next good call clears it."""
    x = make_inputs(200, H=2, dk=128, dv=128, dtype=torch.bfloat16, seed=94, state_std=None)
    args = [t.to(DEV) for t in (x.q, x.k, x.v, x.g, x.beta)]
    out = torch.empty_like(args[2])
    bad = torch.tensor([0, 100, 50, 200], dtype=torch.int32, device=DEV)
    kda.chunk_fwd_noalloc(*args, out=out, final_state=None, cu_seqlens=bad)
    rc, code = kda.workspace_status(None)
    assert rc == kda.KDA_ERR_DEVICE and code == 1
    kda.chunk_fwd_noalloc(*args, out=out, final_state=None)
    assert kda.workspace_status(None) == (kda.KDA_OK, 0)


def test_noalloc_in_a_second_context(kda):
    """The array's address belongs to the CUDA context that loaded the library's module.
    In a second context on the same device (made current with the driver API, inputs
    allocated there by the test) the entry point must look the address up again: its
    results equal kda_chunk_fwd's in the primary context, bit for bit, and afterwards the
    primary context's calls still do."""
    import ctypes

    import numpy as np
    from cuda.bindings import driver as cu

    x = make_inputs(None, H=2, dk=128, dv=128, dtype=torch.bfloat16, seed=95,
                    lengths=[300, 1, 129], state_std=0.02)
    (ref_out, ref_fin), _ = _both(kda, x)  # primary context, no-alloc path
    host = [t.contiguous() for t in (x.q, x.k, x.v, x.g, x.beta, x.initial_state,
                                     x.cu_seqlens)]

    def ok(r):
        err = r[0] if isinstance(r, tuple) else r
        assert err == cu.CUresult.CUDA_SUCCESS, err
        return r[1] if isinstance(r, tuple) and len(r) > 1 else None

    ok(cu.cuInit(0))
    dev = ok(cu.cuDeviceGet(torch.cuda.current_device()))
    ctx = ok(cu.cuCtxCreate(0, dev))  # current on this thread from here on
    bufs = []
    try:
        def dalloc(nbytes):
            p = ok(cu.cuMemAlloc(max(nbytes, 16)))
            bufs.append(p)
            return int(p)

        dptr = []
        for t in host:
            nb = t.numel() * t.element_size()
            p = dalloc(nb)
            ok(cu.cuMemcpyHtoD(p, t.data_ptr(), nb))
            dptr.append(p)
        out_nb = ref_out.numel() * ref_out.element_size()
        fin_nb = ref_fin.numel() * ref_fin.element_size()
        d_out, d_fin = dalloc(out_nb), dalloc(fin_nb)
        shape = kda.make_shape(host[0].shape[0], 2, 128, 128, torch.bfloat16,
                               n_seqs=len(x.lengths), max_seqlen=max(x.lengths))
        P = ctypes.c_void_p
        rc = kda.lib.kda_chunk_fwd_noalloc(*(P(p) for p in dptr), P(d_out), P(d_fin),
                                           ctypes.byref(shape), None)
        assert rc == kda.KDA_OK, rc
        ok(cu.cuCtxSynchronize())
        code = ctypes.c_int32(-1)
        assert kda.lib.kda_workspace_status(None, 0, None, ctypes.byref(code)) == kda.KDA_OK
        assert code.value == 0
        got_out = torch.empty(ref_out.shape, dtype=ref_out.dtype)
        got_fin = torch.empty(ref_fin.shape, dtype=ref_fin.dtype)
        ok(cu.cuMemcpyDtoH(got_out.data_ptr(), d_out, out_nb))
        ok(cu.cuMemcpyDtoH(got_fin.data_ptr(), d_fin, fin_nb))
    finally:
        for p in bufs:
            cu.cuMemFree(p)
        ok(cu.cuCtxDestroy(ctx))  # the primary context is current again
    assert torch.equal(got_out, ref_out.cpu()) and torch.equal(got_fin, ref_fin.cpu())
    # back in the primary context: its cached address is found again and still valid
    (out2, fin2), _ = _both(kda, x)
    assert torch.equal(out2, ref_out) and torch.equal(fin2, ref_fin)
    assert np.isfinite(got_out.float().numpy()).all()


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
