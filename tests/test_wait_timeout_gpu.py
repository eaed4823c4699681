"""GPU test of the tensor-core prefill's bounded waits running out.

Every mbarrier wait in the tensor-core kernels has a limit; when one runs out the CTA records
KDA_ERR_DEVICE (device code 2) in the workspace status word, lets its own copies and
products in flight finish, frees its tensor memory and returns. The test-only build
libkda_shortwait.so points the first wait on the inputs of the intra-chunk kernel (its TMA
loads) and of each walk (its first stage) at a spare mbarrier that nothing arrives at, with a
limit of 64 clocks, so it always runs out however fast the real copies land; every other wait
keeps its limit (a walk that failed tells the CTAs waiting for its state
hand-off that it is not coming). A prefill through it must
return with the status word set and no fault, and afterwards the regular library's prefill
on the same device must still match the oracle.
"""
from __future__ import annotations

import ctypes
import os
import time

import pytest
import torch

from kimi_delta_attention_19_b200.inputs import make_inputs
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


@pytest.mark.timeout(300)
@pytest.mark.parametrize("T,H", [(64, 1), (3000, 2), (2048, 37)])
def test_first_wait_running_out_is_reported_and_context_stays_usable(kda, T, H):
    """(64, 1): one chunk of one head (intra-chunk kernel and one output walk);
    (3000, 2): twelve segments per head (summary walks, combine steps, later output walks);
    (2048, 37): the streamed schedule (the walks wait for tiles that never come)."""
    from kimi_delta_attention_19_b200 import build as kbuild
    assert os.path.exists(kbuild.SHORTWAIT_LIB), "build() makes the short-wait variant"
    short = kda.load_library(kbuild.SHORTWAIT_LIB)
    x = make_inputs(T, H=H, dk=128, dv=128, dtype=torch.bfloat16, seed=600 + T,
                    state_std=0.02)
    q, k, v, g, b = (t.to(DEV) for t in (x.q, x.k, x.v, x.g, x.beta))
    s0 = x.initial_state.to(DEV)
    shape = kda.make_shape(T, H, 128, 128, torch.bfloat16)
    ws = kda.alloc_workspace(shape, DEV)
    out = torch.empty_like(v)
    fin = torch.empty_like(s0)
    P = ctypes.c_void_p
    t0 = time.time()
    rc = short.kda_chunk_fwd(*(P(t.data_ptr()) for t in (q, k, v, g, b, s0)), None,
                             P(out.data_ptr()), P(fin.data_ptr()), ctypes.byref(shape),
                             P(ws.data_ptr()), ws.numel(),
                             P(torch.cuda.current_stream().cuda_stream))
    assert rc == kda.KDA_OK
    status, code = kda.workspace_status(ws)  # synchronises
    elapsed = time.time() - t0
    assert (status, code) == (kda.KDA_ERR_DEVICE, 2), (status, code)
    assert elapsed < 60, elapsed  # every wait that the first one's failure leaves is bounded
    # the context is still usable: the regular library on the same device, same workspace
    out2, fin2 = kda.chunk_fwd(q, k, v, g, b, initial_state=s0, workspace=ws)
    torch.cuda.synchronize()
    assert kda.workspace_status(ws) == (kda.KDA_OK, 0)
    ro, rs = ko.recurrent(x.q, x.k, x.v, x.g, x.beta, initial_state=x.initial_state)
    assert_close(out2, ro, torch.bfloat16, "out after the timed-out call")
    assert_close(fin2, rs, torch.bfloat16, "final_state after the timed-out call")
