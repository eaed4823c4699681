"""CPU tests of the C ABI: the library loads, exports what include/kda.h declares,
and rejects bad arguments before anything is launched (no GPU needed)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kda():
    from kimi_delta_attention_19_b200 import kda as k
    return k


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        with open(os.path.join(ROOT, "include", fn)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names.update(re.findall(r"\b(kda_\w+)\s*\(", text))
    return names


def test_exports_every_declared_symbol(kda):
    declared = _declared_functions()
    assert declared, "no declarations found in include/"
    for name in declared:
        assert hasattr(kda.lib, name), f"libkda.so does not export {name}"
    assert set(kda.EXPORTED) <= declared


def test_status_strings(kda):
    for code in range(5):
        s = kda.lib.kda_status_string(code).decode()
        assert s.startswith("KDA_")
    assert kda.lib.kda_status_string(99).decode() == "KDA_ERR_UNKNOWN"
    assert kda.lib.kda_version().decode().count(".") == 2


def test_workspace_size_is_pure_and_rejects_bad_shapes(kda):
    s = kda.make_shape(8192, 32, 128, 128, torch.bfloat16)
    n1 = kda.workspace_size(s)
    assert n1 > 0 and n1 % 256 == 0
    assert kda.workspace_size(s) == n1
    for bad in (dict(dk=96), dict(dv=32), dict(chunk=32), dict(lb=0.0), dict(lb=-2.0),
                dict(H=0)):
        kw = dict(T=8192, H=32, dk=128, dv=128, dtype=torch.bfloat16)
        kw.update({k: v for k, v in bad.items() if k in kw})
        extra = {k: v for k, v in bad.items() if k not in kw}
        sh = kda.make_shape(kw["T"], kw["H"], kw["dk"], kw["dv"], kw["dtype"], **extra)
        assert kda.workspace_size(sh) == 0, bad


def _fwd(kda, shape, ptrs=None, ws=(1 << 12) * 256, ws_ptr=256 * 1000):
    P = ctypes.c_void_p
    p = dict(q=4096, k=4096, v=4096, g=4096, beta=4096, s0=None, cu=None, out=4096, sT=None)
    if ptrs:
        p.update(ptrs)
    return kda.lib.kda_chunk_fwd(P(p["q"]), P(p["k"]), P(p["v"]), P(p["g"]), P(p["beta"]),
                                 P(p["s0"]), P(p["cu"]), P(p["out"]), P(p["sT"]),
                                 ctypes.byref(shape), P(ws_ptr), ws, None)


def test_chunk_fwd_argument_errors(kda):
    """Every case returns before any CUDA call (these addresses are never dereferenced)."""
    ok = kda.make_shape(128, 2, 64, 64, torch.float32)
    assert _fwd(kda, ok, {"q": None}) == kda.KDA_ERR_INVALID_ARG
    assert _fwd(kda, ok, {"k": 4100}) == kda.KDA_ERR_INVALID_ARG       # misaligned
    assert _fwd(kda, ok, ws=16) == kda.KDA_ERR_INVALID_ARG              # workspace too small
    assert _fwd(kda, ok, ws_ptr=256 * 1000 + 16) == kda.KDA_ERR_INVALID_ARG
    assert _fwd(kda, kda.make_shape(128, 2, 64, 48, torch.float32)) == kda.KDA_ERR_UNSUPPORTED
    assert _fwd(kda, kda.make_shape(128, 2, 64, 64, torch.float32, chunk=32)) == \
        kda.KDA_ERR_UNSUPPORTED
    assert _fwd(kda, kda.make_shape(128, 2, 64, 64, torch.float32, lb=-1.5)) == \
        kda.KDA_ERR_UNSUPPORTED                                          # lb*C < -80
    assert _fwd(kda, kda.make_shape(128, 2, 64, 64, torch.float32, lb=0.5)) == \
        kda.KDA_ERR_INVALID_ARG
    bad_b = kda.make_shape(128, 2, 64, 64, torch.float32, B=2, n_seqs=1)
    assert _fwd(kda, bad_b, {"cu": 4096}) == kda.KDA_ERR_INVALID_ARG    # cu_seqlens needs B=1
    assert _fwd(kda, kda.make_shape(128, 2, 64, 64, torch.float32, prologue=4)) == \
        kda.KDA_ERR_INVALID_ARG                                          # unknown prologue bit
    assert kda.workspace_size(kda.make_shape(128, 2, 64, 64, torch.float32, prologue=8)) == 0
    assert kda.workspace_size(kda.make_shape(128, 2, 64, 64, torch.float32, prologue=3)) > 0
    no_n = kda.make_shape(128, 2, 64, 64, torch.float32, n_seqs=0)
    assert _fwd(kda, no_n, {"cu": 4096}) == kda.KDA_ERR_INVALID_ARG
    assert kda.lib.kda_chunk_fwd(None, None, None, None, None, None, None, None, None, None,
                                 None, 0, None) == kda.KDA_ERR_INVALID_ARG


def test_snapshot_count_and_argument_errors(kda):
    """Snapshot capacity is floor(T_total / (k * 64)); bad snapshot arguments return before
    any CUDA call (the addresses are never dereferenced)."""
    P = ctypes.c_void_p
    sh = kda.make_shape(1000, 2, 64, 64, torch.float32, B=3)
    assert kda.snapshot_count(sh, 1) == 3000 // 64
    assert kda.snapshot_count(sh, 4) == 3000 // 256
    assert kda.snapshot_count(sh, 0) == -1
    assert kda.snapshot_count(kda.make_shape(1000, 2, 64, 48, torch.float32), 1) == -1
    packed = kda.make_shape(700, 2, 64, 64, torch.float32, n_seqs=3)
    assert kda.snapshot_count(packed, 2) == 700 // 128

    def call(k_chunks=1, snaps=8192, n_snaps=46, shape=sh, q=4096):
        return kda.lib.kda_chunk_fwd_snapshots(
            P(q), P(4096), P(4096), P(4096), P(4096), None, None, P(4096), None, k_chunks,
            P(snaps), n_snaps, ctypes.byref(shape), P(256 * 1000), 1 << 20, None)

    assert call(k_chunks=0) == kda.KDA_ERR_INVALID_ARG
    assert call(n_snaps=45) == kda.KDA_ERR_INVALID_ARG          # one slot short
    assert call(snaps=None) == kda.KDA_ERR_INVALID_ARG          # snapshots needed
    assert call(snaps=8200) == kda.KDA_ERR_INVALID_ARG          # misaligned
    assert call(q=None) == kda.KDA_ERR_INVALID_ARG
    assert call(shape=kda.make_shape(1000, 2, 64, 48, torch.float32, B=3)) == \
        kda.KDA_ERR_UNSUPPORTED


def test_backward_workspace_and_argument_errors(kda):
    """kda_chunk_bwd: workspace size is pure and larger than the forward's; bad arguments
    return before any CUDA call (the addresses are never dereferenced)."""
    P = ctypes.c_void_p
    sh = kda.make_shape(1000, 2, 64, 64, torch.float32, B=3)
    nb = int(kda.lib.kda_chunk_bwd_workspace_size(ctypes.byref(sh)))
    assert nb > kda.workspace_size(sh) and nb % 256 == 0
    assert int(kda.lib.kda_chunk_bwd_workspace_size(ctypes.byref(sh))) == nb
    bad = kda.make_shape(1000, 2, 64, 48, torch.float32, B=3)
    assert int(kda.lib.kda_chunk_bwd_workspace_size(ctypes.byref(bad))) == 0
    pro = kda.make_shape(1000, 2, 64, 64, torch.float32, B=3, prologue=3)
    assert int(kda.lib.kda_chunk_bwd_workspace_size(ctypes.byref(pro))) == nb

    def call(shape=sh, q=4096, dq=4096, dstate=None, ws=256 * 1000, wsb=nb):
        return kda.lib.kda_chunk_bwd(P(q), P(4096), P(4096), P(4096), P(4096), None, None,
                                     P(4096), None, P(dq), P(4096), P(4096), P(4096), P(4096),
                                     P(dstate), ctypes.byref(shape), P(ws), wsb, None)

    assert call(q=None) == kda.KDA_ERR_INVALID_ARG
    assert call(dq=None) == kda.KDA_ERR_INVALID_ARG
    assert call(dq=4100) == kda.KDA_ERR_INVALID_ARG            # misaligned gradient
    assert call(dstate=4104) == kda.KDA_ERR_INVALID_ARG        # misaligned d_initial_state
    assert call(wsb=nb - 256) == kda.KDA_ERR_INVALID_ARG       # workspace one step short
    assert call(ws=256 * 1000 + 16) == kda.KDA_ERR_INVALID_ARG
    assert call(shape=bad) == kda.KDA_ERR_UNSUPPORTED
    assert call(shape=kda.make_shape(1000, 2, 64, 64, torch.float32, B=3, prologue=4)) == \
        kda.KDA_ERR_INVALID_ARG


def test_decode_argument_errors(kda):
    P = ctypes.c_void_p
    sh = kda.make_shape(1, 4, 128, 128, torch.bfloat16, B=8)

    def call(state=4096, slots=None, n_slots=8, shape=sh, q=4096, status=None):
        return kda.lib.kda_decode_step(P(q), P(4096), P(4096), P(4096), P(4096), P(state),
                                       P(slots), n_slots, P(4096), ctypes.byref(shape),
                                       P(status), None)

    assert call(state=None) == kda.KDA_ERR_INVALID_ARG
    assert call(n_slots=4) == kda.KDA_ERR_INVALID_ARG          # fewer slots than sequences
    assert call(q=4097) == kda.KDA_ERR_INVALID_ARG
    assert call(slots=4098) == kda.KDA_ERR_INVALID_ARG         # int32 slots misaligned
    assert call(status=4098) == kda.KDA_ERR_INVALID_ARG        # int32 status misaligned
    assert call(shape=kda.make_shape(2, 4, 128, 128, torch.bfloat16, B=8)) == \
        kda.KDA_ERR_INVALID_ARG                                 # decode is one token
    assert call(shape=kda.make_shape(1, 4, 128, 80, torch.bfloat16, B=8)) == \
        kda.KDA_ERR_UNSUPPORTED
    assert call(shape=kda.make_shape(1, 4, 128, 128, torch.bfloat16, B=8, prologue=-1)) == \
        kda.KDA_ERR_INVALID_ARG


def test_binding_rejects_non_contiguous_tensors(kda):
    """A strided view would be read as the wrong memory: the binding refuses it before any
    library call."""
    q = torch.zeros(8, 2, 64).transpose(0, 1)
    with pytest.raises(ValueError, match="contiguous"):
        kda._ptr(q)
    assert kda._ptr(None) is None
    assert kda._ptr(torch.zeros(4, 4)).value is not None


def test_autograd_plumbing_with_stand_in_calls(kda, monkeypatch):
    """kda_attention's autograd wiring on CPU, with stand-ins for the two library calls:
    the options reach both calls, dL/dout and dL/dfinal_state reach the backward call, and
    its six gradients come back to the right inputs (dS0 only when asked for)."""
    seen = {}

    def fwd(q, k, v, g, beta, **kw):
        seen["fwd"] = kw
        return torch.zeros(v.shape), torch.zeros(1, q.shape[1], q.shape[2], v.shape[2])

    def bwd(q, k, v, g, beta, d_out, **kw):
        seen["bwd"] = (d_out.clone(), kw)
        ds0 = torch.full((1, q.shape[1], q.shape[2], v.shape[2]), 6.0)
        return (torch.full_like(q, 1.0), torch.full_like(k, 2.0), torch.full_like(v, 3.0),
                torch.full_like(g, 4.0), torch.full_like(beta, 5.0),
                ds0 if kw["want_d_initial"] else None)

    monkeypatch.setattr(kda, "chunk_fwd", fwd)
    monkeypatch.setattr(kda, "chunk_bwd", bwd)
    q, k, g = (torch.randn(10, 2, 4, requires_grad=True) for _ in range(3))
    v = torch.randn(10, 2, 3, requires_grad=True)
    b = torch.rand(10, 2, requires_grad=True)
    s0 = torch.randn(1, 2, 4, 3, requires_grad=True)
    out, fin = kda.kda_attention(q, k, v, g, b, initial_state=s0, scale=0.3, lb=-0.5,
                                 prologue=1)
    (2.0 * out.sum() + 3.0 * fin.sum()).backward()
    assert seen["fwd"]["scale"] == 0.3 and seen["fwd"]["lb"] == -0.5
    assert seen["fwd"]["prologue"] == 1
    d_out, kw = seen["bwd"]
    assert torch.equal(d_out, torch.full((10, 2, 3), 2.0))
    assert torch.equal(kw["d_final_state"], torch.full((1, 2, 4, 3), 3.0))
    assert kw["want_d_initial"] and kw["initial_state"] is not None and kw["prologue"] == 1
    for t, val in ((q, 1.0), (k, 2.0), (v, 3.0), (g, 4.0), (b, 5.0), (s0, 6.0)):
        assert torch.equal(t.grad, torch.full_like(t, val))
    # no initial state: no dS0 asked for
    out, fin = kda.kda_attention(q, k, v, g, b)
    out.sum().backward()
    assert not seen["bwd"][1]["want_d_initial"]


def test_binding_refuses_without_library(tmp_path, monkeypatch):
    """With libkda.so absent the binding raises instead of falling back."""
    import importlib.util
    src = os.path.join(ROOT, "kimi_delta_attention_19_b200", "kda.py")
    spec = importlib.util.spec_from_file_location("kda_copy", str(tmp_path / "kda.py"))
    with open(src) as f:
        (tmp_path / "kda.py").write_text(f.read())
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)
