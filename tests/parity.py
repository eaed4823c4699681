"""Comparison helpers shared by the GPU parity tests (no method arithmetic here)."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances: fp32 inputs -> relative L2 <= 1e-4; bf16 inputs with fp32 state ->
# relative L2 <= 5e-3 and max-abs <= 3e-2, on outputs and on final states.
TOL = {
    torch.float32: dict(rel_l2=1e-4, max_abs=None),
    torch.bfloat16: dict(rel_l2=5e-3, max_abs=3e-2),
}


def to_f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def errors(got, ref) -> tuple[float, float]:
    g = to_f64(got)
    r = to_f64(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), "non-finite values in GPU result"
    rel = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30))
    mx = float(np.max(np.abs(g - r))) if g.size else 0.0
    return rel, mx


def assert_close(got, ref, dtype: torch.dtype, what: str = ""):
    rel, mx = errors(got, ref)
    tol = TOL[dtype]
    assert rel <= tol["rel_l2"], f"{what}: rel-L2 {rel:.3e} > {tol['rel_l2']:.0e} (max-abs {mx:.3e})"
    if tol["max_abs"] is not None:
        assert mx <= tol["max_abs"], f"{what}: max-abs {mx:.3e} > {tol['max_abs']:.0e}"
    return rel, mx
