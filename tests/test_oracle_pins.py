"""CPU tests: the fp64 oracle against its pins, and the pins against planted mistakes."""
from __future__ import annotations

import multiprocessing as mp
import os
import subprocess
import tempfile

import pytest

from oracle import kda_oracle as ko
from tests import oracle_pins as pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(oracle, pin):
    pin(oracle.load())


def test_chunked_oracle_hand_example():
    """The chunked form on its own reproduces the two-token hand example."""
    import numpy as np
    import torch
    q = torch.tensor([[[1.0]], [[1.0]]])
    k = torch.tensor([[[1.0]], [[-1.0]]])
    v = torch.tensor([[[4.0]], [[0.0]]])
    g = torch.full((2, 1, 1), float(np.log(0.5)))
    b = torch.tensor([[0.5], [0.5]])
    o, s = ko.chunked(q, k, v, g, b, chunk=2, initial_state=np.array([[[[2.0]]]]), scale=1.0)
    assert np.allclose(o[:, 0, 0], [2.5, 0.625], rtol=1e-6)
    assert np.allclose(s[0, 0], [[0.625]], rtol=1e-6)


# Plausible slips, each planted in a copy of the oracle source. Every one must
# be caught by at least one pin, or the pins are too weak to trust the oracle.
MUTANTS = {
    "drop_decay": ("S[i * dv + j] *= decay[i];", ";"),
    "decay_sign": ("decay[i] = exp(gi);", "decay[i] = exp(-gi);"),
    "no_clamp": ("if (gi < J->lb) gi = J->lb;", ";"),
    "erase_sign": ("(vt[j] - w[j])", "(vt[j] + w[j])"),
    "drop_erase": ("(vt[j] - w[j])", "(vt[j])"),
    "drop_beta": ("+= b * kt[i] * (vt[j] - w[j])", "+= kt[i] * (vt[j] - w[j])"),
    "recall_with_query": ("w[j] += kt[i] * S[i * dv + j];", "w[j] += qt[i] * S[i * dv + j];"),
    "no_scale": ("o[j] *= J->scale;", ";"),
    "read_before_write": (
        "        /* S <- S + beta k (v - w)^T */\n"
        "        for (int i = 0; i < dk; ++i)\n"
        "            for (int j = 0; j < dv; ++j) S[i * dv + j] += b * kt[i] * (vt[j] - w[j]);\n",
        ""),
    "transposed_readout": (
        "for (int j = 0; j < dv; ++j) o[j] += qt[i] * S[i * dv + j];",
        "for (int j = 0; j < dv && i < dv && j < dk; ++j) o[i] += qt[j] * S[i * dv + j];"),
    "decay_on_columns": ("S[i * dv + j] *= decay[i];", "S[i * dv + j] *= decay[j % dk];"),
    "snapshot_one_token_late": ("(t - t0 + 1) % J->snap_tokens == 0",
                                "(t - t0) % J->snap_tokens == 0 && t > t0"),
    "snapshot_wrong_sequence": ("J->snap_first[seq] +", "J->snap_first[0] +"),
    "l2norm_by_squared_norm": ("nk = sqrt(nk);", ";"),
    "l2norm_keys_only": ("qt[i] /= nq;", ";"),
    "gate_sign": ("gi = J->lb / (1.0 + exp(-gi));", "gi = J->lb / (1.0 + exp(gi));"),
    "gate_without_bound": ("gi = J->lb / (1.0 + exp(-gi));", "gi = -1.0 / (1.0 + exp(-gi));"),
    "bwd_clamp_mask_dropped": ("J->dg[tk + i] = graw[i] >= J->lb ? dgp[i] : 0.0;",
                               "J->dg[tk + i] = dgp[i];"),
    "bwd_dw_sign": ("dw[j] = -b * du[j];", "dw[j] = b * du[j];"),
    "bwd_state_grad_not_decayed": ("for (int j = 0; j < dv; ++j) dS[i * dv + j] *= decay[i];",
                                   ";"),
    "bwd_dq_from_decayed_prev_state": ("a += S[i * dv + j] * dov[j];",
                                       "a += Sb[i * dv + j] * dov[j];"),
    "bwd_dbeta_without_recall": ("db += du[j] * (vt[j] - w[j]);", "db += du[j] * vt[j];"),
    "bwd_l2norm_without_projection": ("J->dq[tk + i] = (J->dq[tk + i] - qt[i] * pq) / nq;",
                                      "J->dq[tk + i] = J->dq[tk + i] / nq;"),
    "bwd_gate_without_sigmoid_slope": (
        "J->dg[tk + i] *= J->lb * sig[i] * (1.0 - sig[i]);", "J->dg[tk + i] *= J->lb;"),
}


def _mutant_worker(path, q):
    q.put(pins.failing_pins(path))


def _run_isolated(path: str) -> list[str]:
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_mutant_worker, args=(path, q))
    p.start()
    p.join(600)
    if p.exitcode != 0:
        return ["<crashed>"]
    return q.get()


def test_pins_catch_planted_mistakes(tmp_path):
    with open(ko._SRC) as f:
        src = f.read()
    clean = tmp_path / "clean.so"
    ko.build(ko._SRC, str(clean))
    assert _run_isolated(str(clean)) == []
    survivors = []
    for name, (old, new) in MUTANTS.items():
        assert old in src, f"mutant {name}: pattern not found in oracle source"
        msrc = tmp_path / f"{name}.c"
        msrc.write_text(src.replace(old, new, 1))
        so = tmp_path / f"{name}.so"
        ko.build(str(msrc), str(so))
        caught = _run_isolated(str(so))
        if not caught:
            survivors.append(name)
    assert not survivors, f"pins missed planted mistakes: {survivors}"


def test_correlated_key_bound_catches_dropped_inverse_block(monkeypatch):
    """The GPU bound on the correlated-key inputs (rel-L2 1e-2) separates a correct blocked
    inverse from one that drops the off-diagonal block: the oracle's chunked form with that
    mistake planted (A_21 ignored in the 64-token solve) lands far outside the bound, while
    the unmodified chunked form agrees with the token-by-token recurrence."""
    import numpy as np
    from kimi_delta_attention_19_b200.inputs import correlated_key_inputs

    x = correlated_key_inputs(seed=19)
    cu = x.cu_seqlens.tolist()
    args = (x.q, x.k, x.v, x.g, x.beta)
    ro, rs = ko.recurrent(*args, cu_seqlens=cu, initial_state=x.initial_state, lb=-1.0)
    ro, rs = np.asarray(ro, np.float64), np.asarray(rs, np.float64)

    def rel(a, b):
        return float(np.linalg.norm(np.asarray(a) - b) / np.linalg.norm(b))

    co, cs = ko.chunked(*args, chunk=64, cu_seqlens=cu, initial_state=x.initial_state, lb=-1.0)
    assert rel(co, ro) < 1e-9 and rel(cs, rs) < 1e-9
    solve = ko._forward_substitution

    def without_off_diagonal(L, B):
        L2 = L.copy()
        L2[32:, :32] = 0.0
        return solve(L2, B)

    monkeypatch.setattr(ko, "_forward_substitution", without_off_diagonal)
    bo, bs = ko.chunked(*args, chunk=64, cu_seqlens=cu, initial_state=x.initial_state, lb=-1.0)
    assert rel(bo, ro) > 5e-2 and rel(bs, rs) > 5e-2, (rel(bo, ro), rel(bs, rs))
