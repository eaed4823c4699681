"""Pins for the fp64 KDA oracle: facts fixed by the pages and by the mathematics.

Each pin takes the oracle library handle (so the same checks can run against
deliberately broken builds of the oracle) and raises AssertionError on failure.

None of these re-types the oracle's loop. They check it against:
  * hand-worked examples (tests/golden/kda_hand_examples.json);
  * an independently derived chunked closed form (oracle.kda_oracle.chunked);
  * closed forms: beta = 0 pure decay, the delta-rule reach identity, the
    associative-memory recall with orthonormal keys, the one-token expansion;
  * invariants: linearity in (V, S0), the contraction bound, resume/split,
    packed varlen == separate runs, decode == prefill, the decay clamp.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

from kimi_delta_attention_19_b200.inputs import make_inputs
from oracle import kda_oracle as ko

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "kda_hand_examples.json")


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _f32(x):
    return torch.tensor(np.asarray(x, dtype=np.float32))


# --------------------------------------------------------------------------
def pin_golden(lib):
    """Hand-worked examples (decay placement, erase sign, read-out orientation, clamp)."""
    with open(GOLDEN) as f:
        ex = json.load(f)["examples"]
    for e in ex:
        toks = e["tokens"]
        T = len(toks)
        q = _f32([[t["q"]] for t in toks])
        k = _f32([[t["k"]] for t in toks])
        v = _f32([[t["v"]] for t in toks])
        g = _f32([[t["g"]] for t in toks])
        b = _f32([[t["beta"]] for t in toks])
        s0 = np.asarray(e["S0"], dtype=np.float64)[None, None]
        out, fin = ko.recurrent(q, k, v, g, b, initial_state=s0, lb=e["lb"], scale=e["scale"],
                                lib=lib)
        exp_out = np.asarray(e["expected_out"], dtype=np.float64)
        exp_fin = np.asarray(e["expected_final_state"], dtype=np.float64)
        assert out.shape == (T, 1, e["dv"])
        assert np.allclose(out[:, 0], exp_out, rtol=1e-6, atol=1e-7), (e["name"], out[:, 0], exp_out)
        assert np.allclose(fin[0, 0], exp_fin, rtol=1e-6, atol=1e-7), (e["name"], fin[0, 0], exp_fin)


def pin_chunked_agreement(lib):
    """Recurrent == independently derived chunked form for C in {1, 7, 16, 64, T}."""
    lengths = [37, 0, 1, 64, 130]
    x = make_inputs(None, H=2, dk=16, dv=12, dtype=torch.float32, seed=3, lengths=lengths,
                    g_scale=1.0, state_std=0.3)
    cu = x.cu_seqlens.tolist()
    ref_o, ref_s = ko.recurrent(x.q, x.k, x.v, x.g, x.beta, cu_seqlens=cu,
                                initial_state=x.initial_state, lib=lib)
    for C in (1, 7, 16, 64, max(lengths)):
        o, s = ko.chunked(x.q, x.k, x.v, x.g, x.beta, chunk=C, cu_seqlens=cu,
                          initial_state=x.initial_state)
        assert _rel(ref_o, o) < 1e-11, (C, _rel(ref_o, o))
        assert _rel(ref_s, s) < 1e-11, (C, _rel(ref_s, s))
    # bf16 inputs take the same route through the widening step
    xb = make_inputs(70, H=3, dk=8, dv=8, dtype=torch.bfloat16, seed=4, state_std=0.1)
    o1, s1 = ko.recurrent(xb.q, xb.k, xb.v, xb.g, xb.beta, initial_state=xb.initial_state, lib=lib)
    o2, s2 = ko.chunked(xb.q, xb.k, xb.v, xb.g, xb.beta, chunk=16, initial_state=xb.initial_state)
    assert _rel(o1, o2) < 1e-11 and _rel(s1, s2) < 1e-11


def pin_beta_zero_pure_decay(lib):
    """beta = 0: S_t = Diag(exp sum g') S0 and o_t = scale (exp(G_t) * q_t)^T S0."""
    x = make_inputs(23, H=2, dk=8, dv=5, dtype=torch.float32, seed=5, state_std=1.0)
    beta = torch.zeros_like(x.beta)
    out, fin = ko.recurrent(x.q, x.k, x.v, x.g, beta, initial_state=x.initial_state, lib=lib)
    G = np.cumsum(np.maximum(x.g.double().numpy(), -1.0), axis=0)      # [T, H, dk]
    S0 = x.initial_state.double().numpy()[0]                           # [H, dk, dv]
    scale = 1.0 / np.sqrt(8)
    for h in range(2):
        assert np.allclose(fin[0, h], np.exp(G[-1, h])[:, None] * S0[h], rtol=1e-12, atol=1e-14)
        expect = scale * (np.exp(G[:, h]) * x.q[:, h].double().numpy()) @ S0[h]
        assert np.allclose(out[:, h], expect, rtol=1e-12, atol=1e-14)
    # g = 0 as well: the state never changes
    out, fin = ko.recurrent(x.q, x.k, x.v, torch.zeros_like(x.g), beta,
                            initial_state=x.initial_state, lib=lib)
    assert np.array_equal(fin[0], S0)


def _exact_unit_keys(T, dk, rng):
    """Keys with four entries of +-1/2: exactly unit norm in binary floating point."""
    k = np.zeros((T, dk), dtype=np.float32)
    for t in range(T):
        idx = rng.choice(dk, 4, replace=False)
        k[t, idx] = rng.choice([-0.5, 0.5], 4)
    return k


def pin_delta_rule_reach(lib):
    """|k| = 1, beta = 1: S_t^T k_t = v_t for any g and S0 (since (I - k k^T) k = 0).

    With q_t = k_t the read-out is therefore scale * v_t at every token.
    """
    rng = np.random.default_rng(11)
    T, H, dk, dv = 40, 1, 16, 6
    k = _exact_unit_keys(T, dk, rng)[:, None]
    v = rng.standard_normal((T, H, dv)).astype(np.float32)
    g = (-rng.random((T, H, dk))).astype(np.float32)
    s0 = rng.standard_normal((1, H, dk, dv))
    b = np.ones((T, H), dtype=np.float32)
    out, _ = ko.recurrent(k, k, v, g, b, initial_state=s0, scale=0.25, lib=lib)
    assert np.allclose(out, 0.25 * v.astype(np.float64), rtol=1e-12, atol=1e-12)


def pin_general_beta_reach(lib):
    """S_t^T k_t = (1 - b_t) (D_t S_{t-1})^T k_t + b_t v_t for unit k_t and any b_t."""
    rng = np.random.default_rng(12)
    T, dk, dv = 9, 16, 7
    k = _exact_unit_keys(T, dk, rng)[:, None]
    v = rng.standard_normal((T, 1, dv)).astype(np.float32)
    g = (-rng.random((T, 1, dk))).astype(np.float32)
    b = rng.random((T, 1)).astype(np.float32)
    s0 = rng.standard_normal((1, 1, dk, dv))
    _, s_prev = ko.recurrent(k[:-1], k[:-1], v[:-1], g[:-1], b[:-1], initial_state=s0, lib=lib)
    out, _ = ko.recurrent(k, k, v, g, b, initial_state=s0, scale=1.0, lib=lib)
    kt = k[-1, 0].astype(np.float64)
    D = np.exp(np.maximum(g[-1, 0].astype(np.float64), -1.0))
    bt = float(b[-1, 0])
    expect = (1 - bt) * (D[:, None] * s_prev[0, 0]).T @ kt + bt * v[-1, 0].astype(np.float64)
    assert np.allclose(out[-1, 0], expect, rtol=1e-12, atol=1e-12)


def pin_associative_memory(lib):
    """g = 0, beta = 1, S0 = 0, orthonormal keys k_1..k_n: querying k_i recalls v_i.

    Keys are rows of a 16x16 Sylvester-Hadamard matrix / 4 (exact in binary).
    Recall tokens carry beta = 0 so they leave the state unchanged.
    """
    dk, dv, n = 16, 5, 12
    Hd = np.array([[1.0]])
    while Hd.shape[0] < dk:
        Hd = np.block([[Hd, Hd], [Hd, -Hd]])
    keys = (Hd[:n] / 4.0).astype(np.float32)
    rng = np.random.default_rng(13)
    vals = rng.standard_normal((n, dv)).astype(np.float32)
    perm = rng.permutation(n)
    k = np.concatenate([keys, keys[perm]])[:, None]
    v = np.concatenate([vals, np.zeros_like(vals)])[:, None]
    b = np.concatenate([np.ones(n), np.zeros(n)]).astype(np.float32)[:, None]
    g = np.zeros((2 * n, 1, dk), dtype=np.float32)
    out, fin = ko.recurrent(k, k, v, g, b, scale=1.0, lib=lib)
    assert np.allclose(out[n:, 0], vals[perm].astype(np.float64), rtol=1e-12, atol=1e-12)
    assert np.allclose(fin[0, 0], keys.T.astype(np.float64) @ vals.astype(np.float64), atol=1e-12)


def pin_one_token_expansion(lib):
    """T = 1: o = scale [(D S0)^T q - b (k.q)(D S0)^T k + b (k.q) v], S1 = D S0 + b k (v - (D S0)^T k)^T."""
    x = make_inputs(1, H=3, dk=6, dv=4, dtype=torch.float32, seed=17, state_std=1.0, g_scale=1.5)
    out, fin = ko.recurrent(x.q, x.k, x.v, x.g, x.beta, initial_state=x.initial_state, lib=lib)
    scale = 1.0 / np.sqrt(6)
    for h in range(3):
        q = x.q[0, h].double().numpy()
        k = x.k[0, h].double().numpy()
        v = x.v[0, h].double().numpy()
        b = float(x.beta[0, h])
        D = np.exp(np.maximum(x.g[0, h].double().numpy(), -1.0))
        DS = D[:, None] * x.initial_state[0, h].double().numpy()
        kq = float(k @ q)
        o = scale * (DS.T @ q - b * kq * (DS.T @ k) + b * kq * v)
        S1 = DS + b * np.outer(k, v - DS.T @ k)
        assert np.allclose(out[0, h], o, rtol=1e-12, atol=1e-13)
        assert np.allclose(fin[0, h], S1, rtol=1e-12, atol=1e-13)


def pin_linearity(lib):
    """For fixed (q, k, g, beta), (V, S0) -> (O, S_T) is linear."""
    x1 = make_inputs(50, H=2, dk=8, dv=6, dtype=torch.float32, seed=21, state_std=0.5)
    x2 = make_inputs(50, H=2, dk=8, dv=6, dtype=torch.float32, seed=22, state_std=0.5)
    a, c = 0.75, -1.25
    o1, s1 = ko.recurrent(x1.q, x1.k, x1.v, x1.g, x1.beta, initial_state=x1.initial_state, lib=lib)
    o2, s2 = ko.recurrent(x1.q, x1.k, x2.v, x1.g, x1.beta, initial_state=x2.initial_state, lib=lib)
    v3 = (a * x1.v + c * x2.v)
    s03 = a * x1.initial_state.double() + c * x2.initial_state.double()
    o3, s3 = ko.recurrent(x1.q, x1.k, v3, x1.g, x1.beta, initial_state=s03, lib=lib)
    # v3 is rounded to f32; compare against the same combination taken in fp64 with a loose bound
    assert _rel(o3, a * o1 + c * o2) < 1e-6
    assert _rel(s3, a * s1 + c * s2) < 1e-6


def pin_contraction_bound(lib):
    """|k| = 1, beta in [0,1], g <= 0: ||S_t||_2 <= ||S_{t-1}||_2 + beta_t ||v_t||."""
    x = make_inputs(30, H=1, dk=8, dv=8, dtype=torch.float32, seed=31, state_std=1.0)
    S = x.initial_state.double()
    prev = np.linalg.norm(S.numpy()[0, 0], 2)
    for t in range(30):
        sl = slice(t, t + 1)
        _, S = ko.recurrent(x.q[sl], x.k[sl], x.v[sl], x.g[sl], x.beta[sl], initial_state=S,
                            lib=lib)
        now = np.linalg.norm(S[0, 0], 2)
        bound = prev + float(x.beta[t, 0]) * float(x.v[t, 0].double().norm())
        assert now <= bound * (1 + 1e-6) + 1e-12, (t, now, bound)
        prev = now
        S = torch.tensor(S)


def pin_resume_and_varlen(lib):
    """Split prefill == one prefill; packed varlen == separate runs; T decode steps == prefill."""
    x = make_inputs(None, H=2, dk=8, dv=4, dtype=torch.float32, seed=41, lengths=[33, 20],
                    state_std=0.5)
    cu = x.cu_seqlens.tolist()
    o_all, s_all = ko.recurrent(x.q, x.k, x.v, x.g, x.beta, cu_seqlens=cu,
                                initial_state=x.initial_state, lib=lib)
    for s in range(2):
        a, e = cu[s], cu[s + 1]
        sl = slice(a, e)
        o, st = ko.recurrent(x.q[sl], x.k[sl], x.v[sl], x.g[sl], x.beta[sl],
                             initial_state=x.initial_state[s:s + 1], lib=lib)
        assert np.array_equal(o, o_all[sl]) and np.array_equal(st[0], s_all[s])
        m = a + (e - a) // 2
        o1, st1 = ko.recurrent(x.q[a:m], x.k[a:m], x.v[a:m], x.g[a:m], x.beta[a:m],
                               initial_state=x.initial_state[s:s + 1], lib=lib)
        o2, st2 = ko.recurrent(x.q[m:e], x.k[m:e], x.v[m:e], x.g[m:e], x.beta[m:e],
                               initial_state=st1, lib=lib)
        assert np.array_equal(np.concatenate([o1, o2]), o_all[sl])
        assert np.array_equal(st2[0], s_all[s])
    # one token per "sequence" = one decode step per sequence, all from the same state
    S = x.initial_state[:1].double().numpy()
    for t in range(cu[1]):
        sl = slice(t, t + 1)
        o, S = ko.recurrent(x.q[sl], x.k[sl], x.v[sl], x.g[sl], x.beta[sl], initial_state=S,
                            lib=lib)
        assert np.array_equal(o[0], o_all[t])
    assert np.array_equal(S[0], s_all[0])


def pin_decay_clamp(lib):
    """Log decays below lb act exactly as lb (the lower bound of the log decay)."""
    x = make_inputs(20, H=2, dk=8, dv=4, dtype=torch.float32, seed=51, g_scale=4.0, state_std=0.5)
    lb = -1.5
    assert float(x.g.min()) < lb
    o1, s1 = ko.recurrent(x.q, x.k, x.v, x.g, x.beta, initial_state=x.initial_state, lb=lb, lib=lib)
    o2, s2 = ko.recurrent(x.q, x.k, x.v, x.g.clamp_min(lb), x.beta,
                          initial_state=x.initial_state, lb=lb, lib=lib)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)
    o3, _ = ko.recurrent(x.q, x.k, x.v, x.g, x.beta, initial_state=x.initial_state, lb=-10.0,
                         lib=lib)
    assert _rel(o1, o3) > 1e-3  # the clamp is active on these inputs


def pin_sampled_rows(lib):
    """Sampled read-out rows equal the same rows of the full read-out."""
    x = make_inputs(None, H=2, dk=8, dv=4, dtype=torch.float32, seed=61, lengths=[17, 0, 30],
                    state_std=0.2)
    cu = x.cu_seqlens.tolist()
    full, s_full = ko.recurrent(x.q, x.k, x.v, x.g, x.beta, cu_seqlens=cu,
                                initial_state=x.initial_state, lib=lib)
    rows = [0, 5, 16, 17, 40, 46]
    part, s_part = ko.recurrent(x.q, x.k, x.v, x.g, x.beta, cu_seqlens=cu,
                                initial_state=x.initial_state, out_rows=rows, lib=lib)
    assert np.array_equal(part, full[rows]) and np.array_equal(s_part, s_full)
    assert np.array_equal(s_full[1], x.initial_state[1].double().numpy())  # empty sequence


def pin_snapshots_are_prefix_states(lib):
    """Snapshot m of a sequence is the state after its first m * P tokens: the final state
    of a separate run over that prefix alone, from the same initial state. Recording the
    snapshots changes neither the read-out nor the final states."""
    x = make_inputs(None, H=2, dk=8, dv=4, dtype=torch.float32, seed=71,
                    lengths=[25, 7, 0, 16, 31], state_std=0.5)
    cu = x.cu_seqlens.tolist()
    P = 8
    out, fin, snaps, first = ko.recurrent_snapshots(
        x.q, x.k, x.v, x.g, x.beta, snapshot_tokens=P, cu_seqlens=cu,
        initial_state=x.initial_state, want_out=True, lib=lib)
    o_ref, s_ref = ko.recurrent(x.q, x.k, x.v, x.g, x.beta, cu_seqlens=cu,
                                initial_state=x.initial_state, lib=lib)
    assert np.array_equal(out, o_ref) and np.array_equal(fin, s_ref)
    counts = [(cu[s + 1] - cu[s]) // P for s in range(len(cu) - 1)]
    assert counts == [3, 0, 0, 2, 3] and snaps.shape[0] == sum(counts)
    for s, cnt in enumerate(counts):
        for m in range(1, cnt + 1):
            sl = slice(cu[s], cu[s] + m * P)
            _, st = ko.recurrent(x.q[sl], x.k[sl], x.v[sl], x.g[sl], x.beta[sl],
                                 initial_state=x.initial_state[s:s + 1], lib=lib)
            assert np.array_equal(snaps[first[s] + m - 1], st[0]), (s, m)
    assert np.array_equal(snaps[first[3] + 1], fin[3])  # 16 tokens: the last one is final


def _unit_rows(T, H, d, rng):
    """Rows with entries +-1/2 (d = 4): unit L2 norm exactly in binary; L1 norm 2."""
    return rng.choice([-0.5, 0.5], size=(T, H, d)).astype(np.float32)


def pin_prologue_l2norm(lib):
    """The q/k normalisation prologue: unit rows pass through unchanged (exact), and the
    result does not change when any token's q or k row is scaled by a positive factor
    (powers of two, so the scaled inputs and their norms are exact)."""
    rng = np.random.default_rng(81)
    T, H, d = 24, 2, 4
    x = make_inputs(T, H=H, dk=d, dv=3, dtype=torch.float32, seed=81, state_std=0.5)
    q, k = _f32(_unit_rows(T, H, d, rng)), _f32(_unit_rows(T, H, d, rng))
    o1, s1 = ko.recurrent(q, k, x.v, x.g, x.beta, initial_state=x.initial_state, lib=lib)
    o2, s2 = ko.recurrent(q, k, x.v, x.g, x.beta, initial_state=x.initial_state,
                          prologue=ko.QK_L2NORM, lib=lib)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)
    # raw rows of any length: scale invariance, and the unit-row result is reproduced
    cq = torch.tensor(rng.choice([0.25, 2.0, 8.0, 0.5], size=(T, H, 1)), dtype=torch.float32)
    ck = torch.tensor(rng.choice([4.0, 0.125, 2.0, 16.0], size=(T, H, 1)), dtype=torch.float32)
    o3, s3 = ko.recurrent(q * cq, k * ck, x.v, x.g, x.beta, initial_state=x.initial_state,
                          prologue=ko.QK_L2NORM, lib=lib)
    assert np.array_equal(o3, o1) and np.array_equal(s3, s1)
    # general rows: normalising twice is normalising once
    y = make_inputs(T, H=H, dk=8, dv=3, dtype=torch.float32, seed=82, state_std=0.5)
    qr, kr = y.q * 3.0, y.k * 0.5
    o4, s4 = ko.recurrent(qr * cq, kr * ck, y.v, y.g, y.beta, initial_state=y.initial_state,
                          prologue=ko.QK_L2NORM, lib=lib)
    o5, s5 = ko.recurrent(qr, kr, y.v, y.g, y.beta, initial_state=y.initial_state,
                          prologue=ko.QK_L2NORM, lib=lib)
    assert _rel(o4, o5) < 1e-13 and _rel(s4, s5) < 1e-13
    o6, _ = ko.recurrent(qr, kr, y.v, y.g, y.beta, initial_state=y.initial_state, lib=lib)
    assert _rel(o6, o5) > 1e-2  # the prologue is active on these inputs


def pin_prologue_gate(lib):
    """The gate prologue log decay = lb * sigmoid(a): a = 0 gives exactly lb / 2; a large
    positive pre-activation gives the bound lb, a large negative one no decay."""
    lb = -0.75
    x = make_inputs(20, H=2, dk=8, dv=4, dtype=torch.float32, seed=83, state_std=0.5)
    run = dict(initial_state=x.initial_state, lb=lb, lib=lib)
    zero = torch.zeros_like(x.g)
    o1, s1 = ko.recurrent(x.q, x.k, x.v, zero, x.beta, prologue=ko.GATE_SIGMOID, **run)
    o2, s2 = ko.recurrent(x.q, x.k, x.v, torch.full_like(x.g, lb / 2), x.beta, **run)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)
    o3, s3 = ko.recurrent(x.q, x.k, x.v, torch.full_like(x.g, 40.0), x.beta,
                          prologue=ko.GATE_SIGMOID, **run)
    o4, s4 = ko.recurrent(x.q, x.k, x.v, torch.full_like(x.g, lb), x.beta, **run)
    assert _rel(o3, o4) < 1e-12 and _rel(s3, s4) < 1e-12
    o5, s5 = ko.recurrent(x.q, x.k, x.v, torch.full_like(x.g, -40.0), x.beta,
                          prologue=ko.GATE_SIGMOID, **run)
    o6, s6 = ko.recurrent(x.q, x.k, x.v, zero, x.beta, **run)
    assert _rel(o5, o6) < 1e-12 and _rel(s5, s6) < 1e-12
    # both prologues together: each acts on its own inputs
    both = ko.QK_L2NORM | ko.GATE_SIGMOID
    o7, s7 = ko.recurrent(x.q * 4.0, x.k * 0.5, x.v, zero, x.beta, prologue=both, **run)
    o8, s8 = ko.recurrent(x.q, x.k, x.v, zero, x.beta, prologue=both, **run)
    assert np.array_equal(o7, o8) and np.array_equal(s7, s8)
    assert _rel(o8, o1) < 1e-5 and _rel(s8, s1) < 1e-5  # q, k are unit rows up to fp32


def pin_backward_finite_differences(lib):
    """The reverse-mode gradients equal central finite differences of the independently
    derived chunked fp64 form, element by element for q, k, v, g, beta and S0, with
    L = sum(d_out * o) + sum(d_final * S_final); varlen with an empty sequence, and the
    clamp active on some gates (their gradient is zero)."""
    rng = np.random.default_rng(91)
    lb = -1.2
    x = make_inputs(None, H=2, dk=3, dv=2, dtype=torch.float32, seed=91, lengths=[4, 0, 5],
                    state_std=0.5, g_scale=2.0)
    cu = x.cu_seqlens.tolist()
    T = cu[-1]
    do = rng.standard_normal((T, 2, 2))
    dS = rng.standard_normal((3, 2, 3, 2))
    got = ko.backward(x.q, x.k, x.v, x.g, x.beta, d_out=do, d_final=dS, cu_seqlens=cu,
                      initial_state=x.initial_state, lb=lb, lib=lib)
    vals = {n: ko._widen(getattr(x, n)).copy() for n in ("q", "k", "v", "g", "beta")}
    vals["s0"] = x.initial_state.double().numpy().copy()
    assert (vals["g"] < lb - 1e-3).any() and (vals["g"] > lb + 1e-3).any()

    def loss():
        o, s = ko.chunked(vals["q"], vals["k"], vals["v"], vals["g"], vals["beta"], chunk=3,
                          cu_seqlens=cu, initial_state=vals["s0"], lb=lb)
        return float(np.sum(do * o) + np.sum(dS * s))
    h = 1e-6
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("beta", "dbeta"),
                      ("s0", "ds0")):
        arr = vals[name]
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            if name == "g" and abs(arr[idx] - lb) < 1e-3:
                fd[idx] = got[key][idx]  # the kink of the clamp: no finite difference
                continue
            x0 = arr[idx]
            arr[idx] = x0 + h
            lp = loss()
            arr[idx] = x0 - h
            lm = loss()
            arr[idx] = x0
            fd[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(fd - got[key]))
        assert err <= 1e-6 * max(1.0, np.max(np.abs(fd))), (name, err)
    assert np.all(got["dg"][ko._widen(x.g) < lb] == 0.0)


def pin_backward_beta_zero(lib):
    """beta = 0 leaves only the decay: S_t = Diag(gamma_t) S0 with gamma_t the product of
    the clamped decays, so dq_t = scale gamma_t * (S0 do_t), dS0 = sum_t scale (gamma_t * q_t)
    do_t^T + Diag(gamma_T) dS_final, and dk = dv = 0."""
    rng = np.random.default_rng(93)
    x = make_inputs(11, H=2, dk=4, dv=3, dtype=torch.float32, seed=93, state_std=0.5)
    beta = torch.zeros_like(x.beta)
    do = rng.standard_normal((11, 2, 3))
    dS = rng.standard_normal((1, 2, 4, 3))
    sc = 0.7
    got = ko.backward(x.q, x.k, x.v, x.g, beta, d_out=do, d_final=dS,
                      initial_state=x.initial_state, scale=sc, lib=lib)
    G = np.exp(np.cumsum(np.maximum(ko._widen(x.g), -1.0), axis=0))  # [T, H, dk]
    Q = ko._widen(x.q)
    S0 = x.initial_state.double().numpy()[0]
    for h in range(2):
        dq = sc * G[:, h, :] * (do[:, h, :] @ S0[h].T)
        ds0 = sc * (G[:, h, :] * Q[:, h, :]).T @ do[:, h, :] + G[-1, h, :, None] * dS[0, h]
        assert np.allclose(got["dq"][:, h], dq, rtol=1e-12, atol=1e-14)
        assert np.allclose(got["ds0"][0, h], ds0, rtol=1e-12, atol=1e-14)
    assert np.all(got["dk"] == 0.0) and np.all(got["dv"] == 0.0)


def pin_backward_prologue_finite_differences(lib):
    """With the raw-input prologue the gradients are those of the raw q, k and gate
    pre-activations: central finite differences of the chunked fp64 form fed with
    q / |q|, k / |k| and lb * sigmoid(a) formed in fp64 here."""
    rng = np.random.default_rng(95)
    lb = -0.8
    x = make_inputs(None, H=1, dk=3, dv=2, dtype=torch.float32, seed=95, lengths=[5, 3],
                    state_std=0.5, raw=True)
    cu = x.cu_seqlens.tolist()
    T = cu[-1]
    do = rng.standard_normal((T, 1, 2))
    dS = rng.standard_normal((2, 1, 3, 2))
    got = ko.backward(x.q, x.k, x.v, x.g, x.beta, d_out=do, d_final=dS, cu_seqlens=cu,
                      initial_state=x.initial_state, lb=lb,
                      prologue=ko.QK_L2NORM | ko.GATE_SIGMOID, lib=lib)
    vals = {n: ko._widen(getattr(x, n)).copy() for n in ("q", "k", "g")}
    fixed = {n: ko._widen(getattr(x, n)) for n in ("v", "beta")}

    def loss():
        qn = vals["q"] / np.linalg.norm(vals["q"], axis=-1, keepdims=True)
        kn = vals["k"] / np.linalg.norm(vals["k"], axis=-1, keepdims=True)
        gg = lb / (1.0 + np.exp(-vals["g"]))
        o, s = ko.chunked(qn, kn, fixed["v"], gg, fixed["beta"], chunk=2, cu_seqlens=cu,
                          initial_state=x.initial_state.double().numpy(), lb=lb)
        return float(np.sum(do * o) + np.sum(dS * s))
    h = 1e-6
    for name, key in (("q", "dq"), ("k", "dk"), ("g", "dg")):
        arr = vals[name]
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            x0 = arr[idx]
            arr[idx] = x0 + h
            lp = loss()
            arr[idx] = x0 - h
            lm = loss()
            arr[idx] = x0
            fd[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(fd - got[key]))
        assert err <= 1e-6 * max(1.0, np.max(np.abs(fd))), (name, err)


ALL_PINS = [pin_golden, pin_chunked_agreement, pin_beta_zero_pure_decay, pin_delta_rule_reach,
            pin_general_beta_reach, pin_associative_memory, pin_one_token_expansion,
            pin_linearity, pin_contraction_bound, pin_resume_and_varlen, pin_decay_clamp,
            pin_sampled_rows, pin_snapshots_are_prefix_states, pin_prologue_l2norm,
            pin_prologue_gate, pin_backward_finite_differences, pin_backward_beta_zero,
            pin_backward_prologue_finite_differences]


def failing_pins(lib_path: str) -> list[str]:
    """Names of the pins that fail (or crash) against the oracle library at lib_path."""
    lib = ko.load(lib_path)
    bad = []
    for p in ALL_PINS:
        try:
            p(lib)
        except Exception:  # noqa: BLE001 -- any failure counts as caught
            bad.append(p.__name__)
    return bad
