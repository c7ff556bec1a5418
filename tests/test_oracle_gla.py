"""Pins for the oracle's gated linear attention (GLA) token loop.

The gate G_t = alpha_t 1^T of "Linear Attention and Retentive Networks ...", Gated Linear
Attention (GLA) and Hardware-Software Co-Design, scales row i (key feature i) of the state by
alpha_t[i].  The loop is checked against things that are not itself:
  - a brute-force parallel form written from the products of the gates:
    o_t = sum_{s<=t} sum_i q_t[i] k_s[i] (prod_{r=s+1..t} alpha_r[i]) v_s, plus the initial
    state read out through prod_{r=0..t} alpha_r;
  - gates constant per head, alpha_t[i] = gamma_h: the retention loop (the oracle's pinned
    forward with per-head decay);
  - gates of 1: plain causal linear attention, a cumulative sum;
  - a gate of 0 at token t0 for one feature: that feature's history before t0 is gone.
Planted mistakes in copies of the loop must each fail one of these.
"""

from __future__ import annotations

import numpy as np
import pytest

from oracle.oracle import SRC, Oracle, build, default_oracle


def _problem(seed, T=11, dk=4, dv=3, H=2):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((1, H, T, d)).astype(np.float32) for d in (dk, dk, dv))
    alpha = (1.0 / (1.0 + np.exp(-rng.normal(1.5, 1.0, (1, H, T, dk))))).astype(np.float32)
    S0 = rng.standard_normal((1, H, dk, dv))
    return q, k, v, alpha, S0


def _brute(q, k, v, alpha, S0):
    q, k, v, a = (x.astype(np.float64) for x in (q, k, v, alpha))
    B, H, T, dk = q.shape
    out = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            for t in range(T):
                for s in range(t + 1):
                    decay = np.prod(a[b, h, s + 1:t + 1], axis=0)          # [dk]
                    out[b, h, t] += np.sum(q[b, h, t] * k[b, h, s] * decay) * v[b, h, s]
                init = np.prod(a[b, h, :t + 1], axis=0)                     # [dk]
                out[b, h, t] += (q[b, h, t] * init) @ S0[b, h]
    return out


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def _gla_pins(o: Oracle) -> dict[str, bool]:
    res = {}
    q, k, v, alpha, S0 = _problem(1)
    out, S = o.gla_forward(q, k, v, alpha, S_init=S0)
    res["brute_force_parallel_form"] = _rel(out, _brute(q, k, v, alpha, S0)) < 1e-12
    gam = [float(np.float32(0.8)), float(np.float32(0.95))]  # the gates' float32 values
    ac = np.broadcast_to(np.asarray(gam, dtype=np.float32)[None, :, None, None], alpha.shape).copy()
    out_g, S_g = o.gla_forward(q, k, v, ac, S_init=S0)
    out_r, S_r, _ = o.forward(q, k, v, feature_map="identity", gamma=gam, normalize=False,
                              S_init=S0)
    res["constant_gates_are_retention"] = _rel(out_g, out_r) < 1e-12 and _rel(S_g, S_r) < 1e-12
    ones = np.ones_like(alpha)
    out_1, S_1 = o.gla_forward(q, k, v, ones)
    kv = np.einsum("bhti,bhtj->bhtij", k.astype(np.float64), v.astype(np.float64))
    cum = np.cumsum(kv, axis=2)
    res["unit_gates_are_a_cumulative_sum"] = (
        _rel(out_1, np.einsum("bhti,bhtij->bhtj", q.astype(np.float64), cum)) < 1e-12
        and _rel(S_1, cum[:, :, -1]) < 1e-12)
    # a zero gate on feature 1 at token 5 erases that row's history: with the keys of feature
    # 1 zero from token 5 on, row 1 of S_final is exactly zero
    a0 = alpha.copy()
    a0[:, :, 5, 1] = 0.0
    k0 = k.copy()
    k0[:, :, 5:, 1] = 0.0
    _, S0z = o.gla_forward(q, k0, v, a0, S_init=S0)
    res["zero_gate_forgets"] = float(np.max(np.abs(S0z[:, :, 1]))) == 0.0 and \
        float(np.min(np.abs(S0z[:, :, 0]))) > 0.0
    return res


def test_gla_pins_hold():
    res = _gla_pins(default_oracle())
    assert all(res.values()), res


GLA_MUTANTS = {
    "gate_applied_after_the_update": (
        "Si[j] = gate * Si[j] + ki * static_cast<double>(v[t * dv + j]);",
        "Si[j] = gate * (Si[j] + ki * static_cast<double>(v[t * dv + j]));"),
    "gate_on_the_value_side": (
        "const double gate = static_cast<double>(al[t * dk + i]);",
        "const double gate = static_cast<double>(al[t * dk + (i % dv)]);"),
    "state_read_before_the_update": (
        "acc += static_cast<double>(q[t * dk + i]) * S[static_cast<size_t>(i) * dv + j];",
        "acc += static_cast<double>(q[t * dk + i]) * (S[static_cast<size_t>(i) * dv + j] - "
        "static_cast<double>(k[t * dk + i]) * static_cast<double>(v[t * dv + j]));"),
    "initial_state_ignored": (
        "for (size_t e = 0; e < S.size(); ++e) S[e] = p.S_init[bh * dk * dv + e];\n  for (long long t = 0; t < T; ++t) {\n    for (int i = 0; i < dk; ++i) {\n      const double gate",
        "for (size_t e = 0; e < S.size(); ++e) S[e] = 0.0;\n  for (long long t = 0; t < T; ++t) {\n    for (int i = 0; i < dk; ++i) {\n      const double gate"),
}


@pytest.mark.parametrize("name", sorted(GLA_MUTANTS))
def test_gla_mutant_is_caught(tmp_path, name):
    text = SRC.read_text()
    old, new = GLA_MUTANTS[name]
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    src = tmp_path / f"{name}.cpp"
    src.write_text(text.replace(old, new))
    res = _gla_pins(Oracle(build(src, tmp_path / f"{name}.so", force=True)))
    assert not all(res.values()), f"mutant {name} passed every GLA pin"
