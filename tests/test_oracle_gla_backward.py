"""Pins for the oracle's gated-loop backward (la_oracle_gla_backward).

Checked against: central finite differences of the oracle's own gated forward (every input,
the gates included); float64 autograd through a brute-force parallel form built from products
of the gates; and, for gates constant per head, the retention backward (the oracle's pinned
la_oracle_backward).  The reverse sweep recomputes S from checkpoints every max(64,
ceil(sqrt(T))) tokens, so the sequences here cross block boundaries.  Planted mistakes must each fail a pin.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle.oracle import SRC, Oracle, build, default_oracle


def _problem(seed, T=70, dk=3, dv=2, H=2):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((1, H, T, d)).astype(np.float32) * 0.8 for d in (dk, dk, dv))
    alpha = (1.0 / (1.0 + np.exp(-rng.normal(1.5, 1.0, (1, H, T, dk))))).astype(np.float32)
    do = rng.standard_normal((1, H, T, dv))
    S0 = rng.standard_normal((1, H, dk, dv)) * 0.5
    dSf = rng.standard_normal((1, H, dk, dv))
    return q, k, v, alpha, do, S0, dSf


def _loss(o, q, k, v, a, do, S0, dSf):
    out, S = o.gla_forward(q, k, v, a, S_init=S0)
    return float(np.sum(do * out) + np.sum(dSf * S))


def _fd(o, q, k, v, a, do, S0, dSf):
    h = 2.0 ** -12
    grads = []
    for which in ("q", "k", "v", "a"):
        arr = {"q": q, "k": k, "v": v, "a": a}[which]
        g = np.zeros(arr.shape)
        for idx in np.ndindex(arr.shape):
            args = {"q": q, "k": k, "v": v, "a": a}
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += np.float32(h)
            minus[idx] -= np.float32(h)
            args[which] = plus
            lp = _loss(o, args["q"], args["k"], args["v"], args["a"], do, S0, dSf)
            args[which] = minus
            lm = _loss(o, args["q"], args["k"], args["v"], args["a"], do, S0, dSf)
            g[idx] = (lp - lm) / (float(plus[idx]) - float(minus[idx]))
        grads.append(g)
    g = np.zeros(S0.shape)
    for idx in np.ndindex(S0.shape):
        plus, minus = S0.copy(), S0.copy()
        plus[idx] += 1e-6
        minus[idx] -= 1e-6
        g[idx] = (_loss(o, q, k, v, a, do, plus, dSf) - _loss(o, q, k, v, a, do, minus, dSf)) / 2e-6
    grads.append(g)
    return grads  # dq, dk, dv, dalpha, dS_init


def _autograd_parallel(q, k, v, a, do, S0, dSf):
    Q, K, V, A = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v, a))
    S_init = torch.tensor(S0, dtype=torch.float64, requires_grad=True)
    T = q.shape[2]
    ones = torch.ones_like(A[:, :, 0])
    outs = []
    for t in range(T):
        o_t = torch.zeros_like(V[:, :, 0])
        for s in range(t + 1):
            prod = ones
            for r in range(s + 1, t + 1):
                prod = prod * A[:, :, r]
            o_t = o_t + (Q[:, :, t] * K[:, :, s] * prod).sum(-1, keepdim=True) * V[:, :, s]
        prod0 = ones
        for r in range(t + 1):
            prod0 = prod0 * A[:, :, r]
        o_t = o_t + torch.einsum("bhi,bhij->bhj", Q[:, :, t] * prod0, S_init)
        outs.append(o_t)
    out = torch.stack(outs, dim=2)
    S = torch.zeros_like(S_init)
    for s in range(T):
        prod = ones
        for r in range(s + 1, T):
            prod = prod * A[:, :, r]
        S = S + torch.einsum("bhi,bhj->bhij", K[:, :, s] * prod, V[:, :, s])
    prod0 = ones
    for r in range(T):
        prod0 = prod0 * A[:, :, r]
    S = S + prod0[..., None] * S_init
    L = (torch.tensor(do) * out).sum() + (torch.tensor(dSf) * S).sum()
    return [x.numpy() for x in torch.autograd.grad(L, (Q, K, V, A, S_init))]


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def _pins(o: Oracle) -> dict[str, bool]:
    res = {}
    q, k, v, a, do, S0, dSf = _problem(1)
    got = o.gla_backward(q, k, v, a, do, S_init=S0, dS_final=dSf)
    fd = _fd(o, q, k, v, a, do, S0, dSf)
    res["finite_differences"] = all(_rel(x, y) < 1e-5 for x, y in zip(got, fd))
    qs, ks, vs, as_, dos, S0s, dSfs = (x[:, :, :9] if x.ndim == 4 and x.shape[2] == 70 else x
                                       for x in _problem(2))
    got_s = o.gla_backward(qs, ks, vs, as_, dos, S_init=S0s, dS_final=dSfs)
    ag = _autograd_parallel(qs, ks, vs, as_, dos, S0s, dSfs)
    res["autograd_parallel"] = all(_rel(x, y) < 1e-10 for x, y in zip(got_s, ag))
    gam = [float(np.float32(0.9)), float(np.float32(0.6))]
    ac = np.broadcast_to(np.asarray(gam, dtype=np.float32)[None, :, None, None], a.shape).copy()
    g_gla = o.gla_backward(q, k, v, ac, do, S_init=S0, dS_final=dSf)
    g_ret = o.backward(q, k, v, do, feature_map="identity", gamma=gam, S_init=S0, dS_final=dSf)
    res["constant_gates_are_retention"] = all(_rel(x, y) < 1e-11 for x, y in
                                              zip((g_gla[0], g_gla[1], g_gla[2], g_gla[4]), g_ret[:4]))
    return res


def test_gla_backward_long_sequence_crosses_many_checkpoints():
    """T = 4500: the checkpoint interval is ceil(sqrt(T)) = 68 tokens, so the reverse sweep
    recomputes 67 blocks; with gates constant per head the gradients must equal the retention
    backward's (the oracle's separately pinned la_oracle_backward)."""
    o = default_oracle()
    q, k, v, a, do, S0, dSf = _problem(7, T=4500)
    gam = [float(np.float32(0.999)), float(np.float32(0.97))]
    ac = np.broadcast_to(np.asarray(gam, dtype=np.float32)[None, :, None, None], a.shape).copy()
    g_gla = o.gla_backward(q, k, v, ac, do, S_init=S0, dS_final=dSf)
    g_ret = o.backward(q, k, v, do, feature_map="identity", gamma=gam, S_init=S0, dS_final=dSf)
    for x, y in zip((g_gla[0], g_gla[1], g_gla[2], g_gla[4]), g_ret[:4]):
        assert _rel(x, y) < 1e-10


def test_gla_backward_pins_hold():
    res = _pins(default_oracle())
    assert all(res.values()), res


MUTANTS = {
    "gate_gradient_uses_the_new_state": (
        "ga += G[static_cast<size_t>(i) * dv + j] * Sp[static_cast<size_t>(i) * dv + j];",
        "ga += G[static_cast<size_t>(i) * dv + j] * Sb[static_cast<size_t>(i) * dv + j];"),
    "reverse_sweep_without_the_gate": (
        "for (int j = 0; j < dv; ++j) G[static_cast<size_t>(i) * dv + j] *= at;",
        "for (int j = 0; j < dv; ++j) G[static_cast<size_t>(i) * dv + j] *= 1.0;"),
    "checkpoint_after_the_step": (
        "if (t % kGlaCheck == 0) std::copy(S.begin(), S.end(), checks.begin() + (t / kGlaCheck) * sd);\n    step(S, t);",
        "step(S, t);\n    if (t % kGlaCheck == 0) std::copy(S.begin(), S.end(), checks.begin() + (t / kGlaCheck) * sd);"),
    "dv_contracts_with_q": (
        "acc += G[static_cast<size_t>(i) * dv + j] * static_cast<double>(k[t * dk + i]);",
        "acc += G[static_cast<size_t>(i) * dv + j] * static_cast<double>(q[t * dk + i]);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_gla_backward_mutant_is_caught(tmp_path, name):
    text = SRC.read_text()
    old, new = MUTANTS[name]
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    src = tmp_path / f"{name}.cpp"
    src.write_text(text.replace(old, new))
    res = _pins(Oracle(build(src, tmp_path / f"{name}.so", force=True)))
    assert not all(res.values()), f"mutant {name} passed every pin"
