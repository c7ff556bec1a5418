"""Pins for the oracle's backward pass (the unnormalised form's gradients).

Nothing here restates the backward's formulas.  The gradients are checked against:
  - central finite differences of the oracle's own forward pass (the loss
    L = sum(dout * out) + sum(dS_final * S_final));
  - float64 autograd through an independent form: the parallel (masked quadratic) form
    of "Linear Attention and Retentive Networks ...", A. Parallel Representation,
    ((phi(Q) phi(K)^T) .* D) V plus the initial state's decayed readout;
  - gamma = 0, where only the diagonal of D survives and the gradients have closed forms.
Planted mistakes in copies of the backward must each fail one of these.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle.oracle import SRC, Oracle, build, default_oracle


def _phi(x, fm):
    return x if fm == "identity" else torch.where(x > 0, x + 1.0, torch.exp(x))


def _problem(seed, fm, T=9, dk=3, dv=4, H=2):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((1, H, T, d)).astype(np.float32) * 0.7 for d in (dk, dk, dv))
    if fm == "elu1":  # keep inputs away from ELU's kink, where differences lose accuracy
        q, k = (np.where(np.abs(a) < 0.05, a + 0.1, a).astype(np.float32) for a in (q, k))
    dout = rng.standard_normal((1, H, T, dv))
    S0 = rng.standard_normal((1, H, dk, dv)) * 0.5
    dSf = rng.standard_normal((1, H, dk, dv))
    return q, k, v, dout, S0, dSf


def _loss(o: Oracle, q, k, v, dout, S0, dSf, fm, gamma):
    out, S, _ = o.forward(q, k, v, feature_map=fm, gamma=gamma, normalize=False, S_init=S0)
    return float(np.sum(dout * out) + np.sum(dSf * S))


def _finite_differences(o, q, k, v, dout, S0, dSf, fm, gamma):
    # Inputs are float32: step 2^-10 is exactly representable on top of values of this size.
    h = 2.0 ** -10
    grads = []
    for which, arr in (("q", q), ("k", k), ("v", v)):
        g = np.zeros(arr.shape)
        for idx in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += np.float32(h)
            minus[idx] -= np.float32(h)
            args = {"q": q, "k": k, "v": v}
            args[which] = plus
            lp = _loss(o, args["q"], args["k"], args["v"], dout, S0, dSf, fm, gamma)
            args[which] = minus
            lm = _loss(o, args["q"], args["k"], args["v"], dout, S0, dSf, fm, gamma)
            g[idx] = (lp - lm) / (float(plus[idx]) - float(minus[idx]))
        grads.append(g)
    g = np.zeros(S0.shape)
    for idx in np.ndindex(S0.shape):
        plus, minus = S0.copy(), S0.copy()
        plus[idx] += 1e-6
        minus[idx] -= 1e-6
        g[idx] = (_loss(o, q, k, v, dout, plus, dSf, fm, gamma)
                  - _loss(o, q, k, v, dout, minus, dSf, fm, gamma)) / 2e-6
    grads.append(g)
    return grads


def _autograd_parallel(q, k, v, dout, S0, dSf, fm, gamma):
    T = q.shape[2]
    Q, K, V = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    S_init = torch.tensor(S0, dtype=torch.float64, requires_grad=True)
    g = torch.tensor([1.0] * q.shape[1] if gamma is None else gamma, dtype=torch.float64)
    t = torch.arange(T, dtype=torch.float64)
    dist = t[:, None] - t[None, :]
    D = torch.where(dist >= 0, g[:, None, None] ** dist.clamp(min=0), torch.zeros(()))  # [H,T,T]
    fq, fk = _phi(Q, fm), _phi(K, fm)
    out = ((fq @ fk.transpose(-1, -2)) * D) @ V + (g[:, None, None] ** (t[:, None] + 1)) * (fq @ S_init)
    S = torch.einsum("bhti,bhtj,ht->bhij", fk, V, g[:, None] ** (T - 1 - t)) + \
        (g ** T)[None, :, None, None] * S_init
    L = (torch.tensor(dout) * out).sum() + (torch.tensor(dSf) * S).sum()
    return [x.numpy() for x in torch.autograd.grad(L, (Q, K, V, S_init))]


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def _backward_pins(o: Oracle) -> dict[str, bool]:
    res = {}
    for fm in ("identity", "elu1"):
        for gamma in (None, [0.9, 0.6]):
            tag = f"{fm}_{'decay' if gamma else 'nodecay'}"
            q, k, v, dout, S0, dSf = _problem(1, fm)
            got = o.backward(q, k, v, dout, feature_map=fm, gamma=gamma, S_init=S0, dS_final=dSf)
            fd = _finite_differences(o, q, k, v, dout, S0, dSf, fm, gamma)
            res[f"finite_differences_{tag}"] = all(_rel(a, b) < 1e-5 for a, b in zip(got, fd))
            ag = _autograd_parallel(q, k, v, dout, S0, dSf, fm, gamma)
            res[f"autograd_parallel_{tag}"] = all(_rel(a, b) < 1e-10 for a, b in zip(got, ag))
    # gamma = 0: o_t = (phi(q_t) . phi(k_t)) v_t, so
    # dq_t = (do_t . v_t) phi(k_t) phi'(q_t), dk_t = (do_t . v_t) phi(q_t) phi'(k_t),
    # dv_t = (phi(q_t) . phi(k_t)) do_t, and nothing reaches S_init.
    q, k, v, dout, S0, dSf = _problem(2, "elu1")
    dq, dk, dv, dS0 = o.backward(q, k, v, dout, feature_map="elu1", gamma=[0.0, 0.0], S_init=S0)
    fq, fk = (_phi(torch.tensor(a, dtype=torch.float64), "elu1").numpy() for a in (q, k))
    dphi = lambda a: np.where(a > 0, 1.0, np.exp(a.astype(np.float64)))
    dov = np.sum(dout * v, -1, keepdims=True)
    res["gamma_zero"] = (_rel(dq, dov * fk * dphi(q)) < 1e-13 and _rel(dk, dov * fq * dphi(k)) < 1e-13
                         and _rel(dv, np.sum(fq * fk, -1, keepdims=True) * dout) < 1e-13
                         and float(np.max(np.abs(dS0))) == 0.0)
    return res


def test_backward_pins_hold():
    res = _backward_pins(default_oracle())
    assert all(res.values()), res


BACKWARD_MUTANTS = {
    "reverse_sweep_decays_current_token": ("Gi[j] += fq * dout[t * dv + j];",
                                           "Gi[j] += fq * dout[t * dv + j] * g;"),
    "reverse_sweep_without_decay": ("for (double& x : G) x *= g;", "for (double& x : G) x *= 1.0;"),
    "dq_without_feature_derivative": (
        "p.dq[(bh * T + t) * dk + i] = acc * feature_map_derivative(x, p.fm);",
        "p.dq[(bh * T + t) * dk + i] = acc;"),
    "dv_uses_query_features": (
        "acc += G[static_cast<size_t>(i) * dv + j] * fk[i];",
        "acc += G[static_cast<size_t>(i) * dv + j] * "
        "feature_map(static_cast<double>(q[t * dk + i]), p.fm);"),
    "final_state_gradient_dropped": ("G[e] = p.dS_final[bh * dk * dv + e];", "G[e] = 0.0;"),
    "dq_contracts_the_state_with_v": ("acc += Si[j] * dout[t * dv + j];",
                                      "acc += Si[j] * static_cast<double>(v[t * dv + j]);"),
}


@pytest.mark.parametrize("name", sorted(BACKWARD_MUTANTS))
def test_backward_mutant_is_caught(tmp_path, name):
    text = SRC.read_text()
    old, new = BACKWARD_MUTANTS[name]
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    src = tmp_path / f"{name}.cpp"
    src.write_text(text.replace(old, new))
    res = _backward_pins(Oracle(build(src, tmp_path / f"{name}.so", force=True)))
    assert not all(res.values()), f"mutant {name} passed every backward pin"
