"""Pins for the oracle's backward pass (both forms' gradients).

Nothing here restates the backward's formulas.  The gradients are checked against:
  - central finite differences of the oracle's own forward pass (the loss
    L = sum(dout * out) + sum(dS_final * S_final) (+ sum(dZ_final * Z_final) normalised));
  - float64 autograd through an independent form: the parallel (masked quadratic) form
    of "Linear Attention and Retentive Networks ...", A. Parallel Representation,
    ((phi(Q) phi(K)^T) .* D) V plus the initial state's decayed readout, divided for the
    normalised form by the same masked sums of ones plus eps ("Log-Depth Chunked
    Linear-Attention Scan", Implementation notes: the ratio with eps);
  - gamma = 0, where only the diagonal of D survives and the gradients have closed forms;
  - the normalised form with constant value rows, whose output is that row whatever q and
    k are, so their gradients vanish.
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
    Z0 = rng.uniform(0.5, 2.0, (1, H, dk))  # a positive normaliser keeps denominators > 0
    dZf = rng.standard_normal((1, H, dk))
    return q, k, v, dout, S0, dSf, Z0, dZf


def _loss(o: Oracle, q, k, v, dout, S0, dSf, fm, gamma, norm=False, eps=0.0, Z0=None, dZf=None):
    out, S, Z = o.forward(q, k, v, feature_map=fm, gamma=gamma, normalize=norm, eps=eps,
                          S_init=S0, Z_init=Z0 if norm else None)
    L = float(np.sum(dout * out) + np.sum(dSf * S))
    return L + (float(np.sum(dZf * Z)) if norm else 0.0)


def _finite_differences(o, q, k, v, dout, S0, dSf, fm, gamma, norm=False, eps=0.0, Z0=None,
                        dZf=None):
    # Inputs are float32: step 2^-10 is exactly representable on top of values of this size.
    h = 2.0 ** -10
    loss = lambda q_, k_, v_, S_, Z_: _loss(o, q_, k_, v_, dout, S_, dSf, fm, gamma, norm, eps,
                                            Z_, dZf)
    grads = []
    for which, arr in (("q", q), ("k", k), ("v", v)):
        g = np.zeros(arr.shape)
        for idx in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += np.float32(h)
            minus[idx] -= np.float32(h)
            args = {"q": q, "k": k, "v": v}
            args[which] = plus
            lp = loss(args["q"], args["k"], args["v"], S0, Z0)
            args[which] = minus
            lm = loss(args["q"], args["k"], args["v"], S0, Z0)
            g[idx] = (lp - lm) / (float(plus[idx]) - float(minus[idx]))
        grads.append(g)
    for which, arr in (("S", S0), ("Z", Z0)):
        if which == "Z" and not norm:
            grads.append(np.zeros(Z0.shape))
            continue
        g = np.zeros(arr.shape)
        for idx in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += 1e-6
            minus[idx] -= 1e-6
            sp, sm = (plus, minus) if which == "S" else (S0, S0)
            zp, zm = (plus, minus) if which == "Z" else (Z0, Z0)
            g[idx] = (loss(q, k, v, sp, zp) - loss(q, k, v, sm, zm)) / 2e-6
        grads.append(g)
    return grads


def _autograd_parallel(q, k, v, dout, S0, dSf, fm, gamma, norm=False, eps=0.0, Z0=None,
                       dZf=None):
    T = q.shape[2]
    Q, K, V = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    S_init = torch.tensor(S0, dtype=torch.float64, requires_grad=True)
    Z_init = torch.tensor(Z0, dtype=torch.float64, requires_grad=True)
    g = torch.tensor([1.0] * q.shape[1] if gamma is None else gamma, dtype=torch.float64)
    t = torch.arange(T, dtype=torch.float64)
    dist = t[:, None] - t[None, :]
    D = torch.where(dist >= 0, g[:, None, None] ** dist.clamp(min=0), torch.zeros(()))  # [H,T,T]
    fq, fk = _phi(Q, fm), _phi(K, fm)
    A = (fq @ fk.transpose(-1, -2)) * D
    theta = g[:, None, None] ** (t[:, None] + 1)                                        # [H,T,1]
    num = A @ V + theta * (fq @ S_init)
    wS = g[:, None] ** (T - 1 - t)                                                      # [H,T]
    S = torch.einsum("bhti,bhtj,ht->bhij", fk, V, wS) + (g ** T)[None, :, None, None] * S_init
    L = (torch.tensor(dSf) * S).sum()
    if norm:
        den = A.sum(-1, keepdim=True) + theta * (fq @ Z_init[..., None]) + eps
        out = num / den
        Z = torch.einsum("bhti,ht->bhi", fk, wS) + (g ** T)[None, :, None] * Z_init
        L = L + (torch.tensor(dZf) * Z).sum()
    else:
        out = num
    L = L + (torch.tensor(dout) * out).sum()
    grads = torch.autograd.grad(L, (Q, K, V, S_init, Z_init), allow_unused=True)
    return [np.zeros(Z0.shape) if x is None else x.numpy() for x in grads]


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def _backward_pins(o: Oracle) -> dict[str, bool]:
    res = {}
    for fm in ("identity", "elu1"):
        for gamma in (None, [0.9, 0.6]):
            tag = f"{fm}_{'decay' if gamma else 'nodecay'}"
            q, k, v, dout, S0, dSf, Z0, dZf = _problem(1, fm)
            got = o.backward(q, k, v, dout, feature_map=fm, gamma=gamma, S_init=S0, dS_final=dSf)
            fd = _finite_differences(o, q, k, v, dout, S0, dSf, fm, gamma, Z0=Z0)
            res[f"finite_differences_{tag}"] = all(_rel(a, b) < 1e-5 for a, b in zip(got[:4], fd))
            ag = _autograd_parallel(q, k, v, dout, S0, dSf, fm, gamma, Z0=Z0)
            res[f"autograd_parallel_{tag}"] = all(_rel(a, b) < 1e-10 for a, b in zip(got[:4], ag))
            res[f"no_normaliser_gradient_{tag}"] = float(np.max(np.abs(got[4]))) == 0.0
    # The normalised form (ELU + 1, whose features keep the denominators positive), with an
    # initial normaliser, a final normaliser gradient and eps.
    for gamma in (None, [0.9, 0.6]):
        tag = f"normalised_{'decay' if gamma else 'nodecay'}"
        q, k, v, dout, S0, dSf, Z0, dZf = _problem(3, "elu1")
        kw = dict(norm=True, eps=0.25, Z0=Z0, dZf=dZf)
        got = o.backward(q, k, v, dout, feature_map="elu1", gamma=gamma, normalize=True,
                         eps=0.25, S_init=S0, Z_init=Z0, dS_final=dSf, dZ_final=dZf)
        fd = _finite_differences(o, q, k, v, dout, S0, dSf, "elu1", gamma, **kw)
        res[f"finite_differences_{tag}"] = all(_rel(a, b) < 1e-5 for a, b in zip(got, fd))
        ag = _autograd_parallel(q, k, v, dout, S0, dSf, "elu1", gamma, **kw)
        res[f"autograd_parallel_{tag}"] = all(_rel(a, b) < 1e-10 for a, b in zip(got, ag))
    # gamma = 0: o_t = (phi(q_t) . phi(k_t)) v_t, so
    # dq_t = (do_t . v_t) phi(k_t) phi'(q_t), dk_t = (do_t . v_t) phi(q_t) phi'(k_t),
    # dv_t = (phi(q_t) . phi(k_t)) do_t, and nothing reaches S_init.
    q, k, v, dout, S0, dSf, Z0, dZf = _problem(2, "elu1")
    dq, dk, dv, dS0, _ = o.backward(q, k, v, dout, feature_map="elu1", gamma=[0.0, 0.0],
                                    S_init=S0)
    fq, fk = (_phi(torch.tensor(a, dtype=torch.float64), "elu1").numpy() for a in (q, k))
    dphi = lambda a: np.where(a > 0, 1.0, np.exp(a.astype(np.float64)))
    dov = np.sum(dout * v, -1, keepdims=True)
    res["gamma_zero"] = (_rel(dq, dov * fk * dphi(q)) < 1e-13 and _rel(dk, dov * fq * dphi(k)) < 1e-13
                         and _rel(dv, np.sum(fq * fk, -1, keepdims=True) * dout) < 1e-13
                         and float(np.max(np.abs(dS0))) == 0.0)
    # gamma = 0, normalised with eps: o_t = c_t v_t with c_t = a_t / (a_t + eps), a_t =
    # phi(q_t) . phi(k_t); dc/da = eps / (a + eps)^2.
    eps = 0.5
    dq, dk, dv, dS0, dZ0 = o.backward(q, k, v, dout, feature_map="elu1", gamma=[0.0, 0.0],
                                      normalize=True, eps=eps, S_init=S0, Z_init=Z0)
    a = np.sum(fq * fk, -1, keepdims=True)
    dc = dov * eps / (a + eps) ** 2
    res["gamma_zero_normalised"] = (
        _rel(dq, dc * fk * dphi(q)) < 1e-13 and _rel(dk, dc * fq * dphi(k)) < 1e-13
        and _rel(dv, a / (a + eps) * dout) < 1e-13
        and float(np.max(np.abs(dS0))) == 0.0 and float(np.max(np.abs(dZ0))) == 0.0)
    # Normalised, eps = 0, no initial state, every v row the same vector: o_t is that row
    # whatever q and k are, so dq = dk = 0 (to rounding) and sum_t dv_t = sum_t do_t.
    q, k, v, dout, _, _, _, _ = _problem(4, "elu1")
    v = np.broadcast_to(v[:, :, :1], v.shape).copy()
    for gamma in (None, [0.8, 0.3]):
        dq, dk, dv, _, _ = o.backward(q, k, v, dout, feature_map="elu1", gamma=gamma,
                                      normalize=True)
        scale = float(np.max(np.abs(dout))) * float(np.max(np.abs(v)))
        res[f"constant_v_{'decay' if gamma else 'nodecay'}"] = (
            float(np.max(np.abs(dq))) < 1e-12 * scale and float(np.max(np.abs(dk))) < 1e-12 * scale
            and _rel(dv.sum(2), dout.sum(2)) < 1e-12)
    return res


def test_backward_pins_hold():
    res = _backward_pins(default_oracle())
    assert all(res.values()), res


BACKWARD_MUTANTS = {
    "reverse_sweep_decays_current_token": ("Gi[j] += fqi * dnt[j];",
                                           "Gi[j] += fqi * dnt[j] * g;"),
    "reverse_sweep_without_decay": ("for (double& x : G) x *= g;", "for (double& x : G) x *= 1.0;"),
    "dq_without_feature_derivative": (
        "p.dq[(bh * T + t) * dk + i] = acc * feature_map_derivative(x, p.fm);",
        "p.dq[(bh * T + t) * dk + i] = acc;"),
    "dv_uses_query_features": (
        "acc += G[static_cast<size_t>(i) * dv + j] * fk[i];",
        "acc += G[static_cast<size_t>(i) * dv + j] * "
        "feature_map(static_cast<double>(q[t * dk + i]), p.fm);"),
    "final_state_gradient_dropped": ("G[e] = p.dS_final[bh * dk * dv + e];", "G[e] = 0.0;"),
    "dq_contracts_the_state_with_v": (
        "acc += Si[j] * dn[static_cast<size_t>(t) * dv + j];",
        "acc += Si[j] * static_cast<double>(v[t * dv + j]);"),
    "denominator_gradient_sign": ("dd[static_cast<size_t>(t)] = -don / (den * den);",
                                  "dd[static_cast<size_t>(t)] = don / (den * den);"),
    "numerator_gradient_not_divided": (
        "dn[static_cast<size_t>(t) * dv + j] = dout[t * dv + j] / den;",
        "dn[static_cast<size_t>(t) * dv + j] = dout[t * dv + j];"),
    "dq_drops_the_normaliser_term": ("acc += Z[i] * dd[static_cast<size_t>(t)];", "acc += 0.0;"),
    "dk_drops_the_normaliser_gradient": ("double acc = gz[i];", "double acc = 0.0;"),
    "normaliser_gradient_without_decay": ("for (double& x : gz) x *= g;",
                                          "for (double& x : gz) x *= 1.0;"),
    "eps_dropped": ("den = p.eps;", "den = 0.0;"),
    "final_normaliser_gradient_dropped": ("gz[i] = p.dZ_final[bh * dk + i];", "gz[i] = 0.0;"),
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
