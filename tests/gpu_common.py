"""Helpers for the GPU parity tests: run the CUDA path through the C ABI, run the oracle
on the same inputs, compare with the tolerances the tests state."""

from __future__ import annotations

import numpy as np
import torch

from chunked_causal_linear_b200 import binding as B
from oracle.oracle import default_oracle

# max |err| <= TOL * rms(oracle), per output tensor.
TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).numpy()


def rms(x: np.ndarray) -> float:
    return float(np.sqrt(np.mean(np.square(x)))) if x.size else 0.0


def max_rel_rms(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    r = rms(ref)
    if r == 0.0:
        return float(np.max(np.abs(got - ref))) if got.size else 0.0
    return float(np.max(np.abs(got - ref))) / r


def assert_close(got, ref, tol, what=""):
    err = max_rel_rms(got, ref)
    assert np.all(np.isfinite(np.asarray(got))), f"{what}: non-finite values"
    assert err <= tol, f"{what}: max|err|/rms = {err:.3e} > {tol:.1e}"
    return err


def assert_close_rounded_out(got, ref, tol, what=""):
    """Bound for an output stored in bf16: the stated tolerance plus the output's own
    rounding, |err_i| <= tol * rms(ref) + 2^-8 |ref_i| (round-to-nearest-even bf16 moves
    a value by at most 2^-9 relative; 2^-8 also covers a rounding-boundary flip caused by
    the computation's own error)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    bound = tol * (float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0) + 2.0 ** -8 * np.abs(ref)
    excess = np.abs(got - ref) - bound
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    assert float(np.max(excess, initial=-1.0)) <= 0.0, f"{what}: worst excess {np.max(excess):.3e}"


def gpu_prefill(q, k, v, *, C, feature_map, gamma, normalize, **kw):
    """Prefill through the C ABI; bf16 inputs write a float32 output unless told otherwise."""
    if q.dtype == torch.bfloat16:
        kw.setdefault("out_dtype", "f32")
    out, S, Z = B.lin_attn_prefill(q, k, v, chunk=C, feature_map=feature_map, gamma=gamma,
                                   normalize=normalize, **kw)
    torch.cuda.synchronize()
    return out, S, Z


def oracle_prefill(q, k, v, *, feature_map, gamma, normalize, heads=None, want_out=True,
                   S_init=None, Z_init=None):
    """Oracle on host copies of q, k, v (and of the initial state, when given).

    `heads` selects (b, h) pairs (default: all); the selected pairs run as one oracle call
    (one thread each) and come back stacked as [n, T, d] / [n, dk, dv] / [n, dk].
    """
    g = None if gamma is None else np.asarray(gamma, dtype=np.float64)
    if heads is None:
        s0 = None if S_init is None else to_np(S_init).astype(np.float64)
        z0 = None if Z_init is None else to_np(Z_init).astype(np.float64)
        return default_oracle().forward(to_np(q), to_np(k), to_np(v), feature_map=feature_map,
                                        gamma=g, normalize=normalize, want_out=want_out,
                                        S_init=s0, Z_init=z0)
    sel = lambda t: torch.stack([t[b, h] for b, h in heads])[None]
    gs = None if g is None else np.array([g[h] for _, h in heads])
    o, S, Z = default_oracle().forward(to_np(sel(q)), to_np(sel(k)), to_np(sel(v)),
                                       feature_map=feature_map, gamma=gs, normalize=normalize,
                                       want_out=want_out)
    return (None if o is None else o[0]), S[0], Z[0]


def gammas_for(H, seed=0):
    rng = np.random.default_rng(seed)
    return [float(np.float32(x)) for x in rng.uniform(0.85, 0.999, size=H)]
