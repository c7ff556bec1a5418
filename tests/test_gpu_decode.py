"""The decode step (one recurrent token for every (b, h)) against the oracle.

The oracle's token loop run for one token from a given state (S_init, Z_init) is the
decode step of "Linear Attention and Retentive Networks ..." (B. Recurrent
Representation).  Shapes cover the clustered tile kernel (dk a multiple of 16 up to 128,
dv a multiple of 4 up to 256: one CTA per 16 state rows, partial outputs added across the
cluster) and the per-head kernel every other shape takes.  Tolerances: 1e-4 rms (float32
inputs), 2e-2 rms plus the output's bf16 rounding (bf16 inputs and output).
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from chunked_causal_linear_b200 import binding as B
from gpu_common import (TOL_BF16, TOL_F32, assert_close, assert_close_rounded_out, gammas_for,
                        to_np)
from oracle.oracle import default_oracle

pytestmark = pytest.mark.gpu


def _case(Bn, H, dk, dv, dtype, seed):
    rng = np.random.default_rng(seed)
    S0 = (rng.standard_normal((Bn, H, dk, dv)) * 0.3).astype(np.float32)
    Z0 = rng.uniform(1, 5, size=(Bn, H, dk)).astype(np.float32)
    qkv = [torch.tensor(rng.standard_normal((Bn, H, d)) * 0.5, dtype=torch.float32)
           for d in (dk, dk, dv)]
    if dtype == "bf16":
        qkv = [t.to(torch.bfloat16) for t in qkv]
    return S0, Z0, qkv


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 48), (64, 64), (64, 128), (128, 128),
                                   (128, 256), (128, 32), (96, 100), (100, 64), (8, 8)])
@pytest.mark.parametrize("fm,norm,decay", [("elu1", True, False), ("identity", False, True),
                                           ("elu1", True, True), ("elu1", False, False)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_from_a_given_state(dk, dv, fm, norm, decay, dtype):
    Bn, H = 2, 3
    S0, Z0, (q, k, v) = _case(Bn, H, dk, dv, dtype, seed=dk * 1000 + dv)
    gamma = gammas_for(H, 7) if decay else None
    S = torch.tensor(S0, device="cuda")
    Z = torch.tensor(Z0, device="cuda")
    out = B.lin_attn_decode_step(q.cuda(), k.cuda(), v.cuda(), S, Z, feature_map=fm,
                                 gamma=gamma, normalize=norm)
    torch.cuda.synchronize()
    f = lambda t: t.float().numpy()[:, :, None]
    o_ref, S_ref, Z_ref = default_oracle().forward(
        f(q), f(k), f(v), feature_map=fm, normalize=norm,
        gamma=None if gamma is None else np.asarray(gamma, dtype=np.float64),
        S_init=S0, Z_init=Z0)
    if dtype == "f32":
        assert_close(to_np(out), o_ref[:, :, 0], TOL_F32, "out")
        tol = TOL_F32
    else:
        assert_close_rounded_out(to_np(out), o_ref[:, :, 0], TOL_BF16, "out")
        tol = TOL_BF16
    assert_close(to_np(S), S_ref, tol, "S")
    # Z is updated (Z <- gamma Z + psi(k)) whenever it is given, normalised or not.
    assert_close(to_np(Z), Z_ref, tol, "Z")


@pytest.mark.parametrize("dk,dv", [(128, 256), (128, 100), (128, 64), (64, 48), (128, 128)])
@pytest.mark.parametrize("fm,norm,decay", [("elu1", True, False), ("identity", False, True)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_64_row_tiles_every_rows_per_thread(dk, dv, fm, norm, decay, dtype):
    """Enough heads for the 64-row tiles (B.H.dk / 64 >= 2 x 148), at value widths that give a
    thread 4, 8 and 16 state rows (dv <= 64, 100 or 128, 256)."""
    Bn, H = (4, 40) if dk == 128 else (8, 40)
    S0, Z0, (q, k, v) = _case(Bn, H, dk, dv, dtype, seed=7 * dk + dv)
    gamma = gammas_for(H, 5) if decay else None
    S = torch.tensor(S0, device="cuda")
    Z = torch.tensor(Z0, device="cuda")
    out = B.lin_attn_decode_step(q.cuda(), k.cuda(), v.cuda(), S, Z, feature_map=fm,
                                 gamma=gamma, normalize=norm)
    torch.cuda.synchronize()
    f = lambda t: t.float().numpy()[:, :, None]
    o_ref, S_ref, Z_ref = default_oracle().forward(
        f(q), f(k), f(v), feature_map=fm, normalize=norm,
        gamma=None if gamma is None else np.asarray(gamma, dtype=np.float64),
        S_init=S0, Z_init=Z0)
    if dtype == "f32":
        assert_close(to_np(out), o_ref[:, :, 0], TOL_F32, "out")
        tol = TOL_F32
    else:
        assert_close_rounded_out(to_np(out), o_ref[:, :, 0], TOL_BF16, "out")
        tol = TOL_BF16
    assert_close(to_np(S), S_ref, tol, "S")
    assert_close(to_np(Z), Z_ref, tol, "Z")


def test_decode_many_heads_and_repeated_steps():
    """B.H = 256 (the size the decode benchmark starts at), eight steps in a row, each step's
    output against the oracle's token loop over the same eight tokens."""
    Bn, H, dk, dv, steps = 8, 32, 128, 128, 8
    rng = np.random.default_rng(11)
    S0 = (rng.standard_normal((Bn, H, dk, dv)) * 0.1).astype(np.float32)
    toks = [torch.tensor(rng.standard_normal((Bn, H, steps, d)) / np.sqrt(128),
                         dtype=torch.float32).to(torch.bfloat16) for d in (dk, dk, dv)]
    gamma = [float(np.float32(1 - 2.0 ** (-5 - 3 * h / 31))) for h in range(H)]
    S = torch.tensor(S0, device="cuda")
    outs = []
    for t in range(steps):
        q, k, v = (x[:, :, t].contiguous().cuda() for x in toks)
        outs.append(B.lin_attn_decode_step(q, k, v, S, None, feature_map="identity",
                                           gamma=gamma, normalize=False))
    torch.cuda.synchronize()
    o_ref, S_ref, _ = default_oracle().forward(
        *(x.float().numpy() for x in toks), feature_map="identity", normalize=False,
        gamma=np.asarray(gamma, dtype=np.float64), S_init=S0)
    got = np.stack([to_np(o) for o in outs], axis=2)
    assert_close_rounded_out(got, o_ref, TOL_BF16, "outputs")
    assert_close(to_np(S), S_ref, TOL_BF16, "S")
