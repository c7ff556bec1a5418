"""GPU parity of the backward pass (the unnormalised form's gradients) against the oracle.

The oracle's backward is the fp64 reverse sweep of the state gradient, pinned by finite
differences and by autograd through the parallel form (test_oracle_backward.py).  The CUDA
path runs three prefills plus element-wise kernels; each gradient is compared element by
element on the same inputs (bf16 inputs: the oracle gets the same bf16-rounded values).
Tolerances: max |err| <= 2e-2 * rms(oracle) for bf16 inputs, 1e-4 * rms for float32.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from chunked_causal_linear_b200 import binding as B
from chunked_causal_linear_b200.workloads import WORKLOADS, Workload, make_inputs
from gpu_common import (TOL_BF16, TOL_F32, assert_close, assert_close_rounded_out, gammas_for,
                        to_np)
from oracle.oracle import default_oracle

pytestmark = pytest.mark.gpu

# (feature map, decay)
MODES = {"retention": ("identity", True), "identity": ("identity", False),
         "elu1": ("elu1", False), "elu1_decay": ("elu1", True)}


def _problem(mode, T, *, dtype="bf16", dk=128, dv=128, Bn=2, H=3, seed=0, states=False):
    fm, decay = MODES[mode]
    d = max(dk, dv)
    w = Workload("bwd", B=Bn, H=H, T=T, dk=dk, dv=dv, C=64, dtype=dtype,
                 scale=1.0 / math.sqrt(d) if fm == "identity" else 0.5, feature_map=fm,
                 decay=decay, normalize=False)
    q, k, v = make_inputs(w, seed=seed, device="cuda", gen_device="cpu")
    g = torch.Generator().manual_seed(1000 + seed)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    do = torch.randn((Bn, H, T, dv), generator=g).to(tdt).cuda()
    gamma = gammas_for(H, seed) if decay else None
    S0 = dSf = None
    if states:
        S0 = (torch.randn((Bn, H, dk, dv), generator=g) * 0.3).cuda()
        dSf = torch.randn((Bn, H, dk, dv), generator=g).cuda()
    return fm, q, k, v, do, gamma, S0, dSf


def _oracle(fm, q, k, v, do, gamma, S0, dSf):
    return default_oracle().backward(to_np(q), to_np(k), to_np(v), to_np(do).astype(np.float64),
                                     feature_map=fm, gamma=gamma,
                                     S_init=None if S0 is None else to_np(S0).astype(np.float64),
                                     dS_final=None if dSf is None else to_np(dSf).astype(np.float64))


def _check(got, ref, tol, rounded=False):
    names = ("grad_q", "grad_k", "grad_v", "grad_S_init")
    for name, g, r in zip(names, got, ref):
        if g is None:
            continue
        if rounded and name != "grad_S_init":
            assert_close_rounded_out(to_np(g), r, tol, name)
        else:
            assert_close(to_np(g), r, tol, name)


@pytest.mark.parametrize("mode", sorted(MODES))
@pytest.mark.parametrize("path,algorithm,T", [
    ("tensor_core", "auto", 1000), ("tensor_core", "auto", 3001), ("tensor_core", "chunked", 700),
    ("fma", "chunked", 333)])
def test_backward_matches_oracle(mode, path, algorithm, T):
    # T = 3001 at C = 64 is 47 chunks, a ragged last chunk; the log-depth scan's reduce /
    # totals / sweep kernels run in every pass.
    fm, q, k, v, do, gamma, _, _ = _problem(mode, T)
    got = B.lin_attn_backward(q, k, v, do, feature_map=fm, gamma=gamma, out_dtype="f32",
                              kernel_path=path, algorithm=algorithm)
    torch.cuda.synchronize()
    _check(got, _oracle(fm, q, k, v, do, gamma, None, None), TOL_BF16)


@pytest.mark.parametrize("mode", sorted(MODES))
@pytest.mark.parametrize("algorithm", ["auto", "chunked"])
def test_backward_with_initial_and_final_states(mode, algorithm):
    fm, q, k, v, do, gamma, S0, dSf = _problem(mode, 1500, states=True)
    got = B.lin_attn_backward(q, k, v, do, S_init=S0, grad_S_final=dSf, want_grad_S_init=True,
                              feature_map=fm, gamma=gamma, out_dtype="f32", algorithm=algorithm,
                              segment_chunks=3 if algorithm == "auto" else 0)
    torch.cuda.synchronize()
    _check(got, _oracle(fm, q, k, v, do, gamma, S0, dSf), TOL_BF16)


@pytest.mark.parametrize("mode", ["retention", "elu1_decay"])
def test_backward_small_and_extreme_decays(mode):
    # gamma = 0, 1e-7 (below 2^-20: the final-state gradient's terms are added directly),
    # 2^-19 (just above: divided by gamma), 0.5 and 1.
    fm, q, k, v, do, _, S0, dSf = _problem(mode, 700, H=5, states=True)
    gamma = [0.0, 1e-7, 2.0 ** -19, 0.5, 1.0]
    got = B.lin_attn_backward(q, k, v, do, S_init=S0, grad_S_final=dSf, want_grad_S_init=True,
                              feature_map=fm, gamma=gamma, out_dtype="f32")
    torch.cuda.synchronize()
    _check(got, _oracle(fm, q, k, v, do, gamma, S0, dSf), TOL_BF16)


@pytest.mark.parametrize("mode", sorted(MODES))
def test_backward_fp32(mode):
    fm, q, k, v, do, gamma, S0, dSf = _problem(mode, 300, dtype="f32", dk=32, dv=48,
                                               states=True)
    got = B.lin_attn_backward(q, k, v, do, S_init=S0, grad_S_final=dSf, want_grad_S_init=True,
                              chunk=32, feature_map=fm, gamma=gamma)
    torch.cuda.synchronize()
    _check(got, _oracle(fm, q, k, v, do, gamma, S0, dSf), TOL_F32)


@pytest.mark.parametrize("mode", ["retention", "elu1"])
def test_backward_bf16_gradients(mode):
    fm, q, k, v, do, gamma, _, _ = _problem(mode, 900)
    got = B.lin_attn_backward(q, k, v, do, feature_map=fm, gamma=gamma)
    torch.cuda.synchronize()
    assert all(g.dtype == torch.bfloat16 for g in got[:3])
    _check(got, _oracle(fm, q, k, v, do, gamma, None, None), TOL_BF16, rounded=True)


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64), (64, 64)])
def test_backward_unequal_head_dims(dk, dv):
    fm, q, k, v, do, gamma, S0, dSf = _problem("retention", 777, dk=dk, dv=dv, states=True)
    got = B.lin_attn_backward(q, k, v, do, S_init=S0, grad_S_final=dSf, want_grad_S_init=True,
                              feature_map=fm, gamma=gamma, out_dtype="f32")
    torch.cuda.synchronize()
    _check(got, _oracle(fm, q, k, v, do, gamma, S0, dSf), TOL_BF16)


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65])
def test_backward_short_sequences(T):
    fm, q, k, v, do, gamma, S0, dSf = _problem("retention", T, states=True)
    got = B.lin_attn_backward(q, k, v, do, S_init=S0, grad_S_final=dSf, want_grad_S_init=True,
                              feature_map=fm, gamma=gamma, out_dtype="f32")
    torch.cuda.synchronize()
    _check(got, _oracle(fm, q, k, v, do, gamma, S0, dSf), TOL_BF16)


def test_backward_zero_tokens():
    fm, q, k, v, do, gamma, S0, dSf = _problem("retention", 0, states=True)
    gq, gk, gv, gS = B.lin_attn_backward(q, k, v, do, S_init=S0, grad_S_final=dSf,
                                         want_grad_S_init=True, feature_map=fm, gamma=gamma)
    torch.cuda.synchronize()
    assert gq.numel() == gk.numel() == gv.numel() == 0
    assert torch.equal(gS, dSf)
    _, _, _, gS0 = B.lin_attn_backward(q, k, v, do, want_grad_S_init=True, feature_map=fm,
                                       gamma=gamma)
    torch.cuda.synchronize()
    assert not torch.any(gS0)


def test_backward_is_deterministic_and_uses_the_given_workspace():
    fm, q, k, v, do, gamma, S0, dSf = _problem("retention", 2000, states=True)
    n = B.lin_attn_backward_workspace_bytes(q, v, S_init=True, grad_S_final=True, gamma=gamma,
                                            out_dtype="f32")
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    kw = dict(S_init=S0, grad_S_final=dSf, want_grad_S_init=True, feature_map=fm, gamma=gamma,
              out_dtype="f32")
    a = B.lin_attn_backward(q, k, v, do, workspace=ws, **kw)
    b = B.lin_attn_backward(q, k, v, do, **kw)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    with pytest.raises(B.LinAttnError):
        B.lin_attn_backward(q, k, v, do, workspace=ws[: n - 256], **kw)


def test_backward_full_size_retention_sampled_heads():
    """The 128k-token retention workload (B=1, H=32, T=131072, d=128) in the benchmark's
    configuration; the oracle recomputes heads 0 and 31 in full."""
    w = WORKLOADS["retention_128k"]
    q, k, v = make_inputs(w, seed=0, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(5)
    do = torch.randn(q.shape[:3] + (w.dv,), generator=g, device="cuda").to(torch.bfloat16)
    got = B.lin_attn_backward(q, k, v, do, feature_map=w.feature_map, gamma=w.gammas(),
                              out_dtype="f32", kernel_path="tensor_core")
    torch.cuda.synchronize()
    gam = w.gammas()
    for h in (0, 31):
        sl = lambda t: t[:, h:h + 1]
        ref = default_oracle().backward(to_np(sl(q)), to_np(sl(k)), to_np(sl(v)),
                                        to_np(sl(do)).astype(np.float64),
                                        feature_map=w.feature_map, gamma=[gam[h]])
        for name, x, r in zip(("grad_q", "grad_k", "grad_v"), got[:3], ref[:3]):
            assert_close(to_np(sl(x)), r, TOL_BF16, f"head {h} {name}")


# ---------------------------------------------------------------------------------------
# The normalised form (ELU+1).

def _norm_problem(T, *, decay=False, dtype="bf16", dk=128, dv=128, H=3, seed=0, states=False):
    w = Workload("bwdn", B=2, H=H, T=T, dk=dk, dv=dv, C=64, dtype=dtype, scale=0.5,
                 feature_map="elu1", decay=decay, normalize=True)
    q, k, v = make_inputs(w, seed=seed, device="cuda", gen_device="cpu")
    g = torch.Generator().manual_seed(2000 + seed)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    do = torch.randn((2, H, T, dv), generator=g).to(tdt).cuda()
    gamma = gammas_for(H, seed) if decay else None
    st = {}
    if states:
        st = dict(S_init=(torch.randn((2, H, dk, dv), generator=g) * 0.3).cuda(),
                  Z_init=(torch.rand((2, H, dk), generator=g) * 5.0 + 1.0).cuda(),
                  grad_S_final=torch.randn((2, H, dk, dv), generator=g).cuda(),
                  grad_Z_final=torch.randn((2, H, dk), generator=g).cuda())
    return q, k, v, do, gamma, st


def _norm_case(q, k, v, do, gamma, st, *, eps=0.0, chunk=64, **kw):
    got = B.lin_attn_backward(q, k, v, do, chunk=chunk, feature_map="elu1", gamma=gamma,
                              normalize=True, eps=eps, want_grad_S_init=True,
                              want_grad_Z_init=True, **st, **kw)
    torch.cuda.synchronize()
    f64 = lambda t: None if t is None else to_np(t).astype(np.float64)
    ref = default_oracle().backward(to_np(q), to_np(k), to_np(v), to_np(do).astype(np.float64),
                                    feature_map="elu1", gamma=gamma, normalize=True, eps=eps,
                                    S_init=f64(st.get("S_init")), Z_init=f64(st.get("Z_init")),
                                    dS_final=f64(st.get("grad_S_final")),
                                    dZ_final=f64(st.get("grad_Z_final")))
    return got, ref


def _check_norm(got, ref, tol, rounded=False):
    for name, g, r in zip(("grad_q", "grad_k", "grad_v", "grad_S_init", "grad_Z_init"), got, ref):
        if rounded and name in ("grad_q", "grad_k", "grad_v"):
            assert_close_rounded_out(to_np(g), r, tol, name)
        else:
            assert_close(to_np(g), r, tol, name)


@pytest.mark.parametrize("decay", [False, True])
@pytest.mark.parametrize("path,algorithm,T", [
    ("tensor_core", "auto", 1000), ("tensor_core", "auto", 3001), ("tensor_core", "chunked", 700),
    ("fma", "chunked", 333)])
def test_normalised_backward_matches_oracle(decay, path, algorithm, T):
    q, k, v, do, gamma, st = _norm_problem(T, decay=decay)
    got, ref = _norm_case(q, k, v, do, gamma, st, out_dtype="f32", kernel_path=path,
                          algorithm=algorithm)
    _check_norm(got, ref, TOL_BF16)


@pytest.mark.parametrize("decay", [False, True])
@pytest.mark.parametrize("T", [1, 65, 1500])
def test_normalised_backward_with_states_and_eps(decay, T):
    q, k, v, do, gamma, st = _norm_problem(T, decay=decay, states=True)
    got, ref = _norm_case(q, k, v, do, gamma, st, eps=0.5, out_dtype="f32")
    _check_norm(got, ref, TOL_BF16)


def test_normalised_backward_fp32():
    q, k, v, do, gamma, st = _norm_problem(300, dtype="f32", dk=32, dv=48, decay=True,
                                           states=True)
    got, ref = _norm_case(q, k, v, do, gamma, st, eps=0.25, chunk=32)
    _check_norm(got, ref, TOL_F32)


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_normalised_backward_other_dims(dk, dv):
    # d = 64 is the 4096-token normalised workload's head size
    q, k, v, do, gamma, st = _norm_problem(2000, dk=dk, dv=dv)
    got, ref = _norm_case(q, k, v, do, gamma, st, out_dtype="f32")
    _check_norm(got, ref, TOL_BF16)


def test_normalised_backward_bf16_gradients():
    q, k, v, do, gamma, st = _norm_problem(900)
    got, ref = _norm_case(q, k, v, do, gamma, st)
    assert all(g.dtype == torch.bfloat16 for g in got[:3])
    _check_norm(got, ref, TOL_BF16, rounded=True)


def test_normalised_backward_zero_tokens():
    q, k, v, do, gamma, st = _norm_problem(0, states=True)
    *_, gS, gZ = B.lin_attn_backward(q, k, v, do, feature_map="elu1", normalize=True,
                                     want_grad_S_init=True, want_grad_Z_init=True, **st)
    torch.cuda.synchronize()
    assert torch.equal(gS, st["grad_S_final"]) and torch.equal(gZ, st["grad_Z_final"])


def test_normalised_backward_full_size_sampled_heads():
    """The 16,000-token normalised workload (B=2, H=32, d=128, ELU+1) in the benchmark's
    configuration; the oracle recomputes (b, h) = (0, 0) and (1, 31) in full."""
    w = WORKLOADS["ragged_b2h32"]
    q, k, v = make_inputs(w, seed=0, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(5)
    do = torch.randn(q.shape[:3] + (w.dv,), generator=g, device="cuda").to(torch.bfloat16)
    got = B.lin_attn_backward(q, k, v, do, feature_map="elu1", normalize=True,
                              out_dtype="f32", kernel_path="tensor_core")
    torch.cuda.synchronize()
    for b, h in ((0, 0), (1, 31)):
        sl = lambda t: t[b:b + 1, h:h + 1]
        ref = default_oracle().backward(to_np(sl(q)), to_np(sl(k)), to_np(sl(v)),
                                        to_np(sl(do)).astype(np.float64), feature_map="elu1",
                                        normalize=True)
        for name, x, r in zip(("grad_q", "grad_k", "grad_v"), got[:3], ref[:3]):
            assert_close(to_np(sl(x)), r, TOL_BF16, f"({b},{h}) {name}")


def test_normalised_backward_small_and_extreme_decays():
    # gamma = 0, 1e-7 (below 2^-20: the final-state gradient's terms are added directly),
    # 2^-19, 0.5 and 1, with every state gradient given and requested
    q, k, v, do, _, st = _norm_problem(700, decay=True, H=5, states=True)
    gamma = [0.0, 1e-7, 2.0 ** -19, 0.5, 1.0]
    got, ref = _norm_case(q, k, v, do, gamma, st, eps=0.1, out_dtype="f32")
    _check_norm(got, ref, TOL_BF16)
