"""Prefill from a given initial state, states-only runs, the state fold of a sequence
split into parts, and the sequence-sharded prefill emulated part by part on one GPU.

The oracle's token loop takes the same initial state (S_0 = S_init, Z_0 = Z_init), so the
comparisons are element by element against it at the usual tolerances.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from chunked_causal_linear_b200 import binding as B
from chunked_causal_linear_b200.ranks import RankInfo
from chunked_causal_linear_b200.seqshard import part_ranges, prefill_sequence_sharded
from chunked_causal_linear_b200.workloads import Workload, make_inputs
from gpu_common import TOL_BF16, TOL_F32, assert_close, gammas_for, to_np
from oracle.oracle import default_oracle

pytestmark = pytest.mark.gpu

MODES = {"retention": ("identity", True, False), "norm": ("elu1", False, True)}


def _problem(mode, T, dtype="bf16", d=128, H=3, seed=0):
    fm, decay, norm = MODES[mode]
    w = Workload("init", B=2, H=H, T=T, dk=d, dv=d, C=64, dtype=dtype,
                 scale=1.0 / math.sqrt(d) if fm == "identity" else 0.5, feature_map=fm,
                 decay=decay, normalize=norm)
    q, k, v = make_inputs(w, seed=seed, device="cuda", gen_device="cpu")
    gamma = gammas_for(H, seed) if decay else None
    g = torch.Generator().manual_seed(100 + seed)
    S0 = (torch.randn((2, H, d, d), generator=g) * 0.3).cuda()
    # A plausible accumulated normaliser: positive, so that denominators stay positive.
    Z0 = (torch.rand((2, H, d), generator=g) * 5.0 + 1.0).cuda() if norm else None
    return w, q, k, v, gamma, S0, Z0


def _oracle(w, q, k, v, gamma, S0, Z0, want_out=True):
    return default_oracle().forward(to_np(q), to_np(k), to_np(v), feature_map=w.feature_map,
                                    gamma=gamma, normalize=w.normalize,
                                    S_init=to_np(S0).astype(np.float64),
                                    Z_init=None if Z0 is None else to_np(Z0).astype(np.float64),
                                    want_out=want_out)


@pytest.mark.parametrize("mode", sorted(MODES))
@pytest.mark.parametrize("path,algorithm,scan,T", [
    ("tensor_core", "segmented", "logdepth", 1000), ("tensor_core", "segmented", "logdepth", 5000),
    ("tensor_core", "chunked", "logdepth", 1000), ("tensor_core", "chunked", "logdepth", 3000),
    ("tensor_core", "chunked", "sequential", 1000), ("fma", "chunked", "logdepth", 700)])
def test_prefill_from_an_initial_state(mode, path, algorithm, scan, T):
    # T = 3000 at C = 64 is 47 chunks: the log-depth scan's reduce / totals / sweep path;
    # T = 1000 (16 chunks) its single in-place pass; segmented T = 5000 with two-chunk
    # segments scans 40 segments.
    w, q, k, v, gamma, S0, Z0 = _problem(mode, T)
    out, S, Z = B.lin_attn_prefill(q, k, v, chunk=64, feature_map=w.feature_map, gamma=gamma,
                                   normalize=w.normalize, scan=scan, kernel_path=path,
                                   algorithm=algorithm, out_dtype="f32", S_init=S0, Z_init=Z0,
                                   segment_chunks=2 if algorithm == "segmented" else 0)
    torch.cuda.synchronize()
    o_ref, S_ref, Z_ref = _oracle(w, q, k, v, gamma, S0, Z0)
    assert_close(to_np(out), o_ref, TOL_BF16, "out")
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final")
    if w.normalize:
        assert_close(to_np(Z), Z_ref, TOL_BF16, "Z_final")


def test_fp32_prefill_from_an_initial_state():
    w, q, k, v, gamma, S0, Z0 = _problem("norm", 300, dtype="f32", d=32)
    out, S, Z = B.lin_attn_prefill(q, k, v, chunk=32, feature_map="elu1", normalize=True,
                                   S_init=S0, Z_init=Z0)
    torch.cuda.synchronize()
    o_ref, S_ref, Z_ref = _oracle(w, q, k, v, None, S0, Z0)
    assert_close(to_np(out), o_ref, TOL_F32, "out")
    assert_close(to_np(S), S_ref, TOL_F32, "S_final")
    assert_close(to_np(Z), Z_ref, TOL_F32, "Z_final")


@pytest.mark.parametrize("mode", sorted(MODES))
@pytest.mark.parametrize("algorithm", ["chunked", "segmented"])
def test_states_only_and_in_place_state(mode, algorithm):
    w, q, k, v, gamma, S0, Z0 = _problem(mode, 1000)
    kw = dict(chunk=64, feature_map=w.feature_map, gamma=gamma, normalize=w.normalize,
              kernel_path="tensor_core", algorithm=algorithm, out_dtype="f32")
    out, S, Z = B.lin_attn_prefill(q, k, v, S_init=S0, Z_init=Z0, **kw)
    # states only: the same final state, bit for bit, and no output written
    none, S2, Z2 = B.lin_attn_prefill(q, k, v, S_init=S0, Z_init=Z0, states_only=True, **kw)
    # the state updated in place (S_init is S_final)
    S3, Z3 = S0.clone(), (Z0.clone() if Z0 is not None else None)
    out3, _, _ = B.lin_attn_prefill(q, k, v, None, S3, Z3, S_init=S3, Z_init=Z3, **kw)
    torch.cuda.synchronize()
    assert none is None
    assert torch.equal(S2, S) and torch.equal(S3, S) and torch.equal(out3, out)
    if w.normalize:
        assert torch.equal(Z2, Z) and torch.equal(Z3, Z)


def test_zero_tokens_return_the_initial_state():
    w, q, k, v, _, S0, Z0 = _problem("norm", 0)
    _, S, Z = B.lin_attn_prefill(q, k, v, feature_map="elu1", normalize=True, S_init=S0,
                                 Z_init=Z0)
    torch.cuda.synchronize()
    assert torch.equal(S, S0) and torch.equal(Z, Z0)


@pytest.mark.parametrize("decay", [False, True])
def test_combine_states_folds_parts_in_order(decay):
    g = torch.Generator().manual_seed(7)
    parts, Bn, H, d = 5, 2, 3, 16
    Sp = torch.randn((parts, Bn, H, d, d), generator=g).cuda()
    Zp = torch.rand((parts, Bn, H, d), generator=g).cuda()
    toks = [64, 128, 3, 0, 200]
    gamma = [0.9, 0.5, 1.0] if decay else None
    gm = np.ones(H) if gamma is None else np.asarray(gamma, dtype=np.float32)
    for upto in range(parts + 1):
        S, Z = B.lin_attn_combine_states(Sp, Zp, upto, toks, gamma=gamma)
        torch.cuda.synchronize()
        P, Q = np.zeros((Bn, H, d, d)), np.zeros((Bn, H, d))
        for j in range(upto):
            a = gm.astype(np.float64) ** toks[j]
            P = a[None, :, None, None] * P + to_np(Sp[j])
            Q = a[None, :, None] * Q + to_np(Zp[j])
        np.testing.assert_allclose(to_np(S), P, rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(to_np(Z), Q, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("mode", sorted(MODES))
@pytest.mark.parametrize("world", [2, 4])
def test_sequence_sharded_prefill_part_by_part(mode, world):
    # The ranks of a sequence-sharded prefill run one after another on one GPU (nothing
    # waits on another rank): each range's states-only pass, then each rank's fold and
    # prefill from the gathered states.  The concatenated outputs must match the oracle
    # on the whole sequence, and the last range's final state the sequence's.
    w, q, k, v, gamma, _, _ = _problem(mode, 2500)
    kw = dict(chunk=64, feature_map=w.feature_map, kernel_path="tensor_core", out_dtype="f32")
    rng = part_ranges(w.T, world, 64)
    toks = [n for _, n in rng]
    sl = lambda t, s0, n: t[:, :, s0:s0 + n].contiguous()
    states = [B.lin_attn_prefill(sl(q, s0, n), sl(k, s0, n), sl(v, s0, n), gamma=gamma,
                                 normalize=w.normalize, states_only=True, **kw)
              for s0, n in rng]
    S_all = torch.stack([s[1] for s in states])
    Z_all = torch.stack([s[2] for s in states]) if w.normalize else None
    outs, finals = [], []
    for r, (s0, n) in enumerate(rng):
        # the collective is replaced by the stack of every range's state
        def gather(x, info, S_loc=states[r][1]):
            return S_all if x is S_loc else Z_all

        out, S_fin, Z_fin, _, _ = prefill_sequence_sharded(
            sl(q, s0, n), sl(k, s0, n), sl(v, s0, n), info=RankInfo(r, world, 0),
            part_tokens=toks, gamma=gamma, normalize=w.normalize,
            prefill=_reuse_first_pass(states[r]), gather=gather, **kw)
        outs.append(out)
        finals.append((S_fin, Z_fin))
    torch.cuda.synchronize()
    o_ref, S_ref, Z_ref = default_oracle().forward(to_np(q), to_np(k), to_np(v),
                                                   feature_map=w.feature_map, gamma=gamma,
                                                   normalize=w.normalize)
    assert_close(to_np(torch.cat(outs, dim=2)), o_ref, TOL_BF16, "out")
    assert_close(to_np(finals[-1][0]), S_ref, TOL_BF16, "S_final")
    if w.normalize:
        assert_close(to_np(finals[-1][1]), Z_ref, TOL_BF16, "Z_final")


def _reuse_first_pass(state):
    """The library prefill, except that the states-only pass returns the tensors already
    computed for this range (so that the stacked 'gathered' states are the same objects)."""
    def prefill(q, k, v, out, *, states_only=False, **kw):
        if states_only:
            return state
        return B.lin_attn_prefill(q, k, v, out, **kw)
    return prefill


def test_host_entry_point_with_an_initial_state():
    w, q, k, v, gamma, S0, Z0 = _problem("norm", 500)
    kw = dict(chunk=64, feature_map="elu1", normalize=True, out_dtype="f32")
    out_d, S_d, Z_d = B.lin_attn_prefill(q, k, v, S_init=S0, Z_init=Z0, **kw)
    torch.cuda.synchronize()
    pin = lambda t: t.cpu().pin_memory()
    out_h = torch.empty(out_d.shape, dtype=out_d.dtype).pin_memory()
    S_h = torch.empty(S_d.shape, dtype=torch.float32).pin_memory()
    Z_h = torch.empty(Z_d.shape, dtype=torch.float32).pin_memory()
    B.lin_attn_prefill_host(pin(q), pin(k), pin(v), out_h, S_h, Z_h, S_init=pin(S0),
                            Z_init=pin(Z0), **kw)
    assert torch.equal(out_h, out_d.cpu())
    assert torch.equal(S_h, S_d.cpu()) and torch.equal(Z_h, Z_d.cpu())
