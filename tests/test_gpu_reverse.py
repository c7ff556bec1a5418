"""The reverse-mode prefill (la_prefill_args.reverse): the recurrence run from token T-1
down to token 0 on tensors kept in memory order.

By definition it is the causal prefill of the time-reversed sequence, so the oracle runs
its ordinary token loop on the reversed inputs and its outputs are reversed back (a
permutation, no arithmetic).  Compared element by element at the bf16 tolerance,
max |err| <= 2e-2 * rms(oracle).
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from chunked_causal_linear_b200 import binding as B
from chunked_causal_linear_b200.workloads import Workload, make_inputs
from gpu_common import TOL_BF16, assert_close, gammas_for, to_np
from oracle.oracle import default_oracle

pytestmark = pytest.mark.gpu

MODES = {"retention": ("identity", True, False), "norm": ("elu1", False, True),
         "identity": ("identity", False, False), "elu1_unnorm": ("elu1", False, False)}


def _problem(mode, T, dk=128, seed=0, H=3):
    fm, decay, norm = MODES[mode]
    w = Workload("rev", B=2, H=H, T=T, dk=dk, dv=128, C=64, dtype="bf16",
                 scale=1.0 / math.sqrt(dk) if fm == "identity" else 0.5, feature_map=fm,
                 decay=decay, normalize=norm)
    q, k, v = make_inputs(w, seed=seed, device="cuda", gen_device="cpu")
    return w, q, k, v, (gammas_for(H, seed) if decay else None)


def _oracle_reversed(w, q, k, v, gamma, S0=None, Z0=None):
    flip = lambda a: np.ascontiguousarray(a[:, :, ::-1])
    o, S, Z = default_oracle().forward(flip(to_np(q)), flip(to_np(k)), flip(to_np(v)),
                                       feature_map=w.feature_map, gamma=gamma,
                                       normalize=w.normalize,
                                       S_init=None if S0 is None else to_np(S0).astype(np.float64),
                                       Z_init=None if Z0 is None else to_np(Z0).astype(np.float64))
    return flip(o), S, Z


@pytest.mark.parametrize("mode", sorted(MODES))
@pytest.mark.parametrize("T,lseg", [(1000, 0), (3001, 0), (3001, 3), (130, 1), (63, 0), (1, 0)])
def test_reverse_prefill_matches_the_reversed_sequence(mode, T, lseg):
    w, q, k, v, gamma = _problem(mode, T)
    out, S, Z = B.lin_attn_prefill(q, k, v, chunk=64, feature_map=w.feature_map, gamma=gamma,
                                   normalize=w.normalize, out_dtype="f32", reverse=True,
                                   algorithm="segmented", segment_chunks=lseg)
    torch.cuda.synchronize()
    o_ref, S_ref, Z_ref = _oracle_reversed(w, q, k, v, gamma)
    assert_close(to_np(out), o_ref, TOL_BF16, "out")
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final")
    if w.normalize:
        assert_close(to_np(Z), Z_ref, TOL_BF16, "Z_final")


@pytest.mark.parametrize("mode", ["retention", "norm"])
def test_reverse_prefill_from_a_state_and_states_only(mode):
    w, q, k, v, gamma = _problem(mode, 2000, dk=64)
    g = torch.Generator().manual_seed(3)
    S0 = (torch.randn((2, 3, 64, 128), generator=g) * 0.3).cuda()
    Z0 = (torch.rand((2, 3, 64), generator=g) * 5 + 1).cuda() if w.normalize else None
    kw = dict(chunk=64, feature_map=w.feature_map, gamma=gamma, normalize=w.normalize,
              out_dtype="f32", reverse=True, S_init=S0, Z_init=Z0)
    out, S, Z = B.lin_attn_prefill(q, k, v, **kw)
    _, S2, Z2 = B.lin_attn_prefill(q, k, v, states_only=True, **kw)
    torch.cuda.synchronize()
    o_ref, S_ref, Z_ref = _oracle_reversed(w, q, k, v, gamma, S0, Z0)
    assert_close(to_np(out), o_ref, TOL_BF16, "out")
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final")
    assert torch.equal(S2, S)
    if w.normalize:
        assert_close(to_np(Z), Z_ref, TOL_BF16, "Z_final")
        assert torch.equal(Z2, Z)


def test_reverse_needs_the_segmented_algorithm():
    w, q, k, v, gamma = _problem("retention", 100)
    with pytest.raises(B.LinAttnError):
        B.lin_attn_prefill(q, k, v, feature_map="identity", gamma=gamma, normalize=False,
                           reverse=True, algorithm="chunked")
