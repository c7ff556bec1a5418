"""Failure detection, in the forms that fault nothing.

- A bounded wait that runs out: lin_attn_check_wait_timeout makes one thread wait, with a
  short limit, on an mbarrier nothing arrives on.  The kernel must return, the device
  error word must read 5 and be cleared by reading it, and while it is set the
  tensor-core kernels launched afterwards must skip their work (their output stays as it
  was), after which the same call succeeds again.
- An allocation that fails: with LA_FAULT_INJECT=alloc every library-side workspace
  allocation fails before anything is launched, and the entry points return
  LA_ERR_OUT_OF_MEMORY; a caller workspace avoids the allocation and the call succeeds.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from chunked_causal_linear_b200 import binding as B
from chunked_causal_linear_b200.workloads import Workload, make_gates, make_inputs
from gpu_common import TOL_BF16, assert_close, oracle_prefill, to_np

pytestmark = pytest.mark.gpu

LA_ERR_OUT_OF_MEMORY = 3
WAIT_CHECK_CODE = 5


def _small(T=300):
    w = Workload("fd", B=1, H=2, T=T, dk=128, dv=128, C=64, dtype="bf16", scale=128 ** -0.5,
                 feature_map="identity", decay=True, normalize=False)
    q, k, v = make_inputs(w, seed=21, device="cuda", gen_device="cpu")
    return w, q, k, v, [0.9, 0.99]


def test_wait_timeout_sets_and_clears_the_error_word():
    assert B.lin_attn_device_error() == 0
    B.lin_attn_check_wait_timeout(2000)
    torch.cuda.synchronize()  # the kernel returned: the wait gave up
    assert B.lin_attn_device_error() == WAIT_CHECK_CODE
    assert B.lin_attn_device_error() == 0  # reading cleared it


def test_pending_error_makes_later_kernels_skip_their_work():
    w, q, k, v, gamma = _small()
    kw = dict(chunk=64, feature_map="identity", gamma=gamma, normalize=False,
              out_dtype="f32", kernel_path="tensor_core", algorithm="segmented")
    out = torch.full((1, 2, w.T, 128), float("nan"), device="cuda")
    B.lin_attn_check_wait_timeout(1000)
    B.lin_attn_prefill(q, k, v, out, **kw)
    torch.cuda.synchronize()
    assert torch.isnan(out).all(), "a kernel ran although an error was pending"
    assert B.lin_attn_device_error() == WAIT_CHECK_CODE
    out2, S2, _ = B.lin_attn_prefill(q, k, v, **kw)
    torch.cuda.synchronize()
    assert B.lin_attn_device_error() == 0
    o_ref, S_ref, _ = oracle_prefill(q, k, v, feature_map="identity", gamma=gamma,
                                     normalize=False)
    assert_close(to_np(out2), o_ref, TOL_BF16, "out after the error was cleared")
    assert_close(to_np(S2), S_ref, TOL_BF16, "S_final after the error was cleared")


def test_wait_check_rejects_bad_limits():
    with pytest.raises(B.LinAttnError):
        B.lin_attn_check_wait_timeout(0)
    with pytest.raises(B.LinAttnError):
        B.lin_attn_check_wait_timeout(2_000_000)


def test_allocation_failure_injection(monkeypatch):
    w, q, k, v, gamma = _small()
    kw = dict(chunk=64, feature_map="identity", gamma=gamma, normalize=False, out_dtype="f32")
    monkeypatch.setenv("LA_FAULT_INJECT", "alloc")
    with pytest.raises(B.LinAttnError) as e:
        B.lin_attn_prefill(q, k, v, **kw)
    assert e.value.status == LA_ERR_OUT_OF_MEMORY
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(3)).to(q.dtype).cuda()
    with pytest.raises(B.LinAttnError) as e:
        B.lin_attn_backward(q, k, v, dout, feature_map="identity", gamma=gamma, out_dtype="f32")
    assert e.value.status == LA_ERR_OUT_OF_MEMORY
    wg = Workload("fdg", B=1, H=2, T=300, dk=64, dv=64, C=64, dtype="bf16", scale=0.125,
                  feature_map="identity", decay=False, normalize=False)
    qg, kg, vg = make_inputs(wg, seed=2, device="cuda", gen_device="cpu")
    ag = make_gates(wg, seed=2, device="cuda", gen_device="cpu")
    with pytest.raises(B.LinAttnError) as e:
        B.lin_attn_gla_prefill(qg, kg, vg, ag, out_dtype="f32")
    assert e.value.status == LA_ERR_OUT_OF_MEMORY
    # A caller workspace needs no allocation: the call succeeds under the same injection.
    ws = torch.empty(B.lin_attn_prefill_workspace_bytes(1, 2, w.T, 128, 128, 64, False),
                     dtype=torch.uint8, device="cuda")
    out, S, _ = B.lin_attn_prefill(q, k, v, workspace=ws, **kw)
    torch.cuda.synchronize()
    monkeypatch.delenv("LA_FAULT_INJECT")
    out2, S2, _ = B.lin_attn_prefill(q, k, v, **kw)
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(S, S2)
    assert B.lin_attn_device_error() == 0
    assert math.isfinite(float(out.abs().max()))
    assert np.isfinite(to_np(S)).all()
