"""The allocation-free prefill entry point, through the C ABI.

lin_attn_prefill_noalloc serves callers that must not allocate device memory while they
run (a fixed memory budget reserved at start-up, a host framework that owns every
allocation, code that cannot handle a failed allocation): its workspace is a fixed array
in the library's device image.  This file checks it against the ordinary entry point,
bit for bit, on two calls in a row (the array is shared and keeps the previous call's
contents), and that a problem too large for the array is refused before anything is
launched.

The file name sorts last so that a run that stops at the first failure has already run
every other test.
"""

from __future__ import annotations

import ctypes
import math

import pytest
import torch

from chunked_causal_linear_b200 import binding as B
from chunked_causal_linear_b200.workloads import Workload, make_inputs
from gpu_common import gammas_for

pytestmark = pytest.mark.gpu


def _problem(fm, decay, norm, T, seed):
    w = Workload("noalloc", B=2, H=4, T=T, dk=128, dv=128, C=64, dtype="bf16",
                 scale=0.5 if fm == "elu1" else 1.0 / math.sqrt(128), feature_map=fm,
                 decay=decay, normalize=norm)
    q, k, v = make_inputs(w, seed=seed, device="cuda", gen_device="cpu")
    return w, q, k, v, (gammas_for(4, seed) if decay else None)


@pytest.mark.parametrize("fm,decay,norm", [("elu1", False, True), ("identity", True, False)])
def test_noalloc_matches_the_allocating_entry_point_twice(fm, decay, norm):
    # Two different problems back to back, each compared with lin_attn_prefill_ex.
    for call, (T, seed) in enumerate(((1000, 11), (777, 12))):
        w, q, k, v, gamma = _problem(fm, decay, norm, T, seed)
        assert B.lin_attn_prefill_workspace_bytes(w.B, w.H, T, 128, 128, 64, norm) \
            <= B.NOALLOC_SCRATCH_BYTES
        kw = dict(chunk=64, feature_map=fm, gamma=gamma, normalize=norm, out_dtype="f32")
        ref_out, ref_S, ref_Z = B.lin_attn_prefill(q, k, v, **kw)
        out = torch.empty_like(ref_out)
        S = torch.empty_like(ref_S)
        Z = torch.empty_like(ref_Z) if norm else None
        B.lin_attn_prefill_noalloc(q, k, v, out, S, Z, **kw)
        torch.cuda.synchronize()
        # The same deterministic kernels run on both paths (no atomics, a fixed order
        # of every sum), so the results agree bit for bit.
        assert torch.equal(out, ref_out), f"call {call} out"
        assert torch.equal(S, ref_S), f"call {call} S_final"
        if norm:
            assert torch.equal(Z, ref_Z), f"call {call} Z_final"
    assert B.lin_attn_device_error() == 0


def test_noalloc_refuses_a_problem_larger_than_its_array():
    # 64 heads of 4096 tokens at d = 128 need far more than the array holds; the call
    # must fail before touching the (never allocated) tensors.
    a = B.PrefillArgs()
    a.B, a.H, a.T, a.dk, a.dv, a.C = 1, 64, 4096, 128, 128, 64
    a.feature_map, a.normalize, a.dtype = 1, 1, 0
    a.q, a.k, a.v, a.out = 0x100000, 0x200000, 0x300000, 0x400000
    assert B.lin_attn_prefill_workspace_bytes(1, 64, 4096, 128, 128, 64, True) \
        > B.NOALLOC_SCRATCH_BYTES
    assert B.load_library().lin_attn_prefill_noalloc(ctypes.byref(a)) == 2
