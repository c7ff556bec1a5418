"""The plain prefill entry points, called directly through the C ABI.

`lin_attn_prefill` (bf16 q, k, v and a bf16 output) and `lin_attn_prefill_f32` (float32
throughout, the CUDA-core FMA kernels) are the two signatures the library's contract names
for one prefill call: (q, k, v, out, S_final, Z_final, B, H, T, dk, dv, C, feature_map,
gamma, normalize, stream).  Every other test goes through `lin_attn_prefill_ex`; these call
the two symbols themselves, with ctypes, and compare with the oracle on the same inputs.

Tolerances: max |err| <= 1e-4 rms(oracle) for the float32 path; for the bf16 output the
stated 2e-2 rms bound plus the output's own rounding (assert_close_rounded_out), and 2e-2
rms for the float32 final states.
"""

from __future__ import annotations

import ctypes
import math

import pytest
import torch

from chunked_causal_linear_b200 import binding as B
from chunked_causal_linear_b200.workloads import WORKLOADS, Workload, make_inputs
from gpu_common import (TOL_BF16, TOL_F32, assert_close, assert_close_rounded_out, gammas_for,
                        oracle_prefill, to_np)

pytestmark = pytest.mark.gpu

LA_ERR_INVALID_ARGUMENT, LA_ERR_UNSUPPORTED = 1, 2


def _call(fn_name, q, k, v, out, S, Z, C, feature_map, gamma, normalize):
    lib = B.load_library()
    Bn, H, T, dk = q.shape
    dv = v.shape[-1]
    garr = None
    gptr = None
    if gamma is not None:
        garr = (ctypes.c_float * H)(*[float(g) for g in gamma])
        gptr = ctypes.cast(garr, ctypes.c_void_p)
    stream = torch.cuda.current_stream().cuda_stream
    st = getattr(lib, fn_name)(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               S.data_ptr(), None if Z is None else Z.data_ptr(), Bn, H, T, dk,
                               dv, C, B.FEATURE_MAPS[feature_map], gptr, int(bool(normalize)),
                               stream)
    torch.cuda.synchronize()
    del garr
    return st


@pytest.mark.parametrize("fm,decay,norm,T", [
    ("elu1", False, True, 1000),    # normalised, ragged (15 full chunks + 40 tokens)
    ("elu1", False, True, 4485),
    ("identity", True, False, 777),  # the retention form, ragged
    ("identity", True, False, 4096),
])
def test_lin_attn_prefill_bf16_output(fm, decay, norm, T):
    w = Workload("plain_bf16", B=2, H=4, T=T, dk=128, dv=128, C=64, dtype="bf16",
                 scale=0.5 if fm == "elu1" else 1.0 / math.sqrt(128), feature_map=fm,
                 decay=decay, normalize=norm)
    q, k, v = make_inputs(w, seed=3, device="cuda", gen_device="cpu")
    gamma = gammas_for(w.H, 3) if decay else None
    out = torch.empty((w.B, w.H, T, w.dv), dtype=torch.bfloat16, device="cuda")
    S = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    Z = torch.empty((w.B, w.H, w.dk), dtype=torch.float32, device="cuda") if norm else None
    assert _call("lin_attn_prefill", q, k, v, out, S, Z, 64, fm, gamma, norm) == B.LA_OK
    o_ref, S_ref, Z_ref = oracle_prefill(q, k, v, feature_map=fm, gamma=gamma, normalize=norm)
    assert_close_rounded_out(to_np(out), o_ref, TOL_BF16, "out (bf16)")
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final")
    if norm:
        assert_close(to_np(Z), Z_ref, TOL_BF16, "Z_final")
    assert B.lin_attn_device_error() == 0


def test_lin_attn_prefill_f32_small_reference_workload():
    """The float32 workload (B1 H2 T256 d32 C32, N(0,1) from seed 0, ELU+1, normalised)
    against the oracle on every element and against the stored oracle values."""
    from golden.make_golden import SAMPLE_T, load_golden
    w = WORKLOADS["pr1_ref"]
    q, k, v = make_inputs(w, seed=0, device="cpu")
    q, k, v = (t.cuda() for t in (q, k, v))
    out = torch.empty((w.B, w.H, w.T, w.dv), dtype=torch.float32, device="cuda")
    S = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    Z = torch.empty((w.B, w.H, w.dk), dtype=torch.float32, device="cuda")
    assert _call("lin_attn_prefill_f32", q, k, v, out, S, Z, w.C, w.feature_map, None,
                 True) == B.LA_OK
    o_ref, S_ref, Z_ref = oracle_prefill(q, k, v, feature_map=w.feature_map, gamma=None,
                                         normalize=True)
    assert_close(to_np(out), o_ref, TOL_F32, "out")
    assert_close(to_np(S), S_ref, TOL_F32, "S_final")
    assert_close(to_np(Z), Z_ref, TOL_F32, "Z_final")
    gold = load_golden()
    assert_close(to_np(out)[:, :, list(SAMPLE_T)], gold["out_sampled"], TOL_F32, "golden out")
    assert_close(to_np(S), gold["S_final"], TOL_F32, "golden S")
    assert_close(to_np(Z), gold["Z_final"], TOL_F32, "golden Z")


def test_lin_attn_prefill_f32_decay_ragged():
    w = Workload("plain_f32", B=1, H=3, T=301, dk=64, dv=32, C=32, dtype="f32", scale=0.5,
                 feature_map="identity", decay=True, normalize=False)
    q, k, v = make_inputs(w, seed=5, device="cpu")
    q, k, v = (t.cuda() for t in (q, k, v))
    gamma = gammas_for(w.H, 5)
    out = torch.empty((w.B, w.H, w.T, w.dv), dtype=torch.float32, device="cuda")
    S = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    assert _call("lin_attn_prefill_f32", q, k, v, out, S, None, w.C, "identity", gamma,
                 False) == B.LA_OK
    o_ref, S_ref, _ = oracle_prefill(q, k, v, feature_map="identity", gamma=gamma,
                                     normalize=False)
    assert_close(to_np(out), o_ref, TOL_F32, "out")
    assert_close(to_np(S), S_ref, TOL_F32, "S_final")


def test_plain_entry_points_reject_bad_arguments():
    """Statuses the contract names, before any launch: identity map with normalisation,
    a decay outside [0, 1], an unsupported head size on the bf16 path."""
    q = torch.zeros((1, 2, 64, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    S = torch.empty((1, 2, 64, 64), dtype=torch.float32, device="cuda")
    Z = torch.empty((1, 2, 64), dtype=torch.float32, device="cuda")
    assert _call("lin_attn_prefill", q, q, q, out, S, Z, 64, "identity", None, True) \
        == LA_ERR_INVALID_ARGUMENT
    assert _call("lin_attn_prefill", q, q, q, out, S, None, 64, "identity", [0.5, 1.5], False) \
        == LA_ERR_INVALID_ARGUMENT
    q3 = torch.zeros((1, 2, 64, 36), dtype=torch.bfloat16, device="cuda")
    o3 = torch.empty_like(q3)
    S3 = torch.empty((1, 2, 36, 36), dtype=torch.float32, device="cuda")
    st = _call("lin_attn_prefill", q3, q3, q3, o3, S3, None, 48, "identity", None, False)
    assert st == LA_ERR_UNSUPPORTED
