"""GPU parity of gated linear attention (lin_attn_gla_prefill) against the oracle's token
loop, element by element on the same inputs (bf16 inputs: the oracle gets the same
bf16-rounded values; the gates are float32 on both sides).  Tolerances: max |err| <=
2e-2 * rms(oracle) for bf16 inputs (both paths), 1e-4 * rms for float32 inputs (CUDA
cores)."""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from chunked_causal_linear_b200 import binding as B
from chunked_causal_linear_b200.workloads import GLA_WORKLOADS, Workload, make_gates, make_inputs
from gpu_common import TOL_BF16, TOL_F32, assert_close, to_np
from oracle.oracle import default_oracle

pytestmark = pytest.mark.gpu


def _problem(T, *, dk=128, dv=128, dtype="bf16", H=3, seed=0, mean=4.0, std=1.0):
    """B2 H3 inputs N(0,1)/sqrt(dk) and gates sigmoid(N(mean, std)), CPU-drawn."""
    w = Workload("gla", B=2, H=H, T=T, dk=dk, dv=dv, C=64, dtype=dtype,
                 scale=1.0 / math.sqrt(dk), feature_map="identity", decay=False, normalize=False)
    q, k, v = make_inputs(w, seed=seed, device="cuda", gen_device="cpu")
    alpha = make_gates(w, seed=seed, device="cuda", gen_device="cpu", mean=mean, std=std)
    return q, k, v, alpha


def _oracle(q, k, v, alpha, S0=None):
    return default_oracle().gla_forward(to_np(q), to_np(k), to_np(v), to_np(alpha),
                                        S_init=None if S0 is None else to_np(S0).astype(np.float64))


@pytest.mark.parametrize("C", [16, 32, 64])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 1000, 3001])
def test_gla_matches_oracle(C, T):
    q, k, v, alpha = _problem(T)
    out, S = B.lin_attn_gla_prefill(q, k, v, alpha, chunk=C, out_dtype="f32")
    torch.cuda.synchronize()
    o_ref, S_ref = _oracle(q, k, v, alpha)
    assert_close(to_np(out), o_ref, TOL_BF16, "out")
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final")


@pytest.mark.parametrize("mean,std", [(0.0, 2.0), (8.0, 1.0), (-3.0, 1.0)])
def test_gla_gate_ranges(mean, std):
    # wide gates, gates near 1, and gates near 0 (state forgotten within a few tokens)
    q, k, v, alpha = _problem(777, mean=mean, std=std)
    out, S = B.lin_attn_gla_prefill(q, k, v, alpha, out_dtype="f32")
    torch.cuda.synchronize()
    o_ref, S_ref = _oracle(q, k, v, alpha)
    assert_close(to_np(out), o_ref, TOL_BF16, "out")
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final")


def test_gla_exact_zero_and_unit_gates_and_initial_state():
    q, k, v, alpha = _problem(500)
    alpha[:, :, 100] = 0.0          # every feature forgets at token 100
    alpha[:, :, 200:260, :64] = 1.0  # no decay on half the features for 60 tokens
    S0 = (torch.randn((2, 3, 128, 128), generator=torch.Generator().manual_seed(9)) * 0.3).cuda()
    out, S = B.lin_attn_gla_prefill(q, k, v, alpha, S_init=S0, out_dtype="f32")
    torch.cuda.synchronize()
    o_ref, S_ref = _oracle(q, k, v, alpha, S0)
    assert_close(to_np(out), o_ref, TOL_BF16, "out")
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final")


@pytest.mark.parametrize("dk,dv", [(64, 64), (32, 48), (128, 64), (8, 8)])
def test_gla_fp32_and_other_dims(dk, dv):
    q, k, v, alpha = _problem(300, dk=dk, dv=dv, dtype="f32")
    out, S = B.lin_attn_gla_prefill(q, k, v, alpha, chunk=32)
    torch.cuda.synchronize()
    o_ref, S_ref = _oracle(q, k, v, alpha)
    assert_close(to_np(out), o_ref, TOL_F32, "out")
    assert_close(to_np(S), S_ref, TOL_F32, "S_final")


def test_gla_bf16_output_and_workspace():
    q, k, v, alpha = _problem(1000)
    ws = torch.empty(B.lin_attn_gla_workspace_bytes(2, 3, 1000, 128, 128, 64), dtype=torch.uint8,
                     device="cuda")
    out, S = B.lin_attn_gla_prefill(q, k, v, alpha, workspace=ws)
    out2, S2 = B.lin_attn_gla_prefill(q, k, v, alpha)
    torch.cuda.synchronize()
    assert out.dtype == torch.bfloat16
    assert torch.equal(out, out2) and torch.equal(S, S2)
    o_ref, _ = _oracle(q, k, v, alpha)
    got, ref = to_np(out).astype(np.float64), o_ref
    assert float(np.max(np.abs(got - ref) - (2e-2 * np.sqrt(np.mean(ref ** 2)) + 2 ** -8 * np.abs(ref)))) <= 0


def test_gla_zero_tokens_return_the_initial_state():
    q, k, v, alpha = _problem(0)
    S0 = torch.randn((2, 3, 128, 128)).cuda()
    _, S = B.lin_attn_gla_prefill(q, k, v, alpha, S_init=S0)
    torch.cuda.synchronize()
    assert torch.equal(S, S0)


def test_gla_full_size_sampled_heads_cuda_cores():
    """The 128k-token gated workload (B=1, H=32, T=131072, d=128) on the CUDA-core path;
    the oracle recomputes heads 0 and 31 in full."""
    w = GLA_WORKLOADS["gla_128k"]
    q, k, v = make_inputs(w, seed=0, device="cuda")
    alpha = make_gates(w, seed=0, device="cuda")
    out, S = B.lin_attn_gla_prefill(q, k, v, alpha, out_dtype="f32", kernel_path="fma")
    torch.cuda.synchronize()
    for h in (0, 31):
        sl = lambda t: t[:, h:h + 1]
        o_ref, S_ref = _oracle(sl(q), sl(k), sl(v), sl(alpha))
        assert_close(to_np(sl(out)), o_ref, TOL_BF16, f"head {h} out")
        assert_close(to_np(sl(S)), S_ref, TOL_BF16, f"head {h} S_final")


# ---------------------------------------------------------------------------------------
# The tensor-core path (the default for bf16, C = 64, dk in {64, 128}, dv = 128): segmented,
# factored operands split into bf16 hi + lo, a renormalised window per feature, and the
# exact CUDA-core fix-up for chunks whose gates fall too fast to factor.  Held to the same
# 2e-2 rms bound as every bf16 path, against the oracle; the CUDA-core path beside it.

def _both_paths(q, k, v, alpha, S0=None, **kw):
    out_t, S_t = B.lin_attn_gla_prefill(q, k, v, alpha, S_init=S0, out_dtype="f32",
                                        kernel_path="tensor_core", **kw)
    out_f, S_f = B.lin_attn_gla_prefill(q, k, v, alpha, S_init=S0, out_dtype="f32",
                                        kernel_path="fma")
    torch.cuda.synchronize()
    assert B.lin_attn_device_error() == 0
    return (out_t, S_t), (out_f, S_f)


@pytest.mark.parametrize("dk", [64, 128])
@pytest.mark.parametrize("mean,std", [(4.0, 1.0), (8.0, 1.0), (0.0, 2.0), (-3.0, 1.0), (2.0, 3.0)])
@pytest.mark.parametrize("seg", [0, 1, 4, 7])
def test_gla_tensor_core_path_gate_ranges(dk, mean, std, seg):
    """Gates near 1 (long windows), moderate, wide, and small (every chunk takes the exact
    fix-up); segments of 1, 4, 7 chunks and the automatic length; ragged T."""
    q, k, v, alpha = _problem(1000, dk=dk, mean=mean, std=std, seed=seg)
    (out, S), (out_f, S_f) = _both_paths(q, k, v, alpha, segment_chunks=seg)
    o_ref, S_ref = _oracle(q, k, v, alpha)
    assert_close(to_np(out), o_ref, TOL_BF16, "out (tensor cores)")
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final (tensor cores)")
    assert_close(to_np(out_f), o_ref, TOL_BF16, "out (CUDA cores)")
    assert_close(to_np(S_f), S_ref, TOL_BF16, "S_final (CUDA cores)")


@pytest.mark.parametrize("T", [1, 63, 64, 65, 129, 3001])
def test_gla_tensor_core_path_lengths_and_initial_state(T):
    q, k, v, alpha = _problem(T, mean=3.0)
    S0 = (torch.randn((2, 3, 128, 128), generator=torch.Generator().manual_seed(T)) * 0.3).cuda()
    (out, S), _ = _both_paths(q, k, v, alpha, S0, segment_chunks=3)
    o_ref, S_ref = _oracle(q, k, v, alpha, S0)
    assert_close(to_np(out), o_ref, TOL_BF16, "out")
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final")


def test_gla_tensor_core_path_mixed_windows_and_zero_gates():
    """One head's features decay at very different rates (a few near 0, most near 1), a
    zero gate on every feature mid-sequence, and unit gates on half the features: windows,
    rebases and steep chunks all occur within the same segments."""
    q, k, v, alpha = _problem(2000, mean=5.0, seed=5)
    alpha[:, :, :, :8] = torch.sigmoid(torch.randn_like(alpha[:, :, :, :8]) - 4.0)
    alpha[:, :, 700] = 0.0
    alpha[:, :, 1000:1500, 64:] = 1.0
    (out, S), _ = _both_paths(q, k, v, alpha, segment_chunks=8)
    o_ref, S_ref = _oracle(q, k, v, alpha)
    assert_close(to_np(out), o_ref, TOL_BF16, "out")
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final")


def test_gla_tensor_core_path_bf16_output():
    q, k, v, alpha = _problem(1000, mean=-1.0)
    out, S = B.lin_attn_gla_prefill(q, k, v, alpha, kernel_path="tensor_core", segment_chunks=4)
    torch.cuda.synchronize()
    assert out.dtype == torch.bfloat16
    o_ref, S_ref = _oracle(q, k, v, alpha)
    got, ref = to_np(out).astype(np.float64), o_ref
    assert float(np.max(np.abs(got - ref) - (2e-2 * np.sqrt(np.mean(ref ** 2)) + 2 ** -8 * np.abs(ref)))) <= 0
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final")


def test_gla_tensor_core_path_refuses_other_shapes():
    q, k, v, alpha = _problem(100, dk=128, dv=64)
    with pytest.raises(B.LinAttnError):
        B.lin_attn_gla_prefill(q, k, v, alpha, kernel_path="tensor_core")


def test_gla_tensor_core_path_full_size_sampled_heads():
    """The 128k-token gated workload in the benchmark's configuration (the default path)."""
    w = GLA_WORKLOADS["gla_128k"]
    q, k, v = make_inputs(w, seed=0, device="cuda")
    alpha = make_gates(w, seed=0, device="cuda")
    out, S = B.lin_attn_gla_prefill(q, k, v, alpha, out_dtype="f32")
    torch.cuda.synchronize()
    assert B.lin_attn_device_error() == 0
    for h in (0, 17, 31):
        sl = lambda t: t[:, h:h + 1]
        o_ref, S_ref = _oracle(sl(q), sl(k), sl(v), sl(alpha))
        assert_close(to_np(sl(out)), o_ref, TOL_BF16, f"head {h} out")
        assert_close(to_np(sl(S)), S_ref, TOL_BF16, f"head {h} S_final")
