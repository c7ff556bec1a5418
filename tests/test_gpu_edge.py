"""GPU edge cases: empty and tiny inputs, padding leaks, causality, determinism, guard
bands, caller workspace, host-buffer entry point, decode continuation, error word."""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from chunked_causal_linear_b200 import binding as B
from chunked_causal_linear_b200.workloads import Workload, make_inputs
from gpu_common import TOL_BF16, TOL_F32, assert_close, gammas_for, oracle_prefill, to_np

pytestmark = pytest.mark.gpu


def _inputs(T, dk=128, dv=128, B_=1, H=2, dtype="bf16", fm="elu1", seed=0):
    w = Workload("edge", B=B_, H=H, T=T, dk=dk, dv=dv, C=64, dtype=dtype,
                 scale=0.5 if fm == "elu1" else 1.0 / math.sqrt(dk), feature_map=fm,
                 decay=fm == "identity", normalize=fm == "elu1")
    return w, *make_inputs(w, seed=seed, device="cuda", gen_device="cpu")


@pytest.mark.parametrize("path", ["tensor_core", "fma"])
def test_zero_length_sequence_zero_fills_states(path):
    q = torch.empty((2, 3, 0, 64), dtype=torch.bfloat16, device="cuda")
    S = torch.full((2, 3, 64, 64), 7.0, device="cuda")
    Z = torch.full((2, 3, 64), 7.0, device="cuda")
    out, S, Z = B.lin_attn_prefill(q, q, q, S_final=S, Z_final=Z, kernel_path=path)
    torch.cuda.synchronize()
    assert out.shape == (2, 3, 0, 64)
    assert not S.any() and not Z.any()


def test_empty_batch_is_a_no_op():
    q = torch.empty((0, 4, 100, 64), dtype=torch.bfloat16, device="cuda")
    out, S, Z = B.lin_attn_prefill(q, q, q)
    torch.cuda.synchronize()
    assert out.numel() == 0


@pytest.mark.parametrize("algorithm", ["chunked", "segmented"])
@pytest.mark.parametrize("fm", ["elu1", "identity"])
def test_padding_does_not_leak_from_the_next_head(fm, algorithm):
    # T = 100: the last chunk holds 36 tokens; a naive load of the full 64-row tile would
    # read the next head's first 28 tokens.  Make those huge.
    w, q, k, v = _inputs(100, fm=fm)
    for t in (q, k, v):
        t[:, 1, :28] = 100.0
    gamma = [0.97, 0.9] if w.decay else None
    out, S, Z = B.lin_attn_prefill(q, k, v, chunk=64, feature_map=fm, gamma=gamma,
                                   normalize=w.normalize, kernel_path="tensor_core",
                                   out_dtype="f32", algorithm=algorithm)
    torch.cuda.synchronize()
    o_ref, S_ref, Z_ref = oracle_prefill(q, k, v, feature_map=fm, gamma=gamma,
                                         normalize=w.normalize, heads=[(0, 0)])
    assert_close(to_np(out[0, 0])[None], o_ref, TOL_BF16, "out head 0")
    assert_close(to_np(S[0, 0])[None], S_ref, TOL_BF16, "S head 0")


@pytest.mark.parametrize("algorithm", ["chunked", "segmented"])
@pytest.mark.parametrize("t0", [0, 1, 63, 64, 100, 200])
def test_causality_bitwise(t0, algorithm):
    w, q, k, v = _inputs(256)
    kw = dict(kernel_path="tensor_core", algorithm=algorithm, segment_chunks=2)
    out1, _, _ = B.lin_attn_prefill(q, k, v, **kw)
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    for t in (q2, k2, v2):
        t[:, :, t0:] = 100.0
    out2, _, _ = B.lin_attn_prefill(q2, k2, v2, **kw)
    torch.cuda.synchronize()
    assert torch.equal(out1[:, :, :t0], out2[:, :, :t0])


@pytest.mark.parametrize("path,algorithm", [("tensor_core", "chunked"),
                                            ("tensor_core", "segmented"), ("fma", "chunked")])
def test_deterministic(path, algorithm):
    w, q, k, v = _inputs(1000)
    a = B.lin_attn_prefill(q, k, v, kernel_path=path, algorithm=algorithm)
    b = B.lin_attn_prefill(q, k, v, kernel_path=path, algorithm=algorithm)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_guard_bands_untouched():
    w, q, k, v = _inputs(300)
    pad = 4096
    n_out = q.shape[0] * q.shape[1] * 300 * 128
    out_buf = torch.full((n_out + 2 * pad,), 12345.0, dtype=torch.float32, device="cuda")
    s_buf = torch.full((2 * 128 * 128 + 2 * pad,), -777.0, device="cuda")
    z_buf = torch.full((2 * 128 + 2 * pad,), -777.0, device="cuda")
    out = out_buf[pad:pad + n_out].view(1, 2, 300, 128)
    S = s_buf[pad:pad + 2 * 128 * 128].view(1, 2, 128, 128)
    Z = z_buf[pad:pad + 2 * 128].view(1, 2, 128)
    B.lin_attn_prefill(q, k, v, out=out, S_final=S, Z_final=Z, kernel_path="tensor_core",
                       out_dtype="f32")
    torch.cuda.synchronize()
    for buf, n, val in ((out_buf, n_out, 12345.0), (s_buf, 2 * 128 * 128, -777.0),
                        (z_buf, 2 * 128, -777.0)):
        assert torch.all(buf[:pad] == val) and torch.all(buf[pad + n:] == val)
    o_ref, S_ref, _ = oracle_prefill(q, k, v, feature_map="elu1", gamma=None, normalize=True)
    assert_close(to_np(out), o_ref, TOL_BF16, "out")


def test_caller_workspace_equals_library_workspace():
    w, q, k, v = _inputs(777, dk=64, dv=64, H=4)
    ws = torch.empty(B.lin_attn_prefill_workspace_bytes(1, 4, 777, 64, 64, 64, True),
                     dtype=torch.uint8, device="cuda")
    a = B.lin_attn_prefill(q, k, v, workspace=ws)
    b = B.lin_attn_prefill(q, k, v)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_workspace_too_small_is_rejected():
    w, q, k, v = _inputs(128, dk=64, dv=64)
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(B.LinAttnError) as e:
        B.lin_attn_prefill(q, k, v, workspace=ws)
    assert e.value.status == 1


@pytest.mark.parametrize("dtype,out_dtype", [("bf16", "as_input"), ("bf16", "f32"),
                                             ("f32", "as_input")])
def test_host_buffer_entry_point_matches_device_path(dtype, out_dtype):
    w, q, k, v = _inputs(500, dk=64, dv=64, H=3, dtype=dtype)
    out_d, S_d, Z_d = B.lin_attn_prefill(q, k, v, out_dtype=out_dtype)
    torch.cuda.synchronize()
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    out_h = torch.empty(out_d.shape, dtype=out_d.dtype).pin_memory()
    S_h = torch.empty((1, 3, 64, 64), dtype=torch.float32).pin_memory()
    Z_h = torch.empty((1, 3, 64), dtype=torch.float32).pin_memory()
    B.lin_attn_prefill_host(qh, kh, vh, out_h, S_h, Z_h, out_dtype=out_dtype)
    assert torch.equal(out_h, out_d.cpu())
    assert torch.equal(S_h, S_d.cpu())
    assert torch.equal(Z_h, Z_d.cpu())


@pytest.mark.parametrize("fm,norm,decay", [("elu1", True, False), ("identity", False, True),
                                           ("elu1", True, True)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_continues_the_prefill(fm, norm, decay, dtype):
    T = 200
    w = Workload("dec", B=2, H=3, T=T + 1, dk=64, dv=64, C=64, dtype=dtype, scale=0.5,
                 feature_map=fm, decay=decay, normalize=norm)
    q, k, v = make_inputs(w, seed=3, device="cuda", gen_device="cpu")
    gamma = gammas_for(3, 5) if decay else None
    _, S, Z = B.lin_attn_prefill(q[:, :, :T].contiguous(), k[:, :, :T].contiguous(),
                                 v[:, :, :T].contiguous(), feature_map=fm, gamma=gamma,
                                 normalize=norm)
    if Z is None:
        Z = torch.zeros((2, 3, 64), device="cuda")
    o_step = B.lin_attn_decode_step(q[:, :, T].contiguous(), k[:, :, T].contiguous(),
                                    v[:, :, T].contiguous(), S, Z, feature_map=fm, gamma=gamma,
                                    normalize=norm)
    torch.cuda.synchronize()
    o_ref, S_ref, Z_ref = oracle_prefill(q, k, v, feature_map=fm, gamma=gamma, normalize=norm)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert_close(to_np(o_step), o_ref[:, :, T], tol, "decode out")
    assert_close(to_np(S), S_ref, tol, "decode S")
    if norm:
        assert_close(to_np(Z), Z_ref, tol, "decode Z")


def test_decode_matches_oracle_from_a_given_state():
    from oracle.oracle import default_oracle
    rng = np.random.default_rng(4)
    S0 = rng.standard_normal((1, 4, 128, 128)).astype(np.float32)
    Z0 = rng.uniform(1, 5, size=(1, 4, 128)).astype(np.float32)
    q, k, v = (torch.tensor(rng.standard_normal((1, 4, 128)) * 0.5, dtype=torch.float32)
               for _ in range(3))
    S = torch.tensor(S0, device="cuda")
    Z = torch.tensor(Z0, device="cuda")
    out = B.lin_attn_decode_step(q.cuda(), k.cuda(), v.cuda(), S, Z)
    torch.cuda.synchronize()
    o_ref, S_ref, Z_ref = default_oracle().forward(q.numpy()[:, :, None], k.numpy()[:, :, None],
                                                   v.numpy()[:, :, None], S_init=S0, Z_init=Z0)
    assert_close(to_np(out), o_ref[:, :, 0], TOL_F32, "out")
    assert_close(to_np(S), S_ref, TOL_F32, "S")
    assert_close(to_np(Z), Z_ref, TOL_F32, "Z")


def test_argument_errors_on_device_tensors():
    w, q, k, v = _inputs(64, dk=64, dv=64)
    with pytest.raises(B.LinAttnError):
        B.lin_attn_prefill(q, k, v, out=q)  # out aliases q
    with pytest.raises(B.LinAttnError):
        B.lin_attn_prefill(q, k, v, feature_map="identity", normalize=True)
    with pytest.raises(B.LinAttnError):
        B.lin_attn_prefill(q, k, v, gamma=[1.5, 0.5])


def test_no_device_error_reported():
    assert B.lin_attn_device_error() == 0


@pytest.mark.parametrize("fm,norm,decay", [("identity", False, True), ("elu1", True, False)])
def test_host_entry_point_pipelines_large_problems(fm, norm, decay):
    # About 100 MB of inputs: the host entry point splits the heads into groups whose
    # copies overlap the kernels.  With the segment length fixed, each (b, h) is computed
    # exactly as by the device entry point, so the results are bitwise equal.
    w = Workload("host_pipe", B=2, H=4, T=16384, dk=128, dv=128, C=64, dtype="bf16",
                 scale=1.0 / math.sqrt(128) if fm == "identity" else 0.5, feature_map=fm,
                 decay=decay, normalize=norm)
    q, k, v = make_inputs(w, seed=9, device="cuda", gen_device="cpu")
    gamma = gammas_for(4, 9) if decay else None
    kw = dict(feature_map=fm, gamma=gamma, normalize=norm, out_dtype="f32", segment_chunks=16)
    out_d, S_d, Z_d = B.lin_attn_prefill(q, k, v, **kw)
    torch.cuda.synchronize()
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    out_h = torch.empty(out_d.shape, dtype=out_d.dtype).pin_memory()
    S_h = torch.empty(S_d.shape, dtype=torch.float32).pin_memory()
    Z_h = torch.empty((2, 4, 128), dtype=torch.float32).pin_memory() if norm else None
    B.lin_attn_prefill_host(qh, kh, vh, out_h, S_h, Z_h, **kw)
    assert torch.equal(out_h, out_d.cpu())
    assert torch.equal(S_h, S_d.cpu())
    if norm:
        assert torch.equal(Z_h, Z_d.cpu())
    assert B.lin_attn_device_error() == 0
