"""GPU parity at the workloads' full sizes, in the launch configuration the benchmark times
(tensor-core kernels, log-depth scan, caller-provided workspace, float32 output).

The oracle recomputes a sample of (b, h) pairs in full (every output row of those pairs
and their final states); the smallest workload is compared on every pair.  Tolerance:
max |err| <= 2e-2 * rms(oracle) per tensor.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from chunked_causal_linear_b200 import binding as B
from chunked_causal_linear_b200.workloads import WORKLOADS, make_inputs
from gpu_common import TOL_BF16, assert_close, oracle_prefill, to_np

pytestmark = pytest.mark.gpu

SAMPLES = {
    "norm_b4h16": None,
    "ragged_b2h32": [(0, 0), (0, 31), (1, 17)],
    "ragged_b2h32_t15990": [(0, 5), (1, 0), (1, 31)],
    "retention_128k": [(0, 0), (0, 31)],
    "scan_depth_1m": [(0, 3)],
}


def run_bench_config(w, q, k, v, scan="logdepth", algorithm="auto"):
    ws = torch.empty(B.lin_attn_prefill_workspace_bytes(w.B, w.H, w.T, w.dk, w.dv, w.C,
                                                        w.normalize),
                     dtype=torch.uint8, device="cuda")
    out, S, Z = B.lin_attn_prefill(q, k, v, chunk=w.C, feature_map=w.feature_map,
                                   gamma=w.gammas(), normalize=w.normalize, scan=scan,
                                   kernel_path="tensor_core", workspace=ws, out_dtype="f32",
                                   algorithm=algorithm)
    torch.cuda.synchronize()
    return out, S, Z


@pytest.mark.parametrize("algorithm", ["auto", "chunked"])
@pytest.mark.parametrize("name", sorted(SAMPLES))
def test_workload_full_size(name, algorithm):
    """`auto` is the benchmark's configuration (segmented for every workload here)."""
    w = WORKLOADS[name]
    q, k, v = make_inputs(w, seed=0, device="cuda")
    out, S, Z = run_bench_config(w, q, k, v, algorithm=algorithm)
    heads = SAMPLES[name]
    o_ref, S_ref, Z_ref = oracle_prefill(q, k, v, feature_map=w.feature_map, gamma=w.gammas(),
                                         normalize=w.normalize, heads=heads)
    if heads is None:
        got_o, got_S, got_Z = to_np(out), to_np(S), (to_np(Z) if w.normalize else None)
    else:
        got_o = np.stack([to_np(out[b, h]) for b, h in heads])
        got_S = np.stack([to_np(S[b, h]) for b, h in heads])
        got_Z = np.stack([to_np(Z[b, h]) for b, h in heads]) if w.normalize else None
    assert_close(got_o, o_ref, TOL_BF16, f"{name} out")
    assert_close(got_S, S_ref, TOL_BF16, f"{name} S_final")
    if w.normalize:
        assert_close(got_Z, Z_ref, TOL_BF16, f"{name} Z_final")


@pytest.mark.parametrize("scan", ["sequential", "logdepth"])
@pytest.mark.parametrize("name", ["retention_128k", "scan_depth_1m"])
def test_scan_modes_full_size_against_oracle(name, scan):
    """Both K2 modes at the chunk counts the scan comparison is timed on (chunked
    arrangement: one scan element per chunk, N_C = 2048 and 16384), each against the
    oracle on sampled heads."""
    w = WORKLOADS[name]
    q, k, v = make_inputs(w, seed=0, device="cuda")
    out, S, Z = run_bench_config(w, q, k, v, scan=scan, algorithm="chunked")
    heads = SAMPLES[name]
    o_ref, S_ref, Z_ref = oracle_prefill(q, k, v, feature_map=w.feature_map, gamma=w.gammas(),
                                         normalize=w.normalize, heads=heads)
    assert_close(np.stack([to_np(out[b, h]) for b, h in heads]), o_ref, TOL_BF16,
                 f"{name} {scan} out")
    assert_close(np.stack([to_np(S[b, h]) for b, h in heads]), S_ref, TOL_BF16,
                 f"{name} {scan} S_final")
    if w.normalize:
        assert_close(np.stack([to_np(Z[b, h]) for b, h in heads]), Z_ref, TOL_BF16,
                     f"{name} {scan} Z_final")


def test_scan_depth_final_states_all_heads():
    w = WORKLOADS["scan_depth_1m"]
    q, k, v = make_inputs(w, seed=0, device="cuda")
    _, S, Z = run_bench_config(w, q, k, v)
    _, S_ref, Z_ref = oracle_prefill(q, k, v, feature_map=w.feature_map, gamma=None,
                                     normalize=True, want_out=False)
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final")
    assert_close(to_np(Z), Z_ref, TOL_BF16, "Z_final")
