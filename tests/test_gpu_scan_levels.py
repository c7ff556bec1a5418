"""The log-depth scan's two levels, against the oracle.

Up to 2048 scan elements the scan is one blocked pass; beyond, segments of Ls >= 16
elements are folded, their folds scanned, and each segment re-scanned
(lin_attn_scan_plan).  These cases take the two-level path with everything that enters the
scan at once: a per-head decay, an initial state (the scan's first element), a ragged last
chunk and the final states, in the chunked arrangement (elements = chunks) and in the
segmented one with one chunk per segment (elements = segments).  Tolerance 2e-2 rms
(bf16 inputs, float32 outputs), both scan modes; the number of kernels each run launches
matches the plan.  A last group covers the boundary between the block level's two forms:
k2_warp_scan up to 32 elements, k2_block_scan beyond.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from chunked_causal_linear_b200 import binding as B
from chunked_causal_linear_b200.workloads import Workload, make_inputs
from gpu_common import TOL_BF16, assert_close, gammas_for, oracle_prefill, to_np

pytestmark = pytest.mark.gpu


def _case(T, fm, decay, norm, seed):
    w = Workload("scan2", B=1, H=2, T=T, dk=64, dv=64, C=64, dtype="bf16",
                 scale=0.5 if fm == "elu1" else 1.0 / math.sqrt(64), feature_map=fm, decay=decay,
                 normalize=norm)
    q, k, v = make_inputs(w, seed=seed, device="cuda", gen_device="cpu")
    g = torch.Generator().manual_seed(seed)
    S0 = (torch.randn((1, 2, 64, 64), generator=g) * 0.3).cuda()
    Z0 = (torch.rand((1, 2, 64), generator=g) + 1.0).cuda() if norm else None
    gamma = [float(np.float32(0.9995)), float(np.float32(0.97))] if decay else None
    return w, q, k, v, S0, Z0, gamma


@pytest.mark.parametrize("scan", ["logdepth", "sequential"])
@pytest.mark.parametrize("algorithm,seg", [("chunked", 0), ("segmented", 1)])
@pytest.mark.parametrize("fm,decay,norm", [("identity", True, False), ("elu1", False, True)])
def test_two_level_scan_against_oracle(scan, algorithm, seg, fm, decay, norm):
    T = 64 * 2500 + 17  # 2501 chunks: past the one-level limit, ragged last chunk
    w, q, k, v, S0, Z0, gamma = _case(T, fm, decay, norm, seed=7)
    kw = dict(chunk=64, feature_map=fm, gamma=gamma, normalize=norm, scan=scan,
              kernel_path="tensor_core", algorithm=algorithm, segment_chunks=seg,
              out_dtype="f32")
    out, S, Z = B.lin_attn_prefill(q, k, v, S_init=S0, Z_init=Z0, **kw)
    torch.cuda.synchronize()
    assert B.lin_attn_device_error() == 0
    o_ref, S_ref, Z_ref = oracle_prefill(q, k, v, feature_map=fm, gamma=gamma, normalize=norm,
                                         S_init=S0, Z_init=Z0)
    assert_close(to_np(out), o_ref, TOL_BF16, "out")
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final")
    if norm:
        assert_close(to_np(Z), Z_ref, TOL_BF16, "Z_final")
    # K1, the scan's kernels (1 for one level or the sequential carry, 3 for two levels), K3.
    n_elem = -(-T // 64) // max(seg, 1) if algorithm == "segmented" else -(-T // 64)
    plan = B.lin_attn_scan_plan(n_elem, scan)
    k2 = 1 if (scan == "sequential" or plan["segments"] == 1) else 3
    out2 = torch.empty_like(out)
    S2 = torch.empty_like(S)
    Z2 = torch.empty_like(Z) if norm else None
    times = B.lin_attn_prefill_timed(q, k, v, out2, S2, Z2, **kw)
    assert len(times) == 2 + k2


def test_scan_plan_shapes_the_launches():
    """One level up to 2048 elements, two beyond, as lin_attn_scan_plan reports."""
    for nc, levels in ((2048, 1), (2049, 2)):
        p = B.lin_attn_scan_plan(nc)
        assert (p["segments"] == 1) == (levels == 1)
        w = Workload("plan", B=1, H=1, T=64 * nc, dk=64, dv=64, C=64, dtype="bf16", scale=0.5,
                     feature_map="elu1", decay=False, normalize=True)
        q, k, v = make_inputs(w, seed=1, device="cuda", gen_device="cpu")
        out = torch.empty((1, 1, w.T, 64), dtype=torch.float32, device="cuda")
        times = B.lin_attn_prefill_timed(q, k, v, out, chunk=64, feature_map="elu1",
                                         normalize=True, kernel_path="tensor_core",
                                         algorithm="chunked", out_dtype="f32")
        assert len(times) == 2 + (1 if levels == 1 else 3)
        assert np.all(np.isfinite(to_np(out)))


@pytest.mark.parametrize("scan_elems", [1, 2, 31, 32, 33, 64])
@pytest.mark.parametrize("fm,decay,norm", [("identity", True, False), ("elu1", True, True)])
def test_warp_and_block_scan_boundary(scan_elems, fm, decay, norm):
    """The block level runs as k2_warp_scan up to 32 elements and as k2_block_scan beyond:
    both against the oracle at the boundary, chunked (elements = chunks) with a ragged last
    chunk, a per-head decay and an initial state."""
    T = 64 * (scan_elems - 1) + 23
    w, q, k, v, S0, Z0, gamma = _case(T, fm, decay, norm, seed=11 + scan_elems)
    kw = dict(chunk=64, feature_map=fm, gamma=gamma, normalize=norm, scan="logdepth",
              kernel_path="tensor_core", algorithm="chunked", out_dtype="f32")
    out, S, Z = B.lin_attn_prefill(q, k, v, S_init=S0, Z_init=Z0, **kw)
    torch.cuda.synchronize()
    assert B.lin_attn_device_error() == 0
    o_ref, S_ref, Z_ref = oracle_prefill(q, k, v, feature_map=fm, gamma=gamma, normalize=norm,
                                         S_init=S0, Z_init=Z0)
    assert_close(to_np(out), o_ref, TOL_BF16, "out")
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final")
    if norm:
        assert_close(to_np(Z), Z_ref, TOL_BF16, "Z_final")
