"""GPU parity on small shapes: every mode, both kernel paths, ragged tails.

Each case runs the CUDA library through the C ABI and compares with the fp64 oracle on
the same inputs: max |err| <= 2e-2 * rms(oracle) for bf16 inputs (tensor-core and FMA
kernels, float32 output), <= 1e-4 * rms(oracle) for float32 inputs (FMA kernels).  A
bf16 output adds its own rounding to that bound (see ``assert_close_rounded_out``).
Sizes span several chunks and a ragged last chunk.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from chunked_causal_linear_b200.workloads import WORKLOADS, Workload, make_inputs
from chunked_causal_linear_b200 import binding as B
from gpu_common import (TOL_BF16, TOL_F32, assert_close, assert_close_rounded_out,
                        gammas_for, gpu_prefill, oracle_prefill, to_np)

pytestmark = pytest.mark.gpu

MODES = {
    "norm": dict(feature_map="elu1", decay=False, normalize=True),
    "unnorm": dict(feature_map="elu1", decay=False, normalize=False),
    "retention": dict(feature_map="identity", decay=True, normalize=False),
    "decay_norm": dict(feature_map="elu1", decay=True, normalize=True),
}


def _case(T, dk, dv, C, mode, dtype="bf16", B=2, H=3, seed=0):
    m = MODES[mode]
    scale = 1.0 / math.sqrt(dk) if m["feature_map"] == "identity" else 0.5
    w = Workload("case", B=B, H=H, T=T, dk=dk, dv=dv, C=C, dtype=dtype, scale=scale,
                 feature_map=m["feature_map"], decay=m["decay"], normalize=m["normalize"])
    q, k, v = make_inputs(w, seed=seed, device="cuda", gen_device="cpu")
    gamma = gammas_for(H, seed) if m["decay"] else None
    return w, q, k, v, gamma


def _check(w, q, k, v, gamma, tol, **kw):
    out, S, Z = gpu_prefill(q, k, v, C=w.C, feature_map=w.feature_map, gamma=gamma,
                            normalize=w.normalize, **kw)
    o_ref, S_ref, Z_ref = oracle_prefill(q, k, v, feature_map=w.feature_map, gamma=gamma,
                                         normalize=w.normalize)
    assert_close(to_np(out), o_ref, tol, "out")
    assert_close(to_np(S), S_ref, tol, "S_final")
    if w.normalize:
        assert_close(to_np(Z), Z_ref, tol, "Z_final")


@pytest.mark.parametrize("mode", sorted(MODES))
@pytest.mark.parametrize("T", [1, 33, 64, 100, 257, 1000])
@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_tensor_core_path(dk, dv, T, mode):
    w, q, k, v, gamma = _case(T, dk, dv, 64, mode)
    _check(w, q, k, v, gamma, TOL_BF16, kernel_path="tensor_core", algorithm="chunked")


@pytest.mark.parametrize("mode", sorted(MODES))
@pytest.mark.parametrize("T,seg", [(1, 0), (64, 1), (100, 1), (257, 2), (1000, 3), (1000, 7),
                                   (1000, 16), (4485, 0), (4485, 5)])
@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 128), (64, 64), (128, 64)])
def test_segmented_path(dk, dv, T, seg, mode):
    """Segments of `seg` chunks (0 = automatic): the prefix carried through several chunks
    inside a segment, segment prefixes from the scan, a ragged last chunk.  dv = 64 runs the
    combine at 128 value lanes with the upper half of V zero."""
    w, q, k, v, gamma = _case(T, dk, dv, 64, mode)
    if mode == "decay_norm":
        # ELU+1 with decay is not offered by the segmented kernels (shared memory); an
        # explicit request is refused and `auto` runs the chunked algorithm.
        with pytest.raises(B.LinAttnError) as e:
            gpu_prefill(q, k, v, C=64, feature_map=w.feature_map, gamma=gamma,
                        normalize=w.normalize, kernel_path="tensor_core", algorithm="segmented")
        assert e.value.status == 2
        _check(w, q, k, v, gamma, TOL_BF16, kernel_path="tensor_core", algorithm="auto")
        return
    _check(w, q, k, v, gamma, TOL_BF16, kernel_path="tensor_core", algorithm="segmented",
           segment_chunks=seg)


@pytest.mark.parametrize("mode", sorted(MODES))
@pytest.mark.parametrize("T", [33, 257])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (32, 64)])
def test_fma_path_bf16(dk, dv, T, mode):
    w, q, k, v, gamma = _case(T, dk, dv, 64 if dk >= 64 else 32, mode)
    _check(w, q, k, v, gamma, TOL_BF16, kernel_path="fma")


@pytest.mark.parametrize("mode", ["norm", "retention", "decay_norm"])
@pytest.mark.parametrize("C", [16, 32, 64])
@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 32), (64, 32), (128, 128)])
@pytest.mark.parametrize("T", [1, 50, 300])
def test_fma_path_f32(T, dk, dv, C, mode):
    w, q, k, v, gamma = _case(T, dk, dv, C, mode, dtype="f32")
    _check(w, q, k, v, gamma, TOL_F32)


@pytest.mark.parametrize("mode", sorted(MODES))
@pytest.mark.parametrize("path", ["tensor_core", "fma"])
@pytest.mark.parametrize("T", [100, 1000])
@pytest.mark.parametrize("algorithm", ["chunked", "segmented"])
@pytest.mark.parametrize("dv", [64, 128])
def test_bf16_output(T, path, mode, algorithm, dv):
    if path == "fma" and algorithm == "segmented":
        pytest.skip("the segmented algorithm runs on the tensor-core kernels only")
    if mode == "decay_norm" and algorithm == "segmented":
        pytest.skip("ELU+1 with decay runs on the chunked algorithm only")
    w, q, k, v, gamma = _case(T, 128, dv, 64, mode)
    out, S, Z = gpu_prefill(q, k, v, C=64, feature_map=w.feature_map, gamma=gamma,
                            normalize=w.normalize, kernel_path=path, out_dtype="as_input",
                            algorithm=algorithm, segment_chunks=3)
    assert out.dtype == torch.bfloat16
    o_ref, S_ref, _ = oracle_prefill(q, k, v, feature_map=w.feature_map, gamma=gamma,
                                     normalize=w.normalize)
    assert_close_rounded_out(to_np(out), o_ref, TOL_BF16, "bf16 out")
    assert_close(to_np(S), S_ref, TOL_BF16, "S_final")


@pytest.mark.parametrize("mode", ["norm", "retention"])
@pytest.mark.parametrize("T", [100, 1000, 64 * 70 + 5])
@pytest.mark.parametrize("dv,algorithm", [(64, "chunked"), (128, "segmented"), (64, "segmented")])
def test_scan_modes_agree_with_oracle(T, mode, dv, algorithm):
    w, q, k, v, gamma = _case(T, 64, dv, 64, mode)
    for scan in ("logdepth", "sequential"):
        _check(w, q, k, v, gamma, TOL_BF16, scan=scan, algorithm=algorithm,
               segment_chunks=2 if algorithm == "segmented" else 0)


def test_pr1_ref_fp32_against_oracle_and_golden():
    from golden.make_golden import SAMPLE_T, load_golden
    w = WORKLOADS["pr1_ref"]
    q, k, v = make_inputs(w, seed=0, device="cuda", gen_device="cpu")
    out, S, Z = gpu_prefill(q, k, v, C=w.C, feature_map=w.feature_map, gamma=None,
                            normalize=True)
    o_ref, S_ref, Z_ref = oracle_prefill(q, k, v, feature_map=w.feature_map, gamma=None,
                                         normalize=True)
    assert_close(to_np(out), o_ref, TOL_F32, "out")
    assert_close(to_np(S), S_ref, TOL_F32, "S_final")
    assert_close(to_np(Z), Z_ref, TOL_F32, "Z_final")
    gold = load_golden()
    assert_close(to_np(out)[:, :, list(SAMPLE_T)], gold["out_sampled"], TOL_F32, "golden out")
    assert_close(to_np(S), gold["S_final"], TOL_F32, "golden S")
    assert_close(to_np(Z), gold["Z_final"], TOL_F32, "golden Z")


@pytest.mark.parametrize("seed", [1])
def test_pr1_ref_fp32_second_seed(seed):
    w = WORKLOADS["pr1_ref"]
    q, k, v = make_inputs(w, seed=seed, device="cuda", gen_device="cpu")
    _check(w, q, k, v, None, TOL_F32)


@pytest.mark.parametrize("algorithm", ["chunked", "segmented"])
@pytest.mark.parametrize("T", [200, 1000])
def test_extreme_decays(algorithm, T):
    # gamma = 0 (each state holds only the current token), decays fast enough that the
    # segment weights gamma^(len - 1 - tau) underflow to zero, gamma = 1/2 (where the
    # segment-summary kernel switches how it forms its weights), and gamma = 1.  Checked
    # per head, so that the gamma = 1 heads' larger outputs do not set the other heads'
    # bound.
    gam = [float(np.float32(x)) for x in (0.0, 0.05, 0.3, 0.5, 0.7, 1.0)]
    w = Workload("extreme_decay", B=1, H=len(gam), T=T, dk=128, dv=128, C=64, dtype="bf16",
                 scale=1.0 / math.sqrt(128), feature_map="identity", decay=True,
                 normalize=False)
    q, k, v = make_inputs(w, seed=7, device="cuda", gen_device="cpu")
    out, S, _ = gpu_prefill(q, k, v, C=64, feature_map="identity", gamma=gam, normalize=False,
                            kernel_path="tensor_core", algorithm=algorithm,
                            segment_chunks=2 if algorithm == "segmented" else 0)
    o_ref, S_ref, _ = oracle_prefill(q, k, v, feature_map="identity", gamma=gam,
                                     normalize=False)
    o, s = to_np(out), to_np(S)
    for h, g in enumerate(gam):
        assert_close(o[:, h], o_ref[:, h], TOL_BF16, f"out, gamma={g}")
        assert_close(s[:, h], S_ref[:, h], TOL_BF16, f"S_final, gamma={g}")


def test_segmented_decay_windows():
    # Segments of 40 chunks with decays whose renormalisation windows are 6 (gamma 0.9)
    # to 16 chunks (gamma >= 0.97) long, so that every head rescales its carried prefix
    # at least twice inside a segment; 0.6 keeps the per-chunk decay.  Ragged tail.
    gam = [float(np.float32(x)) for x in (0.6, 0.9, 0.95, 0.97, 0.99, 1.0)]
    T = 2 * 40 * 64 + 100
    w = Workload("decay_windows", B=1, H=len(gam), T=T, dk=128, dv=128, C=64, dtype="bf16",
                 scale=1.0 / math.sqrt(128), feature_map="identity", decay=True,
                 normalize=False)
    q, k, v = make_inputs(w, seed=3, device="cuda", gen_device="cpu")
    out, S, _ = gpu_prefill(q, k, v, C=64, feature_map="identity", gamma=gam, normalize=False,
                            kernel_path="tensor_core", algorithm="segmented", segment_chunks=40)
    o_ref, S_ref, _ = oracle_prefill(q, k, v, feature_map="identity", gamma=gam,
                                     normalize=False)
    o, s = to_np(out), to_np(S)
    for h, g in enumerate(gam):
        assert_close(o[:, h], o_ref[:, h], TOL_BF16, f"out, gamma={g}")
        assert_close(s[:, h], S_ref[:, h], TOL_BF16, f"S_final, gamma={g}")
