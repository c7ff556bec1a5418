"""The benchmark's algorithmic-byte models and the oracle's thread independence for the
backward and gated loops (CPU only).

The byte models are the figures the roofline fractions divide by; they are checked here
against the per-unit formulas stated beside each kernel (bytes any correct kernel must move),
written out for the 128k-token retention workload, and against each other.
"""

from __future__ import annotations

import numpy as np

import bench
from chunked_causal_linear_b200.workloads import WORKLOADS
from oracle.oracle import default_oracle


def test_forward_kernel_bytes_match_the_per_unit_formulas():
    w = WORKLOADS["retention_128k"]
    BH, T, d, C = 32, 131072, 128, 64
    NC = T // C
    lseg = bench.segment_length(w)
    NS = NC // lseg
    R = d * d
    e_in, e_out = 2, 4
    # k1_seg: k, v once, one record per segment
    assert bench.kernel_bytes(w, "k1_seg", e_out, "segmented") == BH * T * 2 * d * e_in + BH * NS * R * 4
    # k3_seg: q, k, v once, the output once, one prefix per segment
    assert bench.kernel_bytes(w, "k3_seg", e_out, "segmented") == \
        BH * T * 3 * d * e_in + BH * T * d * e_out + BH * NS * R * 4
    # the chunked arrangement's record passes
    assert bench.kernel_bytes(w, "k2_downsweep", e_out, "chunked") > 2 * BH * NC * R * 4


def test_backward_bytes_are_three_prefills_on_the_retention_workload():
    w = WORKLOADS["retention_128k"]
    ops = bench.backward_bytes(w, 4, "auto")
    names = [n for n, _ in ops]
    # reverse-mode passes: no element-wise kernel, three (k1_seg, the scan, k3_seg); 32
    # segments per head, so the scan's block level is the warp scan
    assert names == ["k1_seg", "k2_warp_scan", "k3_seg"] * 3
    k3 = [b for n, b in ops if n == "k3_seg"]
    assert len(set(k3)) == 1 and k3[0] == bench.kernel_bytes(w, "k3_seg", 4, "segmented")


def test_backward_bytes_of_the_normalised_form_add_the_scans():
    w = WORKLOADS["ragged_b2h32"]
    names = [n for n, _ in bench.backward_bytes(w, 4, "auto")]
    for n in ("bwd_z_scan", "bwd_scaled_psi_q", "bwd_g_scan", "bwd_reverse_outputs"):
        assert n in names
    # six prefills: grad_q and dpsi(k) passes on psi's hi and lo halves, grad_v on dn's
    assert names.count("k3_seg") == 6


def test_oracle_backward_and_gla_do_not_depend_on_the_thread_count():
    rng = np.random.default_rng(0)
    q, k, v = (rng.standard_normal((2, 3, 40, 8)).astype(np.float32) for _ in range(3))
    do = rng.standard_normal((2, 3, 40, 8))
    a = (1 / (1 + np.exp(-rng.normal(2, 1, (2, 3, 40, 8))))).astype(np.float32)
    o = default_oracle()
    b1 = o.backward(q, k, v, do, feature_map="elu1", normalize=True, eps=0.1, nthreads=1)
    b4 = o.backward(q, k, v, do, feature_map="elu1", normalize=True, eps=0.1, nthreads=4)
    assert all(np.array_equal(x, y) for x, y in zip(b1, b4))
    g1 = o.gla_forward(q, k, v, a, nthreads=1)
    g4 = o.gla_forward(q, k, v, a, nthreads=4)
    assert all(np.array_equal(x, y) for x, y in zip(g1, g4))


def test_scan_kernel_names_follow_the_element_count():
    """Up to 32 scan elements the block level is k2_warp_scan, beyond it k2_block_scan; two
    levels put the block level between k2_reduce and k2_downsweep."""
    base = WORKLOADS["retention_128k"]
    assert bench.kernel_names(base, "segmented", "logdepth") == ["k1_seg", "k2_warp_scan", "k3_seg"]
    assert bench.kernel_names(base, "chunked", "logdepth") == ["k1_tc", "k2_block_scan", "k3_tc"]
    assert bench.kernel_names(base, "chunked", "sequential") == ["k1_tc", "k2_sequential", "k3_tc"]
    long = base.with_(T=64 * 16384)  # 16384 chunks: two levels over 1024 segments of 16
    assert bench.kernel_names(long, "chunked", "logdepth") == \
        ["k1_tc", "k2_reduce", "k2_block_scan", "k2_downsweep", "k3_tc"]
    assert bench.kernel_bytes(base, "k2_warp_scan", 4, "segmented") == \
        bench.kernel_bytes(base, "k2_block_scan", 4, "segmented")
