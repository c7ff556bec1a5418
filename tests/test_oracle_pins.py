"""Pins for the fp64 CPU oracle (CPU only).

The oracle is a token loop.  Each test below checks it against something that is not
the oracle: closed forms worked out by hand, a different formula the pages state to be
equal (the masked quadratic form, the parallel retention form, the closed-form final
state, chunk summaries combined by a Hillis-Steele scan), or an invariant that the
mathematics fixes (constant values are reproduced exactly by the normalised form,
linearity in v, causality, the gamma = 0 / gamma = 1 special cases).
"""

from __future__ import annotations

import math
from pathlib import Path

import numpy as np
import pytest

import independent_forms as F

GOLDEN = Path(__file__).resolve().parent / "golden"


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    scale = max(float(np.max(np.abs(b))) if b.size else 0.0, 1e-300)
    return float(np.max(np.abs(a - b))) / scale if b.size else 0.0


def rand_qkv(rng, B, H, T, dk, dv, scale=0.5, dtype=np.float32):
    q = (rng.standard_normal((B, H, T, dk)) * scale).astype(dtype)
    k = (rng.standard_normal((B, H, T, dk)) * scale).astype(dtype)
    v = (rng.standard_normal((B, H, T, dv)) * scale).astype(dtype)
    return q, k, v


# ---------------------------------------------------------------------------------------
# Closed forms and hand-derived examples


def test_feature_map_closed_forms(oracle):
    rows = [l.split() for l in (GOLDEN / "feature_map_closed_forms.txt").read_text().splitlines()
            if l.strip() and not l.startswith("#")]
    x = np.array([float(r[0]) for r in rows])
    want = np.array([float(r[1]) for r in rows])
    got = oracle.feature_map(x, "elu1")
    np.testing.assert_allclose(got, want, rtol=2e-16, atol=0)
    np.testing.assert_array_equal(oracle.feature_map(x, "identity"), x)


def _load_examples():
    ex = {}
    for l in (GOLDEN / "worked_scalar_examples.txt").read_text().splitlines():
        if not l.strip() or l.startswith("#"):
            continue
        name, qty, idx, val = l.split()
        ex.setdefault(name, {}).setdefault(qty, {})[int(idx)] = float(val)
    return ex


EXAMPLE_INPUTS = {
    "A": dict(q=[0.5, -1, 2], k=[-1, 0.5, 0], v=[2, -4, 1], fm="elu1", norm=True, gamma=None),
    "B": dict(q=[0.5, -1, 2], k=[-1, 0.5, 0], v=[2, -4, 1], fm="elu1", norm=False, gamma=None),
    "C": dict(q=[0.5, -1, 2], k=[-1, 0.5, 0], v=[2, -4, 1], fm="identity", norm=False,
              gamma=[0.5]),
}


@pytest.mark.parametrize("name", ["A", "B", "C", "D"])
def test_worked_examples(oracle, name):
    ex = _load_examples()[name]
    if name == "D":
        q = np.array([[0, 1], [1, 0]], np.float32).reshape(1, 1, 2, 2)
        k = np.array([[1, 0], [0, 1]], np.float32).reshape(1, 1, 2, 2)
        v = np.array([[1, 2], [3, 4]], np.float32).reshape(1, 1, 2, 2)
        out, S, Z = oracle.forward(q, k, v, feature_map="identity", normalize=False)
    else:
        e = EXAMPLE_INPUTS[name]
        q, k, v = (np.array(e[x], np.float32).reshape(1, 1, 3, 1) for x in "qkv")
        out, S, Z = oracle.forward(q, k, v, feature_map=e["fm"], normalize=e["norm"],
                                   gamma=e["gamma"])
    for qty, arr in (("out", out), ("S_final", S), ("Z_final", Z)):
        flat = arr.reshape(-1)
        for idx, val in ex.get(qty, {}).items():
            assert flat[idx] == pytest.approx(val, rel=1e-14, abs=1e-15), (qty, idx)


# ---------------------------------------------------------------------------------------
# Equal forms


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("T,dk,dv", [(1, 4, 4), (37, 8, 5), (120, 16, 16), (200, 3, 12)])
@pytest.mark.parametrize("normalize", [True, False])
def test_masked_quadratic_form(oracle, seed, T, dk, dv, normalize):
    rng = np.random.default_rng(seed)
    q, k, v = rand_qkv(rng, 2, 2, T, dk, dv)
    out, _, _ = oracle.forward(q, k, v, feature_map="elu1", normalize=normalize)
    ref = F.masked_quadratic(q, k, v, "elu1", normalize)
    assert rel_err(out, ref) < 1e-12


@pytest.mark.parametrize("seed", [0, 1])
@pytest.mark.parametrize("T,dk,dv", [(1, 4, 4), (64, 8, 8), (150, 16, 6)])
def test_retention_parallel_form(oracle, seed, T, dk, dv):
    rng = np.random.default_rng(seed)
    H = 3
    q, k, v = rand_qkv(rng, 2, H, T, dk, dv)
    gammas = [0.96875, 0.5, 0.999]
    out, _, _ = oracle.forward(q, k, v, feature_map="identity", normalize=False, gamma=gammas)
    ref = F.retention_parallel(q, k, v, gammas, "identity", normalize=False)
    assert rel_err(out, ref) < 1e-12


def test_retention_parallel_form_normalised_decay(oracle):
    # Reading: with both decay and normalisation on, the normaliser decays like the state.
    rng = np.random.default_rng(7)
    q, k, v = rand_qkv(rng, 1, 2, 90, 8, 8)
    gammas = [0.9, 0.75]
    out, _, _ = oracle.forward(q, k, v, feature_map="elu1", normalize=True, gamma=gammas)
    ref = F.retention_parallel(q, k, v, gammas, "elu1", normalize=True)
    assert rel_err(out, ref) < 1e-12


@pytest.mark.parametrize("decay", [False, True])
@pytest.mark.parametrize("fm", ["elu1", "identity"])
def test_final_state_closed_form(oracle, decay, fm):
    rng = np.random.default_rng(3)
    q, k, v = rand_qkv(rng, 2, 2, 173, 8, 12)
    gammas = [0.97, 0.8] if decay else None
    _, S, Z = oracle.forward(q, k, v, feature_map=fm, normalize=False, gamma=gammas)
    S_ref, Z_ref = F.final_state_closed(k, v, gammas, fm)
    assert rel_err(S, S_ref) < 1e-12
    assert rel_err(Z, Z_ref) < 1e-12


@pytest.mark.parametrize("T,C", [(1, 4), (5, 4), (8, 4), (37, 8), (64, 8), (100, 32),
                                 (257, 32), (33, 32), (256, 16)])
@pytest.mark.parametrize("mode", ["norm", "decay_unnorm", "decay_norm"])
def test_chunked_scan_equals_sequential(oracle, T, C, mode):
    rng = np.random.default_rng(T * 31 + C)
    q, k, v = rand_qkv(rng, 1, 2, T, 8, 6)
    normalize = mode != "decay_unnorm"
    gammas = [0.96875, 0.7] if mode.startswith("decay") else None
    fm = "identity" if mode == "decay_unnorm" else "elu1"
    out, S, Z = oracle.forward(q, k, v, feature_map=fm, normalize=normalize, gamma=gammas)
    o2, S2, Z2, rounds = F.chunked_scan(q, k, v, C, gammas, fm, normalize)
    assert rel_err(out, o2) < 1e-12
    assert rel_err(S, S2) < 1e-12
    assert rel_err(Z, Z2) < 1e-12
    n_chunks = -(-T // C)
    assert rounds == (math.ceil(math.log2(n_chunks)) if n_chunks > 1 else 0)


# ---------------------------------------------------------------------------------------
# Invariants and special cases


@pytest.mark.parametrize("decay", [False, True])
def test_constant_value_rows_reproduced(oracle, decay):
    rng = np.random.default_rng(11)
    q, k, _ = rand_qkv(rng, 2, 2, 150, 16, 16)
    u = rng.standard_normal(16).astype(np.float32)
    v = np.broadcast_to(u, (2, 2, 150, 16)).copy()
    gammas = [0.9, 0.99] if decay else None
    out, _, _ = oracle.forward(q, k, v, feature_map="elu1", normalize=True, gamma=gammas)
    assert np.max(np.abs(out - u.astype(np.float64))) < 1e-13


@pytest.mark.parametrize("normalize", [True, False])
def test_linearity_in_v(oracle, normalize):
    rng = np.random.default_rng(5)
    q, k, v1 = rand_qkv(rng, 1, 2, 80, 8, 8)
    v2 = (rng.standard_normal(v1.shape) * 0.5).astype(np.float32)
    o1, _, _ = oracle.forward(q, k, v1, normalize=normalize)
    o2, _, _ = oracle.forward(q, k, v2, normalize=normalize)
    o12, _, _ = oracle.forward(q, k, (v1.astype(np.float64) + v2).astype(np.float32),
                               normalize=normalize)
    # v1 + v2 is rounded to float32 once; compare against the same rounded sum's parts.
    ref = o1 + o2
    assert rel_err(o12, ref) < 1e-6


def test_gamma_one_equals_undecayed(oracle):
    rng = np.random.default_rng(9)
    q, k, v = rand_qkv(rng, 1, 3, 70, 8, 8)
    a, Sa, Za = oracle.forward(q, k, v, feature_map="identity", normalize=False,
                               gamma=[1.0, 1.0, 1.0])
    b, Sb, Zb = oracle.forward(q, k, v, feature_map="identity", normalize=False)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(Sa, Sb)
    np.testing.assert_array_equal(Za, Zb)


def test_gamma_zero_keeps_only_the_diagonal(oracle):
    rng = np.random.default_rng(10)
    q, k, v = rand_qkv(rng, 1, 2, 40, 8, 5)
    out, _, _ = oracle.forward(q, k, v, feature_map="elu1", normalize=False, gamma=[0.0, 0.0])
    fq, fk = F.psi(q, "elu1"), F.psi(k, "elu1")
    ref = np.sum(fq * fk, axis=-1, keepdims=True) * v.astype(np.float64)
    assert rel_err(out, ref) < 1e-14


@pytest.mark.parametrize("t0", [0, 1, 31, 32, 99])
def test_causality_bitwise(oracle, t0):
    rng = np.random.default_rng(12)
    q, k, v = rand_qkv(rng, 1, 2, 100, 8, 8)
    out, _, _ = oracle.forward(q, k, v, gamma=[0.9, 0.95])
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[:, :, t0:] = 100.0
    k2[:, :, t0:] = -100.0
    v2[:, :, t0:] = 1e6
    out2, _, _ = oracle.forward(q2, k2, v2, gamma=[0.9, 0.95])
    np.testing.assert_array_equal(out[:, :, :t0], out2[:, :, :t0])


@pytest.mark.parametrize("normalize,fm,gammas", [(True, "elu1", None),
                                                  (False, "identity", [0.9, 0.97])])
def test_decode_continuation(oracle, normalize, fm, gammas):
    rng = np.random.default_rng(13)
    q, k, v = rand_qkv(rng, 2, 2, 61, 8, 8)
    full, S_full, Z_full = oracle.forward(q, k, v, feature_map=fm, normalize=normalize,
                                          gamma=gammas)
    _, S, Z = oracle.forward(q[:, :, :60], k[:, :, :60], v[:, :, :60], feature_map=fm,
                             normalize=normalize, gamma=gammas, want_out=False)
    step, S1, Z1 = oracle.forward(q[:, :, 60:], k[:, :, 60:], v[:, :, 60:], feature_map=fm,
                                  normalize=normalize, gamma=gammas, S_init=S, Z_init=Z)
    np.testing.assert_array_equal(step[:, :, 0], full[:, :, 60])
    np.testing.assert_array_equal(S1, S_full)
    np.testing.assert_array_equal(Z1, Z_full)


def test_empty_sequence(oracle):
    z = np.zeros((1, 2, 0, 8), np.float32)
    out, S, Z = oracle.forward(z, z, z)
    assert out.shape == (1, 2, 0, 8)
    assert not S.any() and not Z.any()


def test_thread_count_does_not_change_results(oracle):
    rng = np.random.default_rng(14)
    q, k, v = rand_qkv(rng, 2, 3, 50, 8, 8)
    a = oracle.forward(q, k, v, nthreads=1)
    b = oracle.forward(q, k, v, nthreads=4)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_pr1_golden_regression(oracle):
    """The committed pr1_ref expected values still come out of the oracle unchanged."""
    from golden.make_golden import load_golden, compute_golden
    stored = load_golden()
    fresh = compute_golden(oracle)
    for key in stored:
        np.testing.assert_array_equal(fresh[key], stored[key])
