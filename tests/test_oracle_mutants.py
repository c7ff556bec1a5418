"""Plants plausible mistakes in a copy of the oracle and checks that the pins catch them.

Each mutant is a text edit of the oracle's C++ source (a dropped term, a wrong index, a
wrong feature-map branch, decay in the wrong place, exclusive instead of inclusive
readout, a stray epsilon).  The edited copy is compiled into a temporary library and
run through a compact version of the pin suite; at least one pin must fail for every
mutant, and none for the unedited source.  Nothing here touches the real oracle.
"""

from __future__ import annotations

import math

import numpy as np
import pytest

import independent_forms as F
from oracle.oracle import SRC, Oracle, build
from test_oracle_pins import EXAMPLE_INPUTS, GOLDEN, _load_examples, rel_err


def _pin_suite(o: Oracle) -> dict[str, bool]:
    res: dict[str, bool] = {}
    rng = np.random.default_rng(0)

    rows = [l.split() for l in (GOLDEN / "feature_map_closed_forms.txt").read_text().splitlines()
            if l.strip() and not l.startswith("#")]
    x = np.array([float(r[0]) for r in rows])
    res["psi_closed_forms"] = bool(np.allclose(o.feature_map(x), [float(r[1]) for r in rows],
                                               rtol=1e-15, atol=0))

    ok = True
    ex = _load_examples()
    for name, e in EXAMPLE_INPUTS.items():
        q, k, v = (np.array(e[c], np.float32).reshape(1, 1, 3, 1) for c in "qkv")
        out, S, Z = o.forward(q, k, v, feature_map=e["fm"], normalize=e["norm"], gamma=e["gamma"])
        for qty, arr in (("out", out), ("S_final", S), ("Z_final", Z)):
            for idx, val in ex[name].get(qty, {}).items():
                ok &= math.isclose(arr.reshape(-1)[idx], val, rel_tol=1e-13, abs_tol=1e-14)
    q = np.array([[0, 1], [1, 0]], np.float32).reshape(1, 1, 2, 2)
    k = np.array([[1, 0], [0, 1]], np.float32).reshape(1, 1, 2, 2)
    v = np.array([[1, 2], [3, 4]], np.float32).reshape(1, 1, 2, 2)
    out, S, Z = o.forward(q, k, v, feature_map="identity", normalize=False)
    for qty, arr in (("out", out), ("S_final", S), ("Z_final", Z)):
        for idx, val in ex["D"].get(qty, {}).items():
            ok &= math.isclose(arr.reshape(-1)[idx], val, rel_tol=1e-13, abs_tol=1e-14)
    res["worked_examples"] = bool(ok)

    q, k, v = (rng.standard_normal((1, 2, 45, d)).astype(np.float32) * 0.5 for d in (6, 6, 5))
    for norm in (True, False):
        out, _, _ = o.forward(q, k, v, normalize=norm)
        res[f"masked_quadratic_norm{int(norm)}"] = rel_err(
            out, F.masked_quadratic(q, k, v, "elu1", norm)) < 1e-12

    g = [0.9, 0.6]
    out, S, Z = o.forward(q, k, v, feature_map="identity", normalize=False, gamma=g)
    res["retention_parallel"] = rel_err(out, F.retention_parallel(q, k, v, g)) < 1e-12
    S_ref, Z_ref = F.final_state_closed(k, v, g, "identity")
    res["final_state_S"] = rel_err(S, S_ref) < 1e-12
    res["final_state_Z"] = rel_err(Z, Z_ref) < 1e-12

    out, S, Z = o.forward(q, k, v, feature_map="elu1", normalize=True, gamma=g)
    o2, S2, Z2, _ = F.chunked_scan(q, k, v, 8, g, "elu1", True)
    res["chunked_scan"] = max(rel_err(out, o2), rel_err(S, S2), rel_err(Z, Z2)) < 1e-12

    u = rng.standard_normal(5).astype(np.float32)
    vc = np.broadcast_to(u, v.shape).copy()
    out, _, _ = o.forward(q, k, vc, normalize=True, gamma=g)
    res["constant_rows"] = float(np.max(np.abs(out - u))) < 1e-13

    out, _, _ = o.forward(q, k, v, normalize=False, gamma=[0.0, 0.0])
    ref = np.sum(F.psi(q, "elu1") * F.psi(k, "elu1"), -1, keepdims=True) * v.astype(np.float64)
    res["gamma_zero"] = rel_err(out, ref) < 1e-14
    return res


MUTANTS = {
    "decay_dropped_on_state": ("Si[j] = g * Si[j] + fk[i]", "Si[j] = Si[j] + fk[i]"),
    "decay_dropped_on_normaliser": ("Z[i] = g * Z[i] + fk[i];", "Z[i] = Z[i] + fk[i];"),
    "decay_applied_to_current_token": (
        "Si[j] = g * Si[j] + fk[i] * static_cast<double>(vt[j]);",
        "Si[j] = g * (Si[j] + fk[i] * static_cast<double>(vt[j]));"),
    "value_index_reversed": ("fk[i] * static_cast<double>(vt[j])",
                             "fk[i] * static_cast<double>(vt[dv - 1 - j])"),
    "feature_map_missing_plus_one": ("x > 0.0 ? x + 1.0 : std::exp(x)",
                                     "x > 0.0 ? x : std::exp(x)"),
    "feature_map_wrong_branch_point": ("x > 0.0 ? x + 1.0 : std::exp(x)",
                                       "x > 0.5 ? x + 1.0 : std::exp(x)"),
    "exclusive_readout": ("num[j] += fq[i] * Si[j];",
                          "num[j] += fq[i] * (Si[j] - fk[i] * static_cast<double>(v[t * dv + j]));"),
    "query_uses_key_map": ("fq[i] = feature_map(static_cast<double>(q[t * dk + i]), p.fm);",
                           "fq[i] = feature_map(static_cast<double>(k[t * dk + i]), p.fm);"),
    "stray_epsilon": ("num[j] / (den + p.eps)", "num[j] / (den + 1e-9)"),
    "normaliser_not_inclusive": ("den += fq[i] * Z[i];", "den += fq[i] * (Z[i] - fk[i]);"),
}


@pytest.fixture(scope="module")
def source_text():
    return SRC.read_text()


def test_unmutated_source_passes_every_pin(tmp_path, source_text):
    lib = build(SRC, tmp_path / "clean.so", force=True)
    res = _pin_suite(Oracle(lib))
    assert all(res.values()), res


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, source_text, name):
    old, new = MUTANTS[name]
    assert source_text.count(old) >= 1, f"mutation site for {name} not found"
    src = tmp_path / f"{name}.cpp"
    src.write_text(source_text.replace(old, new))
    lib = build(src, tmp_path / f"{name}.so", force=True)
    res = _pin_suite(Oracle(lib))
    failed = [k for k, ok in res.items() if not ok]
    assert failed, f"mutant {name} passed every pin"
