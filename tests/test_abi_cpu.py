"""The C-ABI library without a GPU: it loads, exports every symbol the header declares,
sizes the workspace as documented, and rejects bad arguments before touching CUDA."""

from __future__ import annotations

import ctypes
import math
import re
from pathlib import Path

import numpy as np
import pytest

ROOT = Path(__file__).resolve().parent.parent
HEADER = ROOT / "include" / "linattn.h"


@pytest.fixture(scope="module")
def lib():
    from chunked_causal_linear_b200.build import build
    from chunked_causal_linear_b200.binding import load_library
    build()
    return load_library()


def header_functions() -> list[str]:
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(lin_attn_\w+)\s*\(",
                                 text, flags=re.M)))


def test_header_declares_the_expected_entry_points():
    from chunked_causal_linear_b200.binding import EXPORTED_SYMBOLS
    assert header_functions() == sorted(EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name


def test_library_links_no_torch(lib):
    # The libraries the build declared it needs (the dynamic section's NEEDED entries of the
    # library built here), independent of the search path.
    import subprocess
    from chunked_causal_linear_b200.binding import LIB_PATH
    out = subprocess.run(["readelf", "-d", str(LIB_PATH)], capture_output=True, text=True,
                         check=True).stdout
    needed = [l for l in out.splitlines() if "NEEDED" in l]
    assert needed and not any("torch" in l or "c10" in l for l in needed), needed


def test_status_strings_and_version(lib):
    from chunked_causal_linear_b200 import binding as b
    for code, name in b.STATUS_NAMES.items():
        assert b.lin_attn_status_string(code) == name
    assert b.lin_attn_status_string(99) == "LA_ERR_UNKNOWN"
    assert b.lin_attn_version() == 10100


def expected_workspace(B, H, T, dk, dv, C, normalize):
    if B * H == 0 or T == 0:
        return 0
    nc = -(-T // C)
    R = dk * dv + (dk if normalize else 0)
    gmax = min(2048, -(-nc // 16)) if nc > 2048 else 0
    a256 = lambda x: (x + 255) // 256 * 256
    return a256(B * H * nc * R * 4) + a256(B * H * gmax * R * 4)


@pytest.mark.parametrize("shape", [(1, 2, 256, 32, 32, 32, 1), (4, 16, 4096, 64, 64, 64, 1),
                                   (2, 32, 15990, 128, 128, 64, 1),
                                   (1, 32, 131072, 128, 128, 64, 0),
                                   (1, 8, 1048576, 64, 64, 64, 1), (1, 1, 1, 16, 16, 16, 0),
                                   (0, 4, 100, 64, 64, 64, 1), (3, 3, 0, 64, 64, 64, 1)])
def test_workspace_bytes(lib, shape):
    from chunked_causal_linear_b200.binding import lin_attn_prefill_workspace_bytes
    assert lin_attn_prefill_workspace_bytes(*shape) == expected_workspace(*shape)


SCAN_SIZES = (1, 2, 3, 7, 31, 32, 33, 64, 127, 128, 129, 250, 1000, 2047, 2048, 2049, 4096,
              16384, 32768, 32769, 100000, 1 << 20)


@pytest.mark.parametrize("n", SCAN_SIZES)
def test_scan_plan_shape_and_depth(lib, n):
    from chunked_causal_linear_b200 import binding as B
    p = B.lin_attn_scan_plan(n)
    ng, e, ls, g = p["groups"], p["per_group"], p["segment_len"], p["segments"]
    assert ng & (ng - 1) == 0 and 1 <= ng <= 128
    if n <= 2048:
        assert (ls, g) == (n, 1)
        m = n
    else:
        assert ls >= 16 and g == -(-n // ls) and g <= 2048 and (g - 1) * ls < n
        m = g
    assert ng * e >= m and (ng // 2) * e < m or ng == 1
    assert e <= 16 or n > 32768
    want = 2 * e + int(math.log2(ng)) + (2 * ls if n > 2048 else 0)
    assert p["depth"] == want
    if n <= 32768:
        assert p["depth"] <= 2 * 16 + 2 * 16 + 7
    assert B.lin_attn_scan_plan(n, "sequential")["depth"] == n


def _blocked_scan_model(x, a, init, plan):
    """Host restatement of the log-depth arrangement the plan describes (fold each group,
    Hillis-Steele over group folds, re-scan each group), to check that the plan's groups
    and segments cover every element exactly once; returns exclusive prefixes and total."""
    def blocked(xs, as_, init_):
        m = len(xs)
        ng, e = plan_block(m)
        folds, decays = [], []
        for gi in range(ng):
            agg, A = np.zeros_like(xs[0]), 1.0
            for j in range(gi * e, min(m, gi * e + e)):
                agg = as_[j] * agg + xs[j]
                A *= as_[j]
            folds.append(agg)
            decays.append(A)
        d = 1
        while d < ng:
            nf, nd = list(folds), list(decays)
            for gi in range(d, ng):
                nf[gi] = decays[gi] * folds[gi - d] + folds[gi]
                nd[gi] = decays[gi] * decays[gi - d]
            folds, decays = nf, nd
            d *= 2
        out = [None] * m
        total = None
        for gi in range(ng):
            carry = init_ if gi == 0 else decays[gi - 1] * init_ + folds[gi - 1]
            for j in range(gi * e, min(m, gi * e + e)):
                out[j] = carry
                carry = as_[j] * carry + xs[j]
            if min(m, gi * e + e) == m and gi * e < m:
                total = carry
        return out, total

    def plan_block(m):
        ng = 1
        while ng < m and ng < 128:
            ng *= 2
        return ng, -(-m // ng)

    n = len(x)
    if n <= 2048:
        return blocked(x, a, init)
    ls, g = plan["segment_len"], plan["segments"]
    segs = [range(s * ls, min(n, s * ls + ls)) for s in range(g)]
    sx, sa = [], []
    for r in segs:
        agg, A = np.zeros_like(x[0]), 1.0
        for j in r:
            agg = a[j] * agg + x[j]
            A *= a[j]
        sx.append(agg)
        sa.append(A)
    pref, total = blocked(sx, sa, init)
    out = [None] * n
    for s, r in enumerate(segs):
        carry = pref[s]
        for j in r:
            out[j] = carry
            carry = a[j] * carry + x[j]
    return out, total


@pytest.mark.parametrize("n", [1, 5, 64, 129, 2048, 2049, 5000])
def test_scan_plan_covers_every_element(lib, n):
    from chunked_causal_linear_b200 import binding as B
    rng = np.random.default_rng(n)
    x = [rng.standard_normal(2) for _ in range(n)]
    a = list(rng.uniform(0.5, 1.0, n))
    init = rng.standard_normal(2)
    got, total = _blocked_scan_model(x, a, init, B.lin_attn_scan_plan(n))
    carry = init.copy()
    for j in range(n):
        np.testing.assert_allclose(got[j], carry, rtol=1e-12, atol=1e-12)
        carry = a[j] * carry + x[j]
    np.testing.assert_allclose(total, carry, rtol=1e-12, atol=1e-12)


def _args(**kw):
    from chunked_causal_linear_b200.binding import PrefillArgs
    a = PrefillArgs()
    base = dict(q=0x1000, k=0x2000000, v=0x4000000, out=0x6000000, B=1, H=2, T=128, dk=64,
                dv=64, C=64, feature_map=1, normalize=1, eps=0.0, dtype=0, scan_mode=0,
                kernel_path=0)
    base.update(kw)
    for key, val in base.items():
        setattr(a, key, val)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), 1), (dict(T=-5), 1), (dict(dk=0), 1), (dict(dtype=7), 1),
    (dict(feature_map=3), 1), (dict(scan_mode=2), 1), (dict(kernel_path=9), 1),
    (dict(feature_map=0, normalize=1), 1), (dict(eps=-1.0), 1), (dict(eps=float("inf")), 1),
    (dict(dk=5), 2), (dict(dv=256), 2), (dict(C=48), 2), (dict(C=128), 2),
    (dict(kernel_path=1, C=32), 2), (dict(kernel_path=1, dk=32), 2),
    (dict(kernel_path=1, dtype=1), 2),
    (dict(q=0), 1), (dict(out=0), 1), (dict(q=0x1001), 1), (dict(out=0x1008), 1),
    (dict(out=0x1000), 1), (dict(out=0x2000000 + 64), 1),
    (dict(workspace=0x100010), 1),
    (dict(algorithm=3), 1), (dict(algorithm=-1), 1), (dict(segment_chunks=-1), 1),
    (dict(segment_chunks=2000), 1),
    (dict(algorithm=2, dv=64), 2), (dict(algorithm=2, C=32), 2), (dict(algorithm=2, dtype=1), 2),
    (dict(algorithm=2, kernel_path=2), 2),
])
def test_argument_errors_before_any_launch(lib, kw, status):
    a = _args(**kw)
    assert lib.lin_attn_prefill_ex(ctypes.byref(a)) == status


def test_empty_problems_return_ok_without_cuda(lib):
    for kw in (dict(B=0), dict(H=0), dict(T=0, S_final=None, Z_final=None)):
        a = _args(**kw)
        assert lib.lin_attn_prefill_ex(ctypes.byref(a)) == 0
    assert lib.lin_attn_prefill_ex(None) == 1


def test_gamma_validation(lib):
    a = _args(B=0)
    for bad in ([0.5, 1.5], [-0.1, 0.5], [float("nan"), 0.5]):
        arr = (ctypes.c_float * 2)(*bad)
        a.gamma = ctypes.cast(arr, ctypes.c_void_p)
        assert lib.lin_attn_prefill_ex(ctypes.byref(a)) == 1
    arr = (ctypes.c_float * 2)(0.0, 1.0)
    a.gamma = ctypes.cast(arr, ctypes.c_void_p)
    assert lib.lin_attn_prefill_ex(ctypes.byref(a)) == 0
    big = _args(B=0, H=2000)
    arr2 = (ctypes.c_float * 2000)(*([0.5] * 2000))
    big.gamma = ctypes.cast(arr2, ctypes.c_void_p)
    assert lib.lin_attn_prefill_ex(ctypes.byref(big)) == 2


def test_decode_argument_errors(lib):
    f = lib.lin_attn_decode_step
    assert f(None, None, None, None, None, None, 1, 1, 64, 64, 1, None, 1, None) == 1
    assert f(None, None, None, None, None, None, -1, 1, 64, 64, 1, None, 1, None) == 1
    assert f(None, None, None, None, None, None, 1, 1, 512, 64, 1, None, 1, None) == 2
    assert f(None, None, None, None, None, None, 1, 1, 64, 64, 0, None, 1, None) == 1
    assert f(None, None, None, None, None, None, 0, 1, 64, 64, 1, None, 1, None) == 0


def test_binding_fails_loudly_without_library(tmp_path):
    from chunked_causal_linear_b200.binding import load_library
    with pytest.raises(RuntimeError):
        load_library(tmp_path / "missing.so")


@pytest.mark.parametrize("kw,status", [
    (dict(states_only=2), 1), (dict(states_only=-1), 1), (dict(S_init=0x1002), 1),
    (dict(Z_init=0x1001), 1), (dict(states_only=1, out=None, algorithm=2, dv=64), 2),
    (dict(reverse=2), 1), (dict(reverse=-1), 1), (dict(reverse=1, algorithm=1), 2),
    (dict(reverse=1, kernel_path=2), 2),
])
def test_initial_state_and_states_only_argument_errors(lib, kw, status):
    a = _args(**kw)
    assert lib.lin_attn_prefill_ex(ctypes.byref(a)) == status


def test_states_only_needs_no_output_for_an_empty_problem(lib):
    a = _args(B=0, out=None, states_only=1)
    assert lib.lin_attn_prefill_ex(ctypes.byref(a)) == 0


def test_combine_states_argument_errors(lib):
    f = lib.lin_attn_combine_states
    toks = (ctypes.c_longlong * 3)(10, 20, 30)
    g_ok = (ctypes.c_float * 2)(0.5, 1.0)
    g_bad = (ctypes.c_float * 2)(0.5, 1.5)
    S, O = 0x100000, 0x200000
    assert f(S, None, 3, 4, toks, 1, 2, 64, 64, g_ok, O, None, None) == 1   # upto > parts
    assert f(S, None, 3, -1, toks, 1, 2, 64, 64, g_ok, O, None, None) == 1
    assert f(S, None, 65, 1, toks, 1, 2, 64, 64, g_ok, O, None, None) == 2  # > 64 parts
    assert f(S, None, 3, 1, toks, 1, 2, 64, 64, g_bad, O, None, None) == 1  # gamma > 1
    assert f(None, None, 3, 1, toks, 1, 2, 64, 64, g_ok, O, None, None) == 1
    assert f(S, None, 3, 1, toks, 1, 2, 64, 64, g_ok, O, 0x300000, None) == 1  # Z_out, no Z
    neg = (ctypes.c_longlong * 3)(10, -1, 30)
    assert f(S, None, 3, 1, neg, 1, 2, 64, 64, g_ok, O, None, None) == 1
    assert f(S, None, 3, 1, toks, 0, 2, 64, 64, g_ok, O, None, None) == 0   # empty


def _bwd_args(**kw):
    from chunked_causal_linear_b200.binding import BackwardArgs
    a = BackwardArgs()
    base = dict(q=0x1000, k=0x2000000, v=0x4000000, grad_out=0x6000000, grad_q=0x8000000,
                grad_k=0xA000000, grad_v=0xC000000, B=1, H=2, T=128, dk=64, dv=64, C=64,
                feature_map=0, dtype=0, out_dtype=0, scan_mode=0, kernel_path=0)
    base.update(kw)
    for key, val in base.items():
        setattr(a, key, val)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), 1), (dict(dtype=7), 1), (dict(feature_map=3), 1), (dict(out_dtype=5), 1),
    (dict(scan_mode=4), 1), (dict(algorithm=9), 1),
    (dict(dk=5), 2), (dict(dv=256), 2), (dict(C=48), 2), (dict(kernel_path=1, dtype=1), 2),
    (dict(algorithm=2), 2),  # dv = 64: no pass can take the segmented algorithm
    (dict(q=0), 1), (dict(grad_out=0), 1), (dict(grad_q=0), 1), (dict(grad_v=0), 1),
    (dict(q=0x1008), 1), (dict(grad_k=0x8000008), 1),
    (dict(grad_q=0x1000), 1),                       # grad_q is q
    (dict(grad_v=0x6000000 + 256), 1),              # grad_v inside grad_out
    (dict(grad_k=0x8000000 + 16), 1),               # grad_k overlaps grad_q
    (dict(S_init=0x100004), 1), (dict(grad_S_final=0x100008), 1),
    (dict(grad_S_init=0x100002), 1), (dict(workspace=0x100010), 1),
    # the normalised form: ELU+1 only, a valid eps, aligned normaliser states
    (dict(normalize=1), 1), (dict(normalize=2, feature_map=1), 1),
    (dict(normalize=1, feature_map=1, eps=-1.0), 1),
    (dict(normalize=1, feature_map=1, eps=float("nan")), 1),
    (dict(normalize=1, feature_map=1, Z_init=0x100004), 1),
    (dict(normalize=1, feature_map=1, grad_Z_final=0x100008), 1),
    (dict(normalize=1, feature_map=1, grad_Z_init=0x100004), 1),
])
def test_backward_argument_errors_before_any_launch(lib, kw, status):
    a = _bwd_args(**kw)
    assert lib.lin_attn_backward(ctypes.byref(a)) == status


def test_backward_gamma_and_empty_problems(lib):
    assert lib.lin_attn_backward(None) == 1
    for kw in (dict(B=0), dict(H=0)):
        assert lib.lin_attn_backward(ctypes.byref(_bwd_args(**kw))) == 0
    a = _bwd_args(B=0)
    for bad in ([0.5, 1.5], [-0.1, 0.5], [float("nan"), 0.5]):
        arr = (ctypes.c_float * 2)(*bad)
        a.gamma = ctypes.cast(arr, ctypes.c_void_p)
        assert lib.lin_attn_backward(ctypes.byref(a)) == 1
    # the ELU+1 map with a decay has no segmented pass
    arr = (ctypes.c_float * 2)(0.5, 0.9)
    a = _bwd_args(dk=128, dv=128, feature_map=1, algorithm=2)
    a.gamma = ctypes.cast(arr, ctypes.c_void_p)
    assert lib.lin_attn_backward(ctypes.byref(a)) == 2


def test_backward_workspace_bytes(lib):
    import torch
    from chunked_causal_linear_b200 import binding as B
    q = torch.empty(2, 3, 100, 64, dtype=torch.bfloat16)
    v = torch.empty(2, 3, 100, 128, dtype=torch.bfloat16)
    pw = B.lin_attn_prefill_workspace_bytes(2, 3, 100, 64, 128, 64, False)
    al = lambda x: (x + 255) // 256 * 256
    n_k, n_v = 2 * 3 * 100 * 64, 2 * 3 * 100 * 128
    # identity map, bf16 out: four reversed inputs, two bf16 reversed outputs
    want = 2 * al(n_k * 2) + 2 * al(n_v * 2) + al(n_k * 2) + al(n_v * 2) + pw
    assert B.lin_attn_backward_workspace_bytes(q, v) == want
    # ELU+1: psi(q) reversed and psi(k) with their bf16 residuals, float32 reversed
    # outputs, the float32 grad_q precursor, the lo passes' outputs, and the two states of
    # grad_S_final
    ns = al(2 * 3 * 64 * 128 * 4)
    want = (6 * al(n_k * 2) + 2 * al(n_v * 2) + al(n_k * 4) + al(n_v * 4) + al(n_k * 4)
            + 2 * al(n_k * 4) + 2 * ns + pw)
    assert B.lin_attn_backward_workspace_bytes(q, v, feature_map="elu1", grad_S_final=True) == want
    assert B.lin_attn_backward_workspace_bytes(q[:, :, :0], v[:, :, :0]) == 0
    # dk = dv = 128: the reversed passes run as reverse-mode prefills, with no reversed
    # copies; identity map with float32 gradients needs the prefill workspace alone
    q2 = torch.empty(2, 3, 100, 128, dtype=torch.bfloat16)
    pw2 = B.lin_attn_prefill_workspace_bytes(2, 3, 100, 128, 128, 64, False)
    assert B.lin_attn_backward_workspace_bytes(q2, q2, out_dtype="f32") == pw2
    n2 = 2 * 3 * 100 * 128
    want = 4 * al(n2 * 2) + 4 * al(n2 * 4) + pw2  # ELU+1: psi(q), psi(k) hi / lo; Wk, Wq, lo
    assert B.lin_attn_backward_workspace_bytes(q2, q2, feature_map="elu1", out_dtype="f32") == want
    # normalised: the scans' segment records hold segments of at least 64 tokens
    ns_seg = min(-(-148 * 32 // 6), -(-100 // 64))
    ls = -(-100 // ns_seg)
    ns_seg = -(-100 // ls)
    # dn as hi / lo, grad_v's float32 output and its lo pass's, dd, 1 / d, the g term
    extra = (2 * al(n2 * 2) + 2 * al(n2 * 4) + 2 * al(6 * 100 * 4) + al(n2 * 4)
             + al(6 * ns_seg * 128 * 4))
    assert B.lin_attn_backward_workspace_bytes(q2, q2, feature_map="elu1", out_dtype="f32",
                                               normalize=True) == want + extra


def test_gla_argument_errors_before_any_launch(lib):
    from chunked_causal_linear_b200.binding import GlaArgs
    def args(**kw):
        a = GlaArgs()
        base = dict(q=0x1000, k=0x2000000, v=0x4000000, alpha=0x6000000, out=0x8000000, B=1,
                    H=2, T=128, dk=64, dv=64, C=64, dtype=0, out_dtype=0)
        base.update(kw)
        for key, val in base.items():
            setattr(a, key, val)
        return a
    cases = [(dict(B=-1), 1), (dict(dtype=5), 1), (dict(out_dtype=3), 1), (dict(dk=12), 2),
             (dict(dv=136), 2), (dict(C=128), 2), (dict(alpha=0), 1), (dict(out=0), 1),
             (dict(out=0x1000), 1), (dict(out=0x6000000 + 64), 1), (dict(S_init=0x100004), 1),
             (dict(workspace=0x100010), 1), (dict(q=0x1008), 1), (dict(alpha=0x6000004), 1),
             (dict(kernel_path=5), 1), (dict(kernel_path=1, dtype=1), 2),
             (dict(kernel_path=1, C=32), 2), (dict(kernel_path=1, dk=32), 2),
             (dict(kernel_path=1, dv=64), 2), (dict(segment_chunks=-1), 1),
             (dict(segment_chunks=1025), 1), (dict(B=0), 0), (dict(H=0), 0)]
    for kw, status in cases:
        assert lib.lin_attn_gla_prefill(ctypes.byref(args(**kw))) == status, kw
    assert lib.lin_attn_gla_prefill(None) == 1
    # enough for either path: one record of dk*dv + dk floats per chunk (the CUDA cores' chunk
    # records, or the tensor cores' segment records, at most one per chunk), then one flag
    # byte per chunk
    al = lambda x: (x + 255) // 256 * 256
    n = lib.lin_attn_gla_workspace_bytes(2, 3, 100, 64, 32, 64)
    assert n == al(2 * 3 * 2 * (64 * 32 + 64) * 4) + al(2 * 3 * 2)


def test_header_is_plain_c_and_the_binding_structs_match_it(tmp_path):
    """The header compiles as strict C99, and every ctypes struct of the binding has the C
    struct's size and field offsets (a field added or moved on one side only fails here)."""
    import shutil
    import subprocess
    from chunked_causal_linear_b200 import binding as Bnd
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    structs = {"la_prefill_args": Bnd.PrefillArgs, "la_backward_args": Bnd.BackwardArgs,
               "la_gla_args": Bnd.GlaArgs}
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "linattn.h"', 'int main(void) {']
    for cname, py in structs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", str(ROOT / "include"),
                    str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {tuple(l.split()[:2]): int(l.split()[2]) for l in out if l.strip()}
    for cname, py in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)
