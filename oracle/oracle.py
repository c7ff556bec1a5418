"""Test infrastructure only: Python access to the fp64 CPU oracle.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm of
``bench.py`` may import this module.  The CUDA library never calls it.

The oracle itself is ``linattn_oracle.cpp`` (a plain token loop in double precision;
its header states what it computes and which passages of the pages it follows).  This
module compiles it with g++ (no fast-math) and wraps the two exported functions with
numpy arrays.  Nothing here holds arithmetic of the method.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
SRC = HERE / "linattn_oracle.cpp"
LIB = HERE / "liblinattn_oracle.so"

FEATURE_MAPS = {"identity": 0, "elu1": 1}


def build(src: Path = SRC, out: Path = LIB, force: bool = False) -> Path:
    """Compile the oracle into a shared library (skipped when it is up to date)."""
    if not force and out.exists() and out.stat().st_mtime >= src.stat().st_mtime:
        return out
    tmp = out.with_suffix(f".{os.getpid()}.tmp.so")
    cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
           "-fno-fast-math", "-o", str(tmp), str(src)]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


class Oracle:
    """ctypes handle on one compiled copy of the oracle."""

    def __init__(self, lib_path: Path | str | None = None):
        path = Path(lib_path) if lib_path is not None else build()
        self.path = path
        self._lib = ctypes.CDLL(str(path))
        f = self._lib.la_oracle_forward
        f.restype = ctypes.c_int
        f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int, ctypes.c_int, ctypes.c_longlong,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_void_p, ctypes.c_int, ctypes.c_double,
                                              ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        b = self._lib.la_oracle_backward
        b.restype = ctypes.c_int
        b.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int, ctypes.c_int, ctypes.c_longlong,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_int] + \
            [ctypes.c_void_p, ctypes.c_int, ctypes.c_double] + [ctypes.c_void_p] * 9 + [ctypes.c_int]
        gb = self._lib.la_oracle_gla_backward
        gb.restype = ctypes.c_int
        gb.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_int, ctypes.c_longlong,
                                              ctypes.c_int, ctypes.c_int] + [ctypes.c_void_p] * 7 + \
            [ctypes.c_int]
        gl = self._lib.la_oracle_gla_forward
        gl.restype = ctypes.c_int
        gl.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int, ctypes.c_int, ctypes.c_longlong,
                                              ctypes.c_int, ctypes.c_int] + [ctypes.c_void_p] * 3 + \
            [ctypes.c_int]
        g = self._lib.la_oracle_feature_map
        g.restype = ctypes.c_int
        g.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int]

    def feature_map(self, x, feature_map: str = "elu1") -> np.ndarray:
        x = np.ascontiguousarray(x, dtype=np.float64)
        y = np.empty_like(x)
        rc = self._lib.la_oracle_feature_map(x.ctypes.data, y.ctypes.data, x.size,
                                             FEATURE_MAPS[feature_map])
        if rc != 0:
            raise ValueError(f"la_oracle_feature_map returned {rc}")
        return y

    def forward(self, q, k, v, *, feature_map: str = "elu1", gamma=None,
                normalize: bool = True, eps: float = 0.0, S_init=None, Z_init=None,
                want_out: bool = True, nthreads: int = 0):
        """Run the token loop.

        q, k: [B, H, T, dk]; v: [B, H, T, dv] (any float dtype; converted to float32,
        which is exact for bf16 and float32 inputs).  gamma: per-head decays (length H)
        or None.  Returns (out [B,H,T,dv] float64 or None, S_final [B,H,dk,dv],
        Z_final [B,H,dk]).
        """
        q = np.ascontiguousarray(q, dtype=np.float32)
        k = np.ascontiguousarray(k, dtype=np.float32)
        v = np.ascontiguousarray(v, dtype=np.float32)
        B, H, T, dk = q.shape
        dv = v.shape[-1]
        if k.shape != q.shape or v.shape[:3] != (B, H, T):
            raise ValueError("shape mismatch between q, k and v")
        g = None
        if gamma is not None:
            g = np.ascontiguousarray(np.asarray(gamma, dtype=np.float64).reshape(H))
        s0 = None if S_init is None else np.ascontiguousarray(S_init, dtype=np.float64)
        z0 = None if Z_init is None else np.ascontiguousarray(Z_init, dtype=np.float64)
        out = np.empty((B, H, T, dv), dtype=np.float64) if want_out else None
        S = np.empty((B, H, dk, dv), dtype=np.float64)
        Z = np.empty((B, H, dk), dtype=np.float64)

        def ptr(a):
            return None if a is None else a.ctypes.data

        rc = self._lib.la_oracle_forward(ptr(q), ptr(k), ptr(v), B, H, T, dk, dv,
                                         FEATURE_MAPS[feature_map], ptr(g), int(bool(normalize)),
                                         float(eps), ptr(s0), ptr(z0), ptr(out), ptr(S), ptr(Z),
                                         int(nthreads))
        if rc != 0:
            raise ValueError(f"la_oracle_forward returned {rc}")
        return out, S, Z

    def backward(self, q, k, v, dout, *, feature_map: str = "elu1", gamma=None,
                 normalize: bool = False, eps: float = 0.0, S_init=None, Z_init=None,
                 dS_final=None, dZ_final=None, nthreads: int = 0):
        """Gradients of L = <dout, out> + <dS_final, S_final> (+ <dZ_final, Z_final>
        normalised) with respect to q, k, v and the initial state.  Returns (dq, dk, dv,
        dS_init, dZ_init), float64 (dZ_init zero for the unnormalised form)."""
        q = np.ascontiguousarray(q, dtype=np.float32)
        k = np.ascontiguousarray(k, dtype=np.float32)
        v = np.ascontiguousarray(v, dtype=np.float32)
        do = np.ascontiguousarray(dout, dtype=np.float64)
        B, H, T, dk = q.shape
        dv = v.shape[-1]
        if k.shape != q.shape or v.shape[:3] != (B, H, T) or do.shape != v.shape:
            raise ValueError("shape mismatch between q, k, v and dout")
        g = None if gamma is None else np.ascontiguousarray(np.asarray(gamma, dtype=np.float64).reshape(H))
        f64 = lambda a: None if a is None else np.ascontiguousarray(a, dtype=np.float64)
        s0, z0, dsf, dzf = f64(S_init), f64(Z_init), f64(dS_final), f64(dZ_final)
        dq = np.empty((B, H, T, dk)); dk_ = np.empty((B, H, T, dk)); dv_ = np.empty((B, H, T, dv))
        ds0 = np.empty((B, H, dk, dv)); dz0 = np.empty((B, H, dk))
        ptr = lambda a: None if a is None else a.ctypes.data
        rc = self._lib.la_oracle_backward(ptr(q), ptr(k), ptr(v), ptr(do), B, H, T, dk, dv,
                                          FEATURE_MAPS[feature_map], ptr(g), int(bool(normalize)),
                                          float(eps), ptr(s0), ptr(z0), ptr(dsf), ptr(dzf),
                                          ptr(dq), ptr(dk_), ptr(dv_), ptr(ds0), ptr(dz0),
                                          int(nthreads))
        if rc != 0:
            raise ValueError(f"la_oracle_backward returned {rc}")
        return dq, dk_, dv_, ds0, dz0


    def gla_forward(self, q, k, v, alpha, *, S_init=None, want_out: bool = True,
                    nthreads: int = 0):
        """Gated linear attention's token loop: S_t = (alpha_t 1^T) (.) S_{t-1} + k_t^T v_t,
        o_t = q_t S_t.  q, k, alpha [B, H, T, dk]; v [B, H, T, dv].  Returns (out float64 or
        None, S_final [B, H, dk, dv])."""
        q, k, v, al = (np.ascontiguousarray(a, dtype=np.float32) for a in (q, k, v, alpha))
        B, H, T, dk = q.shape
        dv = v.shape[-1]
        if k.shape != q.shape or al.shape != q.shape or v.shape[:3] != (B, H, T):
            raise ValueError("shape mismatch between q, k, v and alpha")
        s0 = None if S_init is None else np.ascontiguousarray(S_init, dtype=np.float64)
        out = np.empty((B, H, T, dv)) if want_out else None
        S = np.empty((B, H, dk, dv))
        ptr = lambda a: None if a is None else a.ctypes.data
        rc = self._lib.la_oracle_gla_forward(ptr(q), ptr(k), ptr(v), ptr(al), B, H, T, dk, dv,
                                             ptr(s0), ptr(out), ptr(S), int(nthreads))
        if rc != 0:
            raise ValueError(f"la_oracle_gla_forward returned {rc}")
        return out, S


    def gla_backward(self, q, k, v, alpha, dout, *, S_init=None, dS_final=None,
                     nthreads: int = 0):
        """Gradients of <dout, out> + <dS_final, S_final> through the gated loop.  Returns
        (dq, dk, dv, dalpha, dS_init), float64."""
        q, k, v, al = (np.ascontiguousarray(a, dtype=np.float32) for a in (q, k, v, alpha))
        do = np.ascontiguousarray(dout, dtype=np.float64)
        B, H, T, dk = q.shape
        dv = v.shape[-1]
        if k.shape != q.shape or al.shape != q.shape or v.shape[:3] != (B, H, T) or do.shape != v.shape:
            raise ValueError("shape mismatch between q, k, v, alpha and dout")
        f64 = lambda a: None if a is None else np.ascontiguousarray(a, dtype=np.float64)
        s0, dsf = f64(S_init), f64(dS_final)
        dq = np.empty((B, H, T, dk)); dk_ = np.empty((B, H, T, dk)); dv_ = np.empty((B, H, T, dv))
        da = np.empty((B, H, T, dk)); ds0 = np.empty((B, H, dk, dv))
        ptr = lambda a: None if a is None else a.ctypes.data
        rc = self._lib.la_oracle_gla_backward(ptr(q), ptr(k), ptr(v), ptr(al), ptr(do), B, H, T,
                                              dk, dv, ptr(s0), ptr(dsf), ptr(dq), ptr(dk_), ptr(dv_),
                                              ptr(da), ptr(ds0), int(nthreads))
        if rc != 0:
            raise ValueError(f"la_oracle_gla_backward returned {rc}")
        return dq, dk_, dv_, da, ds0


_default: Oracle | None = None


def default_oracle() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
