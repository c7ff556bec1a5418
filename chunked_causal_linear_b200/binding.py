"""ctypes binding of ``liblinattn.so`` (include/linattn.h).

Argument marshalling only: every step of the computation runs in the CUDA library.
Tensors are torch CUDA tensors (PyTorch provides device memory and streams); the
functions keep the C entry points' names.  If the shared library is missing, every call
raises -- there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
from pathlib import Path

import torch

LIB_PATH = Path(__file__).resolve().parent / "liblinattn.so"

LA_OK = 0
STATUS_NAMES = {0: "LA_OK", 1: "LA_ERR_INVALID_ARGUMENT", 2: "LA_ERR_UNSUPPORTED",
                3: "LA_ERR_OUT_OF_MEMORY", 4: "LA_ERR_CUDA", 5: "LA_ERR_INTERNAL"}
FEATURE_MAPS = {"identity": 0, "elu1": 1}
SCAN_MODES = {"logdepth": 0, "sequential": 1}
KERNEL_PATHS = {"auto": 0, "tensor_core": 1, "fma": 2}
ALGORITHMS = {"auto": 0, "chunked": 1, "segmented": 2}
DTYPES = {torch.bfloat16: 0, torch.float32: 1}
OUT_DTYPES = {"as_input": 0, "f32": 1}

EXPORTED_SYMBOLS = (
    "lin_attn_prefill", "lin_attn_prefill_f32", "lin_attn_prefill_workspace_bytes",
    "lin_attn_prefill_ex", "lin_attn_prefill_timed", "lin_attn_prefill_host",
    "lin_attn_prefill_host_buffer_bytes", "lin_attn_prefill_noalloc",
    "lin_attn_decode_step", "lin_attn_decode_step_f32", "lin_attn_device_error",
    "lin_attn_status_string", "lin_attn_version", "lin_attn_combine_states",
    "lin_attn_backward", "lin_attn_backward_workspace_bytes", "lin_attn_backward_timed",
    "lin_attn_gla_prefill", "lin_attn_gla_workspace_bytes", "lin_attn_gla_prefill_timed",
    "lin_attn_scan_plan", "lin_attn_check_wait_timeout",
)


class LinAttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS_NAMES.get(status, status)}")
        self.status = status


class PrefillArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("S_final", ctypes.c_void_p), ("Z_final", ctypes.c_void_p),
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_longlong),
        ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("C", ctypes.c_int),
        ("feature_map", ctypes.c_int), ("gamma", ctypes.c_void_p), ("normalize", ctypes.c_int),
        ("eps", ctypes.c_float), ("dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
        ("scan_mode", ctypes.c_int),
        ("kernel_path", ctypes.c_int), ("algorithm", ctypes.c_int),
        ("segment_chunks", ctypes.c_int),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t), ("stream", ctypes.c_void_p),
        ("S_init", ctypes.c_void_p), ("Z_init", ctypes.c_void_p), ("states_only", ctypes.c_int),
        ("reverse", ctypes.c_int),
    ]


class BackwardArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("grad_out", ctypes.c_void_p), ("grad_q", ctypes.c_void_p), ("grad_k", ctypes.c_void_p),
        ("grad_v", ctypes.c_void_p), ("S_init", ctypes.c_void_p),
        ("grad_S_final", ctypes.c_void_p), ("grad_S_init", ctypes.c_void_p),
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_longlong),
        ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("C", ctypes.c_int),
        ("feature_map", ctypes.c_int), ("gamma", ctypes.c_void_p), ("dtype", ctypes.c_int),
        ("out_dtype", ctypes.c_int), ("scan_mode", ctypes.c_int), ("kernel_path", ctypes.c_int),
        ("algorithm", ctypes.c_int), ("segment_chunks", ctypes.c_int),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("stream", ctypes.c_void_p), ("normalize", ctypes.c_int), ("eps", ctypes.c_float),
        ("Z_init", ctypes.c_void_p), ("grad_Z_final", ctypes.c_void_p),
        ("grad_Z_init", ctypes.c_void_p),
    ]


class GlaArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("alpha", ctypes.c_void_p), ("out", ctypes.c_void_p), ("S_final", ctypes.c_void_p),
        ("S_init", ctypes.c_void_p), ("B", ctypes.c_int), ("H", ctypes.c_int),
        ("T", ctypes.c_longlong), ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("C", ctypes.c_int),
        ("dtype", ctypes.c_int), ("out_dtype", ctypes.c_int), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t), ("stream", ctypes.c_void_p),
        ("kernel_path", ctypes.c_int), ("segment_chunks", ctypes.c_int),
    ]


_lib = None


def load_library(path: Path | str | None = None) -> ctypes.CDLL:
    """Loads the CUDA library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = Path(path) if path is not None else LIB_PATH
    if not p.exists():
        raise RuntimeError(f"{p} is missing: build it with `python -m chunked_causal_linear_b200.build`")
    lib = ctypes.CDLL(str(p))
    vp, i, ll, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_size_t
    sig = {
        "lin_attn_prefill": (i, [vp, vp, vp, vp, vp, vp, i, i, ll, i, i, i, i, vp, i, vp]),
        "lin_attn_prefill_f32": (i, [vp, vp, vp, vp, vp, vp, i, i, ll, i, i, i, i, vp, i, vp]),
        "lin_attn_prefill_workspace_bytes": (sz, [i, i, ll, i, i, i, i]),
        "lin_attn_prefill_ex": (i, [ctypes.POINTER(PrefillArgs)]),
        "lin_attn_prefill_timed": (i, [ctypes.POINTER(PrefillArgs), ctypes.POINTER(f), i,
                                       ctypes.POINTER(i)]),
        "lin_attn_prefill_host": (i, [ctypes.POINTER(PrefillArgs), vp, sz]),
        "lin_attn_prefill_noalloc": (i, [ctypes.POINTER(PrefillArgs)]),
        "lin_attn_prefill_host_buffer_bytes": (sz, [ctypes.POINTER(PrefillArgs)]),
        "lin_attn_decode_step": (i, [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, i, vp]),
        "lin_attn_decode_step_f32": (i, [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, i, vp]),
        "lin_attn_device_error": (i, [ctypes.POINTER(ctypes.c_int)]),
        "lin_attn_status_string": (ctypes.c_char_p, [i]),
        "lin_attn_version": (i, []),
        "lin_attn_check_wait_timeout": (i, [ctypes.c_uint, vp]),
        "lin_attn_scan_plan": (i, [ll, i, ctypes.POINTER(i), ctypes.POINTER(i), ctypes.POINTER(i),
                                   ctypes.POINTER(i), ctypes.POINTER(ll)]),
        "lin_attn_combine_states": (i, [vp, vp, i, i, ctypes.POINTER(ll), i, i, i, i, vp, vp,
                                        vp, vp]),
        "lin_attn_backward": (i, [ctypes.POINTER(BackwardArgs)]),
        "lin_attn_backward_workspace_bytes": (sz, [ctypes.POINTER(BackwardArgs)]),
        "lin_attn_backward_timed": (i, [ctypes.POINTER(BackwardArgs), ctypes.POINTER(f),
                                        ctypes.POINTER(ctypes.c_char_p), i, ctypes.POINTER(i)]),
        "lin_attn_gla_prefill": (i, [ctypes.POINTER(GlaArgs)]),
        "lin_attn_gla_workspace_bytes": (sz, [i, i, ll, i, i, i]),
        "lin_attn_gla_prefill_timed": (i, [ctypes.POINTER(GlaArgs), ctypes.POINTER(f), i,
                                           ctypes.POINTER(i)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def _check(fn: str, status: int) -> None:
    if status != LA_OK:
        raise LinAttnError(fn, status)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _gamma_array(gamma, H):
    if gamma is None:
        return None, None
    vals = [float(g) for g in gamma]
    if len(vals) != H:
        raise ValueError(f"gamma needs {H} values, got {len(vals)}")
    arr = (ctypes.c_float * H)(*vals)
    return arr, ctypes.cast(arr, ctypes.c_void_p)


def make_args(q, k, v, out, S_final, Z_final, *, chunk, feature_map, gamma, normalize, eps,
              scan, kernel_path, workspace, stream, out_dtype="as_input", algorithm="auto",
              segment_chunks=0, S_init=None, Z_init=None, states_only=False, reverse=False):
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    garr, gptr = _gamma_array(gamma, H)
    a = PrefillArgs()
    a.q, a.k, a.v, a.out = _ptr(q), _ptr(k), _ptr(v), _ptr(out)
    a.S_final, a.Z_final = _ptr(S_final), _ptr(Z_final)
    a.B, a.H, a.T, a.dk, a.dv, a.C = B, H, T, dk, dv, int(chunk)
    a.feature_map = FEATURE_MAPS[feature_map]
    a.gamma = gptr
    a.normalize = int(bool(normalize))
    a.eps = float(eps)
    a.dtype = DTYPES[q.dtype]
    a.out_dtype = OUT_DTYPES[out_dtype]
    a.scan_mode = SCAN_MODES[scan]
    a.kernel_path = KERNEL_PATHS[kernel_path]
    a.algorithm = ALGORITHMS[algorithm]
    a.segment_chunks = int(segment_chunks)
    a.workspace = _ptr(workspace)
    a.workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    a.stream = stream
    a.S_init, a.Z_init = _ptr(S_init), _ptr(Z_init)
    a.states_only = int(bool(states_only))
    a.reverse = int(bool(reverse))
    return a, garr


def lin_attn_prefill_workspace_bytes(B, H, T, dk, dv, C, normalize) -> int:
    return int(load_library().lin_attn_prefill_workspace_bytes(B, H, T, dk, dv, C, int(bool(normalize))))


def lin_attn_prefill(q, k, v, out=None, S_final=None, Z_final=None, *, chunk=64,
                     feature_map="elu1", gamma=None, normalize=True, eps=0.0, scan="logdepth",
                     kernel_path="auto", workspace=None, stream=None, want_states=True,
                     out_dtype="as_input", algorithm="auto", segment_chunks=0, S_init=None,
                     Z_init=None, states_only=False, reverse=False):
    """Runs the prefill on device tensors q, k [B,H,T,dk], v [B,H,T,dv] (bf16 or float32).

    out_dtype "f32" writes a float32 output for bf16 inputs.  Allocates out / S_final /
    Z_final when not given.  S_init / Z_init: the state before token 0 (device float32,
    may be S_final / Z_final themselves).  states_only: compute the final states only (no
    output; out stays None).  reverse: the anti-causal direction (token T-1 first;
    segmented algorithm only).  Returns (out, S_final, Z_final).
    """
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if out is None and not states_only:
        odt = torch.float32 if out_dtype == "f32" else q.dtype
        out = torch.empty((B, H, T, dv), dtype=odt, device=q.device)
    if want_states and S_final is None:
        S_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    if want_states and normalize and Z_final is None:
        Z_final = torch.empty((B, H, dk), dtype=torch.float32, device=q.device)
    a, keep = make_args(q, k, v, out, S_final, Z_final, chunk=chunk, feature_map=feature_map,
                        gamma=gamma, normalize=normalize, eps=eps, scan=scan,
                        kernel_path=kernel_path, workspace=workspace,
                        stream=_stream_handle(stream), out_dtype=out_dtype, algorithm=algorithm,
                        segment_chunks=segment_chunks, S_init=S_init, Z_init=Z_init,
                        states_only=states_only, reverse=reverse)
    _check("lin_attn_prefill_ex", load_library().lin_attn_prefill_ex(ctypes.byref(a)))
    del keep
    return out, S_final, Z_final


def lin_attn_combine_states(S_parts, Z_parts, upto, part_tokens, *, gamma=None, S_out=None,
                            Z_out=None, stream=None):
    """Incoming state of part `upto` of a sequence split into parts (see the header):
    S_parts [parts,B,H,dk,dv], Z_parts [parts,B,H,dk] or None, part_tokens a list of
    ints.  Returns (S_out, Z_out)."""
    parts, B, H, dk, dv = S_parts.shape
    if S_out is None:
        S_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=S_parts.device)
    if Z_parts is not None and Z_out is None:
        Z_out = torch.empty((B, H, dk), dtype=torch.float32, device=S_parts.device)
    toks = (ctypes.c_longlong * max(1, parts))(*[int(t) for t in part_tokens])
    garr, gptr = _gamma_array(gamma, H)
    _check("lin_attn_combine_states",
           load_library().lin_attn_combine_states(_ptr(S_parts), _ptr(Z_parts), parts, int(upto),
                                                  toks, B, H, dk, dv, gptr, _ptr(S_out),
                                                  _ptr(Z_out), _stream_handle(stream)))
    del garr
    return S_out, Z_out


def lin_attn_prefill_timed(q, k, v, out, S_final=None, Z_final=None, *, chunk=64,
                           feature_map="elu1", gamma=None, normalize=True, eps=0.0,
                           scan="logdepth", kernel_path="auto", workspace=None, stream=None,
                           out_dtype="as_input", algorithm="auto", segment_chunks=0) -> list[float]:
    """Runs the prefill once with an event around every kernel; returns the kernels'
    device durations in milliseconds, in launch order (synchronous)."""
    a, keep = make_args(q, k, v, out, S_final, Z_final, chunk=chunk, feature_map=feature_map,
                        gamma=gamma, normalize=normalize, eps=eps, scan=scan,
                        kernel_path=kernel_path, workspace=workspace,
                        stream=_stream_handle(stream), out_dtype=out_dtype, algorithm=algorithm,
                        segment_chunks=segment_chunks)
    ms = (ctypes.c_float * 8)()
    n = ctypes.c_int(0)
    _check("lin_attn_prefill_timed",
           load_library().lin_attn_prefill_timed(ctypes.byref(a), ms, 8, ctypes.byref(n)))
    del keep
    return [float(ms[i]) for i in range(n.value)]


def lin_attn_prefill_host(q, k, v, out, S_final=None, Z_final=None, *, chunk=64,
                          feature_map="elu1", gamma=None, normalize=True, eps=0.0,
                          scan="logdepth", kernel_path="auto", device_buffer=None, stream=None,
                          out_dtype="as_input", algorithm="auto", segment_chunks=0, S_init=None,
                          Z_init=None, states_only=False):
    """Runs the prefill on HOST tensors (pinned for full copy bandwidth); synchronous.
    S_init / Z_init, when given, are host tensors too."""
    a, keep = make_args(q, k, v, out, S_final, Z_final, chunk=chunk, feature_map=feature_map,
                        gamma=gamma, normalize=normalize, eps=eps, scan=scan,
                        kernel_path=kernel_path, workspace=None, stream=_stream_handle(stream),
                        out_dtype=out_dtype, algorithm=algorithm,
                        segment_chunks=segment_chunks, S_init=S_init, Z_init=Z_init,
                        states_only=states_only)
    nbytes = 0 if device_buffer is None else device_buffer.numel() * device_buffer.element_size()
    _check("lin_attn_prefill_host",
           load_library().lin_attn_prefill_host(ctypes.byref(a), _ptr(device_buffer), nbytes))
    del keep
    return out, S_final, Z_final


def make_backward_args(q, k, v, grad_out, grad_q, grad_k, grad_v, *, S_init=None,
                       grad_S_final=None, grad_S_init=None, chunk=64, feature_map="identity",
                       gamma=None, out_dtype="as_input", scan="logdepth", kernel_path="auto",
                       algorithm="auto", segment_chunks=0, workspace=None, stream=None,
                       normalize=False, eps=0.0, Z_init=None, grad_Z_final=None,
                       grad_Z_init=None):
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    garr, gptr = _gamma_array(gamma, H)
    a = BackwardArgs()
    a.q, a.k, a.v, a.grad_out = _ptr(q), _ptr(k), _ptr(v), _ptr(grad_out)
    a.grad_q, a.grad_k, a.grad_v = _ptr(grad_q), _ptr(grad_k), _ptr(grad_v)
    a.S_init, a.grad_S_final, a.grad_S_init = _ptr(S_init), _ptr(grad_S_final), _ptr(grad_S_init)
    a.B, a.H, a.T, a.dk, a.dv, a.C = B, H, T, dk, dv, int(chunk)
    a.feature_map = FEATURE_MAPS[feature_map]
    a.gamma = gptr
    a.dtype = DTYPES[q.dtype]
    a.out_dtype = OUT_DTYPES[out_dtype]
    a.scan_mode = SCAN_MODES[scan]
    a.kernel_path = KERNEL_PATHS[kernel_path]
    a.algorithm = ALGORITHMS[algorithm]
    a.segment_chunks = int(segment_chunks)
    a.workspace = _ptr(workspace)
    a.workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    a.stream = stream
    a.normalize = int(bool(normalize))
    a.eps = float(eps)
    a.Z_init, a.grad_Z_final, a.grad_Z_init = _ptr(Z_init), _ptr(grad_Z_final), _ptr(grad_Z_init)
    return a, garr


def lin_attn_backward(q, k, v, grad_out, grad_q=None, grad_k=None, grad_v=None, *,
                      S_init=None, grad_S_final=None, want_grad_S_init=False, grad_S_init=None,
                      chunk=64, feature_map="identity", gamma=None, out_dtype="as_input",
                      scan="logdepth", kernel_path="auto", algorithm="auto", segment_chunks=0,
                      workspace=None, stream=None, normalize=False, eps=0.0, Z_init=None,
                      grad_Z_final=None, want_grad_Z_init=False, grad_Z_init=None):
    """Gradients for the loss <grad_out, out> + <grad_S_final, S_final> (+ <grad_Z_final,
    Z_final> normalised; see the header).  q, k [B,H,T,dk], v, grad_out [B,H,T,dv] on the
    device.  Allocates the gradients not given.  Returns (grad_q, grad_k, grad_v, grad_S_init), plus grad_Z_init
    when normalising; the state gradients are None unless requested."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    odt = torch.float32 if out_dtype == "f32" else q.dtype
    mk = lambda d: torch.empty((B, H, T, d), dtype=odt, device=q.device)
    grad_q = mk(dk) if grad_q is None else grad_q
    grad_k = mk(dk) if grad_k is None else grad_k
    grad_v = mk(dv) if grad_v is None else grad_v
    if grad_S_init is None and want_grad_S_init:
        grad_S_init = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    if grad_Z_init is None and want_grad_Z_init:
        grad_Z_init = torch.empty((B, H, dk), dtype=torch.float32, device=q.device)
    a, keep = make_backward_args(q, k, v, grad_out, grad_q, grad_k, grad_v, S_init=S_init,
                                 grad_S_final=grad_S_final, grad_S_init=grad_S_init, chunk=chunk,
                                 feature_map=feature_map, gamma=gamma, out_dtype=out_dtype,
                                 scan=scan, kernel_path=kernel_path, algorithm=algorithm,
                                 segment_chunks=segment_chunks, workspace=workspace,
                                 stream=_stream_handle(stream), normalize=normalize, eps=eps,
                                 Z_init=Z_init, grad_Z_final=grad_Z_final,
                                 grad_Z_init=grad_Z_init)
    _check("lin_attn_backward", load_library().lin_attn_backward(ctypes.byref(a)))
    del keep
    if normalize:
        return grad_q, grad_k, grad_v, grad_S_init, grad_Z_init
    return grad_q, grad_k, grad_v, grad_S_init


def lin_attn_backward_timed(q, k, v, grad_out, grad_q, grad_k, grad_v, *, S_init=None,
                            grad_S_final=None, grad_S_init=None, chunk=64, feature_map="identity",
                            gamma=None, out_dtype="as_input", scan="logdepth", kernel_path="auto",
                            algorithm="auto", segment_chunks=0, workspace=None,
                            stream=None, normalize=False,
                            eps=0.0) -> list[tuple[str, float]]:
    """Runs the backward once with an event around every kernel; returns (name,
    milliseconds) per kernel in launch order (synchronous)."""
    a, keep = make_backward_args(q, k, v, grad_out, grad_q, grad_k, grad_v, S_init=S_init,
                                 grad_S_final=grad_S_final, grad_S_init=grad_S_init, chunk=chunk,
                                 feature_map=feature_map, gamma=gamma, out_dtype=out_dtype,
                                 scan=scan, kernel_path=kernel_path, algorithm=algorithm,
                                 segment_chunks=segment_chunks, workspace=workspace,
                                 stream=_stream_handle(stream), normalize=normalize, eps=eps)
    cap = 48
    ms = (ctypes.c_float * cap)()
    names = (ctypes.c_char_p * cap)()
    n = ctypes.c_int(0)
    _check("lin_attn_backward_timed",
           load_library().lin_attn_backward_timed(ctypes.byref(a), ms, names, cap,
                                                  ctypes.byref(n)))
    del keep
    return [(names[i].decode(), float(ms[i])) for i in range(n.value)]


def lin_attn_backward_workspace_bytes(q, v, *, chunk=64, feature_map="identity",
                                      out_dtype="as_input", S_init=False, grad_S_final=False,
                                      gamma=None, normalize=False, algorithm="auto") -> int:
    """Workspace bytes of lin_attn_backward for these shapes and options (S_init /
    grad_S_final: whether they will be given)."""
    B, H, T, dk = q.shape
    garr, gptr = _gamma_array(gamma, H)
    a = BackwardArgs()
    a.B, a.H, a.T, a.dk, a.dv, a.C = B, H, T, dk, v.shape[-1], int(chunk)
    a.feature_map = FEATURE_MAPS[feature_map]
    a.gamma = gptr
    a.dtype = DTYPES[q.dtype]
    a.out_dtype = OUT_DTYPES[out_dtype]
    a.normalize = int(bool(normalize))
    a.algorithm = ALGORITHMS[algorithm]
    # Only whether the states are given matters to the size; any non-null value says so.
    a.S_init = 16 if S_init else None
    a.grad_S_final = 16 if grad_S_final else None
    n = int(load_library().lin_attn_backward_workspace_bytes(ctypes.byref(a)))
    del garr
    return n


def _gla_args(q, k, v, alpha, out, S_final, S_init, chunk, out_dtype, workspace, stream,
              kernel_path="auto", segment_chunks=0):
    B, H, T, dk = q.shape
    a = GlaArgs()
    a.q, a.k, a.v, a.alpha, a.out = _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(out)
    a.S_final, a.S_init = _ptr(S_final), _ptr(S_init)
    a.B, a.H, a.T, a.dk, a.dv, a.C = B, H, T, dk, v.shape[-1], int(chunk)
    a.dtype = DTYPES[q.dtype]
    a.out_dtype = OUT_DTYPES[out_dtype]
    a.workspace = _ptr(workspace)
    a.workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    a.stream = _stream_handle(stream)
    a.kernel_path = KERNEL_PATHS[kernel_path]
    a.segment_chunks = int(segment_chunks)
    return a


def lin_attn_gla_prefill(q, k, v, alpha, out=None, S_final=None, *, S_init=None, chunk=64,
                         out_dtype="as_input", workspace=None, stream=None, want_state=True,
                         kernel_path="auto", segment_chunks=0):
    """Gated linear attention (see the header): q, k, alpha [B,H,T,dk] (alpha float32),
    v [B,H,T,dv].  Returns (out, S_final)."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        odt = torch.float32 if out_dtype == "f32" else q.dtype
        out = torch.empty((B, H, T, dv), dtype=odt, device=q.device)
    if want_state and S_final is None:
        S_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    a = _gla_args(q, k, v, alpha, out, S_final, S_init, chunk, out_dtype, workspace, stream,
                  kernel_path, segment_chunks)
    _check("lin_attn_gla_prefill", load_library().lin_attn_gla_prefill(ctypes.byref(a)))
    return out, S_final


def lin_attn_gla_workspace_bytes(B, H, T, dk, dv, C) -> int:
    return int(load_library().lin_attn_gla_workspace_bytes(B, H, T, dk, dv, C))


def lin_attn_gla_prefill_timed(q, k, v, alpha, out, S_final=None, *, S_init=None, chunk=64,
                               out_dtype="as_input", workspace=None, stream=None,
                               kernel_path="auto", segment_chunks=0) -> list[float]:
    """One GLA prefill with an event around each kernel; returns their durations in ms, in
    launch order (CUDA cores: K1, K2, K3; tensor cores: gla_k1_seg, gla_scan, gla_k3_seg,
    gla_fixup)."""
    a = _gla_args(q, k, v, alpha, out, S_final, S_init, chunk, out_dtype, workspace, stream,
                  kernel_path, segment_chunks)
    ms = (ctypes.c_float * 8)()
    n = ctypes.c_int(0)
    _check("lin_attn_gla_prefill_timed",
           load_library().lin_attn_gla_prefill_timed(ctypes.byref(a), ms, 8, ctypes.byref(n)))
    return [float(ms[i]) for i in range(n.value)]


NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


def lin_attn_prefill_noalloc(q, k, v, out, S_final=None, Z_final=None, *, chunk=64,
                             feature_map="elu1", gamma=None, normalize=True, eps=0.0,
                             scan="logdepth", kernel_path="auto", stream=None,
                             out_dtype="as_input", algorithm="auto", segment_chunks=0):
    """The prefill with its workspace in the library's fixed device array (no device
    allocation by the library; the caller provides every output tensor)."""
    a, keep = make_args(q, k, v, out, S_final, Z_final, chunk=chunk, feature_map=feature_map,
                        gamma=gamma, normalize=normalize, eps=eps, scan=scan,
                        kernel_path=kernel_path, workspace=None, stream=_stream_handle(stream),
                        out_dtype=out_dtype, algorithm=algorithm,
                        segment_chunks=segment_chunks)
    _check("lin_attn_prefill_noalloc", load_library().lin_attn_prefill_noalloc(ctypes.byref(a)))
    del keep
    return out, S_final, Z_final


def lin_attn_prefill_host_buffer_bytes(q, v, *, chunk=64, normalize=True,
                                       out_dtype="as_input") -> int:
    B, H, T, dk = q.shape
    a = PrefillArgs()
    a.B, a.H, a.T, a.dk, a.dv, a.C = B, H, T, dk, v.shape[-1], int(chunk)
    a.normalize = int(bool(normalize))
    a.dtype = DTYPES[q.dtype]
    a.out_dtype = OUT_DTYPES[out_dtype]
    return int(load_library().lin_attn_prefill_host_buffer_bytes(ctypes.byref(a)))


def lin_attn_decode_step(q, k, v, S, Z=None, out=None, *, feature_map="elu1", gamma=None,
                         normalize=True, stream=None):
    """One decode step: q, k [B,H,dk], v [B,H,dv]; S [B,H,dk,dv] and Z [B,H,dk] updated in place."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    garr, gptr = _gamma_array(gamma, H)
    lib = load_library()
    fn = lib.lin_attn_decode_step_f32 if q.dtype == torch.float32 else lib.lin_attn_decode_step
    _check("lin_attn_decode_step",
           fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(S), _ptr(Z), B, H, dk, dv,
              FEATURE_MAPS[feature_map], gptr, int(bool(normalize)), _stream_handle(stream)))
    del garr
    return out


def lin_attn_device_error() -> int:
    code = ctypes.c_int(0)
    _check("lin_attn_device_error", load_library().lin_attn_device_error(ctypes.byref(code)))
    return code.value


def lin_attn_status_string(status: int) -> str:
    return load_library().lin_attn_status_string(int(status)).decode()


def lin_attn_check_wait_timeout(timeout_us: int = 1000, stream=None) -> None:
    """Launches the library's bounded-wait check (one wait that must give up); read the
    result with lin_attn_device_error() (code 5)."""
    _check("lin_attn_check_wait_timeout",
           load_library().lin_attn_check_wait_timeout(int(timeout_us), _stream_handle(stream)))


def lin_attn_scan_plan(n: int, scan: str = "logdepth") -> dict:
    """K2's shape for a scan over n elements: segment length and count, blocked-scan groups
    and elements per group, and the dependent-step depth."""
    vals = [ctypes.c_int(0) for _ in range(4)]
    depth = ctypes.c_longlong(0)
    _check("lin_attn_scan_plan",
           load_library().lin_attn_scan_plan(int(n), SCAN_MODES[scan],
                                             *(ctypes.byref(x) for x in vals),
                                             ctypes.byref(depth)))
    return {"segment_len": vals[0].value, "segments": vals[1].value, "groups": vals[2].value,
            "per_group": vals[3].value, "depth": depth.value}


def lin_attn_version() -> int:
    return int(load_library().lin_attn_version())
