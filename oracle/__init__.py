"""Python access to the fp64 CPU oracle (``oracle/fa_oracle.c``).

Test infrastructure only: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg use it.  The CUDA library never imports it.

Arrays are ``[B, H, N, d]`` row-major.  Inputs may be bf16 bit patterns
(``numpy.uint16``, or a ``torch.bfloat16`` tensor on the CPU) or ``float64``;
outputs are always ``float64``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fa_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "libfa_oracle.so")

_lock = threading.Lock()
_lib = None

BF16 = 0
F64 = 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math) and return the .so path."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", "-Wall", "-o", tmp, _SRC, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def build_variant(src: str, out_path: str) -> str:
    """Compile another copy of the oracle source (used by tests that plant a
    mistake in a copy and check that the pins catch it)."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", "-o", out_path, src, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    return out_path


def _load(path: str) -> ctypes.CDLL:
    L = ctypes.CDLL(path)
    i64, dbl, vp, ip = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
    L.oracle_fwd.argtypes = [vp, vp, vp, ip, i64, i64, i64, i64, i64, i64, dbl, ip,
                             vp, i64, vp, vp, ip]
    L.oracle_fwd.restype = ip
    L.oracle_bwd.argtypes = [vp, vp, vp, vp, ip, i64, i64, i64, i64, i64, i64, dbl, ip,
                             vp, vp, vp, ip]
    L.oracle_bwd.restype = ip
    L.oracle_bwd_dq_rows.argtypes = [vp, vp, vp, vp, ip, i64, i64, i64, i64, i64, i64,
                                     dbl, ip, vp, i64, vp, ip]
    L.oracle_bwd_dq_rows.restype = ip
    L.oracle_bwd_dkv_rows.argtypes = [vp, vp, vp, vp, ip, i64, i64, i64, i64, i64, i64,
                                      dbl, ip, vp, i64, vp, vp, ip]
    L.oracle_bwd_dkv_rows.restype = ip
    for name in ("oracle_online_row_f64", "oracle_online_row_f32"):
        fn = getattr(L, name)
        fn.argtypes = [vp, vp, i64, i64, i64, vp, vp, vp, vp]
        fn.restype = i64
    L.oracle_full_row_f32.argtypes = [vp, vp, i64, i64, vp, vp, vp]
    L.oracle_full_row_f32.restype = None
    L.oracle_lse_merge.argtypes = [vp, vp, i64, i64, vp, vp]
    L.oracle_lse_merge.restype = None
    L.oracle_e4m3_to_f64.argtypes = [vp, i64, vp]
    L.oracle_e4m3_to_f64.restype = None
    return L


_active = threading.local()


def lib() -> ctypes.CDLL:
    """The oracle library in use: the built one, or a variant selected with
    ``using(path)`` on this thread."""
    global _lib
    v = getattr(_active, "lib", None)
    if v is not None:
        return v
    with _lock:
        if _lib is None:
            _lib = _load(build())
        return _lib


class using:
    """Context manager: route this thread's oracle calls to another build."""

    def __init__(self, path: str):
        self._lib = _load(path)

    def __enter__(self):
        self._prev = getattr(_active, "lib", None)
        _active.lib = self._lib
        return self

    def __exit__(self, *exc):
        _active.lib = self._prev
        return False


def _as_input(x):
    """Return (contiguous numpy array, dtype code) for a bf16 or float64 input."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach()
            if x.device.type != "cpu":
                raise ValueError("oracle inputs must live on the CPU")
            if x.dtype == torch.bfloat16:
                return np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16)), BF16
            x = x.to(torch.float64).numpy()
    except ImportError:  # pragma: no cover - torch is always present here
        pass
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), BF16
    return np.ascontiguousarray(x, dtype=np.float64), F64


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dims(q, k):
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if Bk != B or dk != d:
        raise ValueError("q and k shapes disagree")
    return B, Hq, Hkv, Nq, Nk, d


def fwd(q, k, v, scale, causal, rows=None, nthreads=0):
    """Forward.  Returns (o, lse): o [B,Hq,Nq,d] (or [len(rows), d]), lse likewise.

    ``rows`` lists flattened query rows ``(b * Hq + h) * Nq + i`` to compute
    one by one; ``None`` computes every row."""
    qa, dt = _as_input(q)
    ka, dt2 = _as_input(k)
    va, dt3 = _as_input(v)
    if not (dt == dt2 == dt3):
        raise ValueError("q, k, v must share one dtype")
    B, Hq, Hkv, Nq, Nk, d = _dims(qa, ka)
    if rows is None:
        o = np.empty((B, Hq, Nq, d), np.float64)
        lse = np.empty((B, Hq, Nq), np.float64)
        rp, nr = None, 0
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        o = np.empty((rows.size, d), np.float64)
        lse = np.empty((rows.size,), np.float64)
        rp, nr = _ptr(rows), rows.size
    rc = lib().oracle_fwd(_ptr(qa), _ptr(ka), _ptr(va), dt, B, Hq, Hkv, Nq, Nk, d,
                          float(scale), int(bool(causal)), rp, nr, _ptr(o), _ptr(lse),
                          int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_fwd failed ({rc})")
    return o, lse


def bwd(q, k, v, dout, scale, causal, nthreads=0):
    """Full backward of L = sum(dout * O).  Returns (dq, dk, dv) in float64."""
    qa, dt = _as_input(q)
    ka, _ = _as_input(k)
    va, _ = _as_input(v)
    da, _ = _as_input(dout)
    B, Hq, Hkv, Nq, Nk, d = _dims(qa, ka)
    dq = np.empty((B, Hq, Nq, d), np.float64)
    dk = np.empty((B, Hkv, Nk, d), np.float64)
    dv = np.empty((B, Hkv, Nk, d), np.float64)
    rc = lib().oracle_bwd(_ptr(qa), _ptr(ka), _ptr(va), _ptr(da), dt, B, Hq, Hkv, Nq, Nk, d,
                          float(scale), int(bool(causal)), _ptr(dq), _ptr(dk), _ptr(dv),
                          int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_bwd failed ({rc})")
    return dq, dk, dv


def bwd_dq_rows(q, k, v, dout, scale, causal, rows, nthreads=0):
    """dQ for the listed flattened query rows only.  Returns [len(rows), d]."""
    qa, dt = _as_input(q)
    ka, _ = _as_input(k)
    va, _ = _as_input(v)
    da, _ = _as_input(dout)
    B, Hq, Hkv, Nq, Nk, d = _dims(qa, ka)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    dq = np.empty((rows.size, d), np.float64)
    rc = lib().oracle_bwd_dq_rows(_ptr(qa), _ptr(ka), _ptr(va), _ptr(da), dt, B, Hq, Hkv, Nq,
                                  Nk, d, float(scale), int(bool(causal)), _ptr(rows), rows.size,
                                  _ptr(dq), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_bwd_dq_rows failed ({rc})")
    return dq


def bwd_dkv_rows(q, k, v, dout, scale, causal, keys, nthreads=0):
    """dK and dV for the listed flattened key rows ``(b * Hkv + g) * Nk + j``."""
    qa, dt = _as_input(q)
    ka, _ = _as_input(k)
    va, _ = _as_input(v)
    da, _ = _as_input(dout)
    B, Hq, Hkv, Nq, Nk, d = _dims(qa, ka)
    keys = np.ascontiguousarray(keys, dtype=np.int64)
    dk = np.empty((keys.size, d), np.float64)
    dv = np.empty((keys.size, d), np.float64)
    rc = lib().oracle_bwd_dkv_rows(_ptr(qa), _ptr(ka), _ptr(va), _ptr(da), dt, B, Hq, Hkv, Nq,
                                   Nk, d, float(scale), int(bool(causal)), _ptr(keys), keys.size,
                                   _ptr(dk), _ptr(dv), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_bwd_dkv_rows failed ({rc})")
    return dk, dv


def online_row(s, v, block, precision="f64", trace=False):
    """Blocked online softmax over one row of scores ``s`` [n] with values
    ``v`` [n, dv] (or [n]).  Returns (o [dv], m, l) and, with ``trace``, a list of
    per-block dicts {m, l_rescaled, U_rescaled, l, U}."""
    s = np.ascontiguousarray(s, dtype=np.float64).reshape(-1)
    v = np.ascontiguousarray(v, dtype=np.float64)
    n = s.size
    dv = 1 if v.ndim == 1 else v.shape[1]
    v = v.reshape(n, dv)
    nb = (n + block - 1) // block
    o = np.empty(dv, np.float64)
    m = ctypes.c_double()
    l_ = ctypes.c_double()
    tr = np.empty(max(nb, 1) * (3 + 2 * dv), np.float64) if trace else None
    fn = lib().oracle_online_row_f64 if precision == "f64" else lib().oracle_online_row_f32
    fn(_ptr(s), _ptr(v), n, dv, int(block), _ptr(o), ctypes.byref(m), ctypes.byref(l_),
       _ptr(tr) if trace else None)
    if not trace:
        return o, m.value, l_.value
    recs = []
    for b in range(nb):
        r = tr[b * (3 + 2 * dv):(b + 1) * (3 + 2 * dv)]
        recs.append(dict(m=r[0], l_rescaled=r[1], U_rescaled=r[2:2 + dv].copy(),
                         l=r[2 + dv], U=r[3 + dv:3 + 2 * dv].copy()))
    return o, m.value, l_.value, recs


def full_row_f32(s, v):
    """Whole-row softmax-weighted sum in fp32.  Returns (o [dv], m, l)."""
    s = np.ascontiguousarray(s, dtype=np.float64).reshape(-1)
    v = np.ascontiguousarray(v, dtype=np.float64)
    n = s.size
    dv = 1 if v.ndim == 1 else v.shape[1]
    v = v.reshape(n, dv)
    o = np.empty(dv, np.float64)
    m = ctypes.c_double()
    l_ = ctypes.c_double()
    lib().oracle_full_row_f32(_ptr(s), _ptr(v), n, dv, _ptr(o), ctypes.byref(m), ctypes.byref(l_))
    return o, m.value, l_.value


def lse_merge(o_parts, lse_parts):
    """Merge partial (O_s, lse_s) over disjoint key ranges.  Returns (o, lse)."""
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
    lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float64).reshape(-1)
    nparts = lse_parts.size
    d = o_parts.size // max(nparts, 1)
    o = np.empty(d, np.float64)
    lse = ctypes.c_double()
    lib().oracle_lse_merge(_ptr(o_parts), _ptr(lse_parts), nparts, d, _ptr(o), ctypes.byref(lse))
    return o, lse.value


def e4m3_to_f64(codes) -> np.ndarray:
    """Values of e4m3 bytes (OCP FP8 E4M3, no infinities; 0x7F / 0xFF are NaN),
    same shape as ``codes`` (uint8 array or tensor)."""
    if hasattr(codes, "numpy"):
        codes = codes.contiguous().view(dtype=__import__("torch").uint8).numpy()
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().oracle_e4m3_to_f64(_ptr(c), c.size, _ptr(out))
    return out
