"""Seeded synthetic workloads for exact attention.

This module only draws inputs: iid N(0,1) samples rounded to bf16 (or, on
request, fp16) from a counter-based SplitMix64 stream (see ``synth.c``), in the
shapes of the synthetic workloads below.  It contains no attention arithmetic and is shared
by the tests, the benchmark, the smoke check and the oracle checks, so both
sides of every comparison see identical input bits.

Tensor ids of the per-tensor streams: Q = 1, K = 2, V = 3, dO = 4.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "libsynth.so")
_lock = threading.Lock()
_lib = None

TENSOR_Q, TENSOR_K, TENSOR_V, TENSOR_DO = 1, 2, 3, 4


def build(force: bool = False) -> str:
    os.makedirs(_OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                    "-ffp-contract=off", "-Wall", "-o", tmp, _SRC, "-lm", "-lpthread"],
                   check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _get():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            u64, i64, vp, ip = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
            L.synth_splitmix64_at.argtypes = [u64, u64]
            L.synth_splitmix64_at.restype = u64
            L.synth_normal_bf16.argtypes = [u64, u64, vp, i64, ip]
            L.synth_normal_bf16.restype = None
            L.synth_normal_f32.argtypes = [u64, u64, vp, i64, ip]
            L.synth_normal_f32.restype = None
            _lib = L
        return _lib


def splitmix64_at(state0: int, n: int) -> int:
    """n-th output of the SplitMix64 stream starting at ``state0``."""
    return int(_get().synth_splitmix64_at(state0 & (2**64 - 1), n))


def normal_bf16_bits(seed: int, tensor_id: int, n: int, nthreads: int = 0, out=None) -> np.ndarray:
    """n bf16 bit patterns (uint16) of N(0,1) samples.  ``out`` may be a
    preallocated contiguous uint16 array (e.g. a view of pinned memory)."""
    if out is None:
        out = np.empty(n, np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == n
    _get().synth_normal_bf16(seed, tensor_id, out.ctypes.data_as(ctypes.c_void_p), n, nthreads)
    return out


def normal_f32(seed: int, tensor_id: int, n: int, nthreads: int = 0) -> np.ndarray:
    out = np.empty(n, np.float32)
    _get().synth_normal_f32(seed, tensor_id, out.ctypes.data_as(ctypes.c_void_p), n, nthreads)
    return out


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic attention problem: shapes, masking and the input recipe."""
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    seed: int
    scaled_q_rows: bool = False  # every 64th query row of each head x8
    backward: bool = True

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def fwd_flops(self) -> float:
        """4 * B * Hq * Nq * Nk * d, halved when causal (the reporting rule)."""
        f = 4.0 * self.B * self.Hq * self.Nq * self.Nk * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        return 2.5 * self.fwd_flops()


WORKLOADS = {
    "tiny_mha": Workload("tiny_mha", 1, 1, 1, 128, 128, 64, False, 1001),
    "mha_1k": Workload("mha_1k", 4, 16, 16, 1024, 1024, 64, True, 1002),
    "mha_1k_noncausal": Workload("mha_1k_noncausal", 4, 16, 16, 1024, 1024, 64, False, 1002),
    "mha_4k_long": Workload("mha_4k_long", 2, 32, 32, 4096, 4096, 128, True, 1003,
                            scaled_q_rows=True),
    "gqa_8k": Workload("gqa_8k", 1, 32, 8, 8192, 8192, 128, True, 1004),
    "gqa_decode": Workload("gqa_decode", 64, 32, 8, 1, 8192, 128, False, 1005, backward=False),
}


def make_inputs(w: Workload, nthreads: int = 0, pinned: bool = False, dout: bool = True,
                dtype=None):
    """Return dict(q, k, v[, dout]) of CPU 16-bit tensors for ``w``: bf16 by
    default, or fp16 with ``dtype=torch.float16`` (the same fp32 samples rounded
    to nearest even in the other format).

    Shapes: q/dout [B, Hq, Nq, d], k/v [B, Hkv, Nk, d].  With
    ``w.scaled_q_rows`` query rows i % 64 == 0 of every head are multiplied by 8
    (exact in either format)."""
    import torch
    dtype = torch.bfloat16 if dtype is None else dtype

    def draw(tid, shape):
        n = int(np.prod(shape))
        if dtype == torch.float16:
            f = normal_f32(w.seed, tid, n, nthreads).astype(np.float16)   # IEEE round to nearest even
            t = torch.from_numpy(f).reshape(shape)
            return t.pin_memory() if pinned else t
        t = torch.empty(shape, dtype=torch.bfloat16, pin_memory=pinned)
        bits = t.view(torch.int16).numpy().view(np.uint16).reshape(-1)
        normal_bf16_bits(w.seed, tid, n, nthreads, out=bits)
        return t

    q = draw(TENSOR_Q, (w.B, w.Hq, w.Nq, w.d))
    if w.scaled_q_rows:
        q[:, :, ::64, :] *= 8
    out = dict(q=q, k=draw(TENSOR_K, (w.B, w.Hkv, w.Nk, w.d)),
               v=draw(TENSOR_V, (w.B, w.Hkv, w.Nk, w.d)))
    if dout and w.backward:
        out["dout"] = draw(TENSOR_DO, (w.B, w.Hq, w.Nq, w.d))
    return out


# Per-tensor descale factors of the e4m3 inputs (value = code * descale).  Not
# powers of two, so a descale applied to the wrong tensor changes the result.
FP8_DESCALE = {"q": 0.0173, "k": 0.0191, "v": 0.0137}
E4M3_MAX = 448.0


def make_inputs_fp8(w: Workload, nthreads: int = 0, pinned: bool = False):
    """Return dict(q, k, v) of CPU uint8 tensors of e4m3 codes for ``w``: the
    same N(0,1) fp32 samples as ``make_inputs`` divided by FP8_DESCALE[name],
    clamped to +-448 and rounded to nearest even e4m3 (torch's float8_e4m3fn
    cast).  The dequantised inputs are code * FP8_DESCALE[name]."""
    import torch

    def draw(tid, shape, descale):
        n = int(np.prod(shape))
        f = torch.from_numpy(normal_f32(w.seed, tid, n, nthreads)).div_(descale)
        f.clamp_(-E4M3_MAX, E4M3_MAX)
        t = f.to(torch.float8_e4m3fn).view(torch.uint8).reshape(shape)
        return t.pin_memory() if pinned else t

    return dict(q=draw(TENSOR_Q, (w.B, w.Hq, w.Nq, w.d), FP8_DESCALE["q"]),
                k=draw(TENSOR_K, (w.B, w.Hkv, w.Nk, w.d), FP8_DESCALE["k"]),
                v=draw(TENSOR_V, (w.B, w.Hkv, w.Nk, w.d), FP8_DESCALE["v"]))
