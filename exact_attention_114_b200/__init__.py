"""Python binding of libfa (exact attention for B200, sm_100a).

Argument marshalling only: every function here forwards torch device tensors
(as raw pointers, sizes and the current CUDA stream) to the C ABI declared in
``include/fa.h`` and raises ``FaError`` on a non-OK status.  There is no
fallback: if ``libfa.so`` has not been built, loading fails loudly.

Layouts (BHSD, contiguous): q, o, dout, dq [B, Hq, Nq, d]; k, v, dk, dv
[B, Hkv, Nk, d] in bf16; lse [B, Hq, Nq] in fp32.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

FA_OK = 0
FA_ERR_INVALID_ARGUMENT = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_WORKSPACE = 3
FA_ERR_CUDA = 4
FA_ERR_TIMEOUT = 5
FA_ERR_SLOT_CONFLICT = 6

FA_DTYPE_BF16 = 0
FA_DTYPE_FP16 = 1

_lock = threading.Lock()
_lib = None


class FaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{status_string(status)}: {message}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded libfa.so (raises if it was not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"libfa.so is missing at {LIB_PATH}; build it with "
                    "`python -m exact_attention_114_b200.build` (needs nvcc)")
            L = ctypes.CDLL(LIB_PATH)
            vp, ip, fl, sz, uip = (ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t,
                                   ctypes.c_uint)
            L.fa_abi_version.argtypes = []
            L.fa_abi_version.restype = ip
            L.fa_status_string.argtypes = [ip]
            L.fa_status_string.restype = ctypes.c_char_p
            L.fa_last_error_message.argtypes = []
            L.fa_last_error_message.restype = ctypes.c_char_p
            L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, ip, ip, ip, ip, ip, ip, fl, ip, vp]
            L.fa_fwd.restype = ip
            L.fa_fwd_ex.argtypes = [ip, vp, vp, vp, vp, vp, ip, ip, ip, ip, ip, ip, fl, ip, vp]
            L.fa_fwd_ex.restype = ip
            L.fa_bwd_ex.argtypes = [ip, vp, vp, vp, vp, vp, vp, vp, vp, vp, ip, ip, ip, ip, ip, ip, fl, ip,
                                    vp, sz, vp]
            L.fa_bwd_ex.restype = ip
            L.fa_fwd_fp8_workspace_size.argtypes = [ip, ip, ip, ip]
            L.fa_fwd_fp8_workspace_size.restype = sz
            L.fa_fwd_fp8.argtypes = [vp, vp, vp, fl, fl, fl, vp, vp, ip, ip, ip, ip, ip, ip, fl, ip, vp,
                                     sz, vp]
            L.fa_fwd_fp8.restype = ip
            L.fa_fwd_splitkv_workspace_size.argtypes = [ip, ip, ip, ip, ip, ip, ip]
            L.fa_fwd_splitkv_workspace_size.restype = sz
            L.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, ip, ip, ip, ip, ip, ip, fl, ip, ip, vp,
                                         sz, vp]
            L.fa_fwd_splitkv.restype = ip
            L.fa_fwd_splitkv_noalloc.argtypes = [vp, vp, vp, vp, vp, ip, ip, ip, ip, ip, ip, fl, ip,
                                                  ip, vp]
            L.fa_fwd_splitkv_noalloc.restype = ip
            L.fa_fwd_paged_workspace_size.argtypes = [ip, ip, ip, ip, ip, ip, ip, ip]
            L.fa_fwd_paged_workspace_size.restype = sz
            L.fa_fwd_paged.argtypes = [vp, vp, vp, vp, vp, vp, vp, ip, ip, ip, ip, ip, ip, ip, ip, fl,
                                       ip, ip, vp, sz, vp]
            L.fa_fwd_paged.restype = ip
            L.fa_fwd_paged_ex.argtypes = [ip] + list(L.fa_fwd_paged.argtypes)
            L.fa_fwd_paged_ex.restype = ip
            L.fa_bwd_workspace_size.argtypes = [ip, ip, ip, ip, ip, ip]
            L.fa_bwd_workspace_size.restype = sz
            L.fa_bwd_query_split.argtypes = [ip, ip, ip, ip, ip, ip, ip]
            L.fa_bwd_query_split.restype = ip
            L.fa_fwd_kv_split.argtypes = [ip, ip, ip, ip, ip, ip, ip]
            L.fa_fwd_kv_split.restype = ip
            L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, ip, ip, ip, ip, ip, ip, fl, ip,
                                 vp, sz, vp]
            L.fa_bwd.restype = ip
            L.fa_check_device_status.argtypes = [vp]
            L.fa_check_device_status.restype = ip
            L.fa_selftest_wait_timeout.argtypes = [uip, vp]
            L.fa_selftest_wait_timeout.restype = ip
            L.fa_testhook_tile_slot.argtypes = [ip, uip]
            L.fa_testhook_tile_slot.restype = ip
            _lib = L
        return _lib


def status_string(status: int) -> str:
    try:
        return lib().fa_status_string(int(status)).decode()
    except ImportError:
        return f"status {status}"


def last_error_message() -> str:
    return lib().fa_last_error_message().decode()


def _check(status: int):
    if status != FA_OK:
        raise FaError(status, last_error_message())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dims(q, k):
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if B != Bk or d != dk:
        raise ValueError(f"q {tuple(q.shape)} and k {tuple(k.shape)} disagree")
    return B, Hq, Hkv, Nq, Nk, d


def _require(t, name, dtype, shape=None):
    """t must be a contiguous CUDA tensor of `dtype` (and of `shape`, if given):
    the C ABI only sees a pointer, so a wrong type is read as garbage and a
    short buffer is written past its end."""
    if not t.is_cuda or not t.is_contiguous() or t.dtype != dtype:
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _require_lse(lse, B, Hq, Nq):
    import torch
    if lse is not None:
        _require(lse, "lse", torch.float32, (B, Hq, Nq))


def _ws_bytes(workspace):
    """Size in bytes of a workspace tensor (contiguous, on the device), or 0 for None."""
    if workspace is None:
        return 0
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return workspace.numel() * workspace.element_size()


def _check_io(q, k, v, o, dtype):
    """q, k, v, o of one 16-bit dtype; v shaped like k, o like q."""
    _require(q, "q", dtype)
    _require(k, "k", dtype)
    _require(v, "v", dtype, k.shape)
    if o is not None:
        _require(o, "o", dtype, q.shape)


def _dtype_code(t):
    """FA_DTYPE_* of a 16-bit tensor."""
    import torch
    if t.dtype == torch.bfloat16:
        return FA_DTYPE_BF16
    if t.dtype == torch.float16:
        return FA_DTYPE_FP16
    raise ValueError(f"unsupported dtype {t.dtype} (bf16 or fp16)")


def abi_version() -> int:
    return int(lib().fa_abi_version())


def fa_fwd(q, k, v, o=None, lse=None, *, causal=False, scale=None, stream=None, want_lse=True):
    """Forward: returns (o, lse).  Allocates o / lse when not given.  bf16
    tensors go to fa_fwd, fp16 tensors to fa_fwd_ex."""
    import torch
    B, Hq, Hkv, Nq, Nk, d = _dims(q, k)
    dt = _dtype_code(q)
    _check_io(q, k, v, o, q.dtype)
    _require_lse(lse, B, Hq, Nq)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if dt == FA_DTYPE_BF16:
        _check(lib().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, d,
                            scale, int(bool(causal)), _stream(stream)))
    else:
        _check(lib().fa_fwd_ex(dt, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk,
                               d, scale, int(bool(causal)), _stream(stream)))
    return o, lse


def fa_fwd_fp8_workspace_size(B, Hkv, Nk, d) -> int:
    return int(lib().fa_fwd_fp8_workspace_size(B, Hkv, Nk, d))


def fa_fwd_fp8(q, k, v, descale_q, descale_k, descale_v, o=None, lse=None, *, causal=False,
               scale=None, workspace=None, stream=None, want_lse=True):
    """Forward with e4m3 inputs (uint8 or float8_e4m3fn CUDA tensors, d = 128)
    and per-tensor descales.  Returns (o, lse) with o in bf16."""
    import torch
    B, Hq, Hkv, Nq, Nk, d = _dims(q, k)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if not t.is_cuda or not t.is_contiguous() or t.element_size() != 1:
            raise ValueError(f"{n} must be a contiguous CUDA tensor of e4m3 bytes")
    if tuple(v.shape) != tuple(k.shape):
        raise ValueError(f"v has shape {tuple(v.shape)}, expected {tuple(k.shape)}")
    if o is None:
        o = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    _require(o, "o", torch.bfloat16, q.shape)
    _require_lse(lse, B, Hq, Nq)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    ws_bytes = _ws_bytes(workspace)
    _check(lib().fa_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), float(descale_q), float(descale_k),
                            float(descale_v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, d, scale,
                            int(bool(causal)), _ptr(workspace), ws_bytes, _stream(stream)))
    return o, lse


def fa_fwd_ex(dtype, q, k, v, o, lse, *, causal=False, scale=None, stream=None):
    """The C call fa_fwd_ex with an explicit FA_DTYPE_* code."""
    B, Hq, Hkv, Nq, Nk, d = _dims(q, k)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(lib().fa_fwd_ex(int(dtype), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq,
                           Nk, d, scale, int(bool(causal)), _stream(stream)))
    return o, lse


def fa_fwd_splitkv_workspace_size(B, Hq, Hkv, Nq, Nk, d, num_splits=0) -> int:
    return int(lib().fa_fwd_splitkv_workspace_size(B, Hq, Hkv, Nq, Nk, d, num_splits))


def fa_fwd_splitkv(q, k, v, o=None, lse=None, *, causal=False, scale=None, num_splits=0,
                   workspace=None, stream=None):
    """Split-KV (decode-shape) forward on bf16 tensors.  ``workspace`` is an
    optional device tensor of at least ``fa_fwd_splitkv_workspace_size`` bytes."""
    import torch
    B, Hq, Hkv, Nq, Nk, d = _dims(q, k)
    _check_io(q, k, v, o, torch.bfloat16)
    _require_lse(lse, B, Hq, Nq)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    ws_bytes = _ws_bytes(workspace)
    _check(lib().fa_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq,
                                Nk, d, scale, int(bool(causal)), int(num_splits), _ptr(workspace),
                                ws_bytes, _stream(stream)))
    return o, lse


def fa_fwd_paged_workspace_size(B, Hq, Hkv, Nq, page_size, max_pages_per_seq, d, num_splits=0) -> int:
    return int(lib().fa_fwd_paged_workspace_size(B, Hq, Hkv, Nq, page_size, max_pages_per_seq, d,
                                                 num_splits))


def fa_fwd_paged(q, k_cache, v_cache, block_table, seq_lens, o=None, lse=None, *, causal=False,
                 scale=None, num_splits=0, workspace=None, stream=None):
    """Decode over a paged KV cache.  k_cache/v_cache [num_pages, page_size, Hkv, d] bf16 or
    fp16 (the type of q), block_table int32 [B, max_pages_per_seq], seq_lens int32 [B],
    q [B, Hq, Nq, d]."""
    import torch
    B, Hq, Nq, d = q.shape
    num_pages, page_size, Hkv, dk = k_cache.shape
    if dk != d or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("k_cache / v_cache shapes disagree with q")
    for t, n in ((block_table, "block_table"), (seq_lens, "seq_lens")):
        if not t.is_cuda or t.dtype != torch.int32 or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous CUDA int32 tensor")
    if block_table.dim() != 2 or block_table.shape[0] != B or tuple(seq_lens.shape) != (B,):
        raise ValueError("block_table must be [B, max_pages_per_seq] and seq_lens [B]")
    max_pages = block_table.shape[1]
    dt = _dtype_code(q)
    _require(q, "q", q.dtype)
    _require(k_cache, "k_cache", q.dtype)
    _require(v_cache, "v_cache", q.dtype)
    if o is not None:
        _require(o, "o", q.dtype, q.shape)
    _require_lse(lse, B, Hq, Nq)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    ws_bytes = _ws_bytes(workspace)
    _check(lib().fa_fwd_paged_ex(dt, _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                 _ptr(seq_lens), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, d, page_size,
                                 num_pages, max_pages, scale, int(bool(causal)), int(num_splits),
                                 _ptr(workspace), ws_bytes, _stream(stream)))
    return o, lse


NOALLOC_SCRATCH_BYTES = 8 * 1024 * 1024  # FA_SPLITKV_NOALLOC_SCRATCH_BYTES in fa.h


def fa_fwd_splitkv_noalloc(q, k, v, o, lse, *, causal=False, scale=None, num_splits=0,
                           stream=None):
    """Split-KV forward on bf16 tensors that allocates nothing on the device:
    its partials use a fixed array inside the library.  ``o`` [B, Hq, Nq, d]
    bf16 and ``lse`` [B, Hq, Nq] fp32 must be given (this wrapper allocates
    nothing either).  Calls that overlap on the GPU race on the shared array."""
    import torch
    B, Hq, Hkv, Nq, Nk, d = _dims(q, k)
    if o is None or lse is None:
        raise ValueError("fa_fwd_splitkv_noalloc needs o and lse (it allocates nothing)")
    _check_io(q, k, v, o, torch.bfloat16)
    _require_lse(lse, B, Hq, Nq)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(lib().fa_fwd_splitkv_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv,
                                        Nq, Nk, d, scale, int(bool(causal)), int(num_splits),
                                        _stream(stream)))
    return o, lse


def fa_bwd_workspace_size(B, Hq, Hkv, Nq, Nk, d) -> int:
    return int(lib().fa_bwd_workspace_size(B, Hq, Hkv, Nq, Nk, d))


def fa_fwd_kv_split(B, Hq, Hkv, Nq, Nk, d, causal) -> int:
    """Key shares per work tile of fa_fwd on the current device (1: no split;
    0: bad sizes)."""
    return int(lib().fa_fwd_kv_split(B, Hq, Hkv, Nq, Nk, d, int(bool(causal))))


def fa_bwd_query_split(B, Hq, Hkv, Nq, Nk, d, causal) -> int:
    """CTAs that fa_bwd shares each (key block, kv head) unit between on the
    current device, given a full-size workspace (1: no split; 0: bad sizes)."""
    return int(lib().fa_bwd_query_split(B, Hq, Hkv, Nq, Nk, d, int(bool(causal))))


def fa_bwd(q, k, v, o, dout, lse, dq=None, dk=None, dv=None, *, causal=False, scale=None,
           workspace=None, stream=None):
    """Backward: returns (dq, dk, dv).  Allocates the gradients when not given."""
    import torch
    B, Hq, Hkv, Nq, Nk, d = _dims(q, k)
    dt = _dtype_code(q)
    _check_io(q, k, v, o, q.dtype)
    _require(dout, "dout", q.dtype, q.shape)
    _require(lse, "lse", torch.float32, (B, Hq, Nq))
    for t, n, ref in ((dq, "dq", q), (dk, "dk", k), (dv, "dv", v)):
        if t is not None:
            _require(t, n, q.dtype, ref.shape)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    ws_bytes = _ws_bytes(workspace)
    if dt == FA_DTYPE_BF16:
        _check(lib().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                            _ptr(dk), _ptr(dv), B, Hq, Hkv, Nq, Nk, d, scale, int(bool(causal)),
                            _ptr(workspace), ws_bytes, _stream(stream)))
    else:
        _check(lib().fa_bwd_ex(dt, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                               _ptr(dq), _ptr(dk), _ptr(dv), B, Hq, Hkv, Nq, Nk, d, scale,
                               int(bool(causal)), _ptr(workspace), ws_bytes, _stream(stream)))
    return dq, dk, dv


def fa_check_device_status(stream=None):
    _check(lib().fa_check_device_status(_stream(stream)))


def fa_selftest_wait_timeout(timeout_us: int = 2000, stream=None) -> int:
    """Runs the bounded-wait self-test; returns the raw status (5 = timeout seen)."""
    return int(lib().fa_selftest_wait_timeout(int(timeout_us), _stream(stream)))


def fa_testhook_tile_slot(slot: int, preset_owner: int = 0):
    """Test hook: pin later tiled forward launches to counter slot ``slot``
    (-1 restores the rotation), optionally presetting the slot's owner tag."""
    _check(lib().fa_testhook_tile_slot(int(slot), int(preset_owner)))
