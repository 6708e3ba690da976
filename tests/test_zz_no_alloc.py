"""GPU test of fa_fwd_splitkv_noalloc, the split-KV forward that allocates no
device memory (for callers that may not allocate on their call path, such as
an inference runtime's plugin whose enqueue step must not allocate).

On two calls in a row with different shapes (the fixed scratch keeps the
previous call's contents, which must not leak into the next result) its
output must match the fp64 oracle on the same inputs within the parity
tolerances of the other tests (|O - O_ref| <= 1e-2, |LSE - LSE_ref| <= 1e-3)
and agree with fa_fwd_splitkv given a caller workspace.  The call must leave
the device's stream-ordered memory pool untouched (the allocating entry point
is the positive control), the automatic split count must fit the fixed
scratch, and an explicit split count that does not fit must be refused.
This file is collected last so that a stop at the first failure has run
every other test already.
"""
import ctypes

import pytest
import torch

import exact_attention_114_b200 as fa
import oracle
import synth
from tests import gpu_parity as G

pytestmark = pytest.mark.gpu

# (workload, num_splits): two different shapes, each with several splits
CASES = [
    (synth.WORKLOADS["gqa_decode"].with_(B=8), 4),
    (synth.Workload("decode_append", 4, 16, 2, 2, 3000, 128, True, 4242, backward=False), 5),
]


def _with_workspace(xd, w, splits):
    n = fa.fa_fwd_splitkv_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, splits)
    ws = torch.empty(max(n, 1), dtype=torch.uint8, device="cuda")
    return fa.fa_fwd_splitkv(xd["q"], xd["k"], xd["v"], causal=w.causal, scale=w.scale,
                             num_splits=splits, workspace=ws if n else None)


class DefaultPool:
    """High-water mark of used bytes in the current device's default
    stream-ordered memory pool (the pool cudaMallocAsync draws from), read and
    reset through the driver API."""
    USED_MEM_CURRENT, USED_MEM_HIGH = 7, 8   # CUmemPool_attribute

    def __init__(self):
        self.cu = ctypes.CDLL("libcuda.so.1")
        dev = ctypes.c_int()
        assert self.cu.cuCtxGetDevice(ctypes.byref(dev)) == 0
        self.pool = ctypes.c_void_p()
        assert self.cu.cuDeviceGetDefaultMemPool(ctypes.byref(self.pool), dev) == 0

    def _get(self, attr):
        v = ctypes.c_uint64()
        assert self.cu.cuMemPoolGetAttribute(self.pool, attr, ctypes.byref(v)) == 0
        return v.value

    def reset_high(self):
        zero = ctypes.c_uint64(0)   # the only value the high-water mark can be set to
        assert self.cu.cuMemPoolSetAttribute(self.pool, self.USED_MEM_HIGH, ctypes.byref(zero)) == 0

    def used_high(self):
        return self._get(self.USED_MEM_HIGH)

    def used_current(self):
        return self._get(self.USED_MEM_CURRENT)


def test_noalloc_matches_oracle_and_workspace_entry_point_two_calls():
    for w, splits in CASES:
        assert 0 < fa.fa_fwd_splitkv_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, splits) \
            <= fa.NOALLOC_SCRATCH_BYTES
    hosts = [synth.make_inputs(w) for w, _ in CASES]
    inputs = [G.to_gpu(x) for x in hosts]
    outs = [(torch.empty_like(xd["q"]), torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device="cuda"))
            for (w, _), xd in zip(CASES, inputs)]
    torch.cuda.synchronize()
    pool = DefaultPool()
    base = pool.used_current()
    pool.reset_high()
    for (w, splits), xd, (o, lse) in zip(CASES, inputs, outs):   # two calls in a row
        fa.fa_fwd_splitkv_noalloc(xd["q"], xd["k"], xd["v"], o, lse, causal=w.causal,
                                  scale=w.scale, num_splits=splits)
    torch.cuda.synchronize()
    assert pool.used_high() <= base, "the no-allocation call drew memory from the default pool"
    fa.fa_check_device_status()
    for (w, splits), x, xd, (o, lse) in zip(CASES, hosts, inputs, outs):
        o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, w.causal)
        G.assert_o(G.f64(o), o_ref, what="O (no-alloc vs oracle)",
                   o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, w.causal))
        G.assert_lse(G.f64(lse), lse_ref)
        o_ws, lse_ws = _with_workspace(xd, w, splits)
        torch.cuda.synchronize()
        G.assert_o(G.f64(o), G.f64(o_ws), what="O (no-alloc vs workspace call)")
        G.assert_lse(G.f64(lse), G.f64(lse_ws))
    # positive control: the same call without a workspace allocates from the pool
    w, splits = CASES[0]
    xd = inputs[0]
    pool.reset_high()
    fa.fa_fwd_splitkv(xd["q"], xd["k"], xd["v"], causal=w.causal, scale=w.scale, num_splits=splits)
    torch.cuda.synchronize()
    assert pool.used_high() > base, "the pool's high-water mark did not see an allocating call"


def test_noalloc_automatic_split_count_fits_the_fixed_scratch():
    """A shape whose automatic split count would overflow the fixed scratch
    runs with fewer splits and still matches the oracle on sampled rows."""
    # on 148 SMs the automatic choice for this shape is 19 splits, 8.8 MB of partials
    w = synth.Workload("decode_big", 7, 32, 8, 4, 8192, 128, True, 4343, backward=False)
    assert fa.fa_fwd_splitkv_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, 0) \
        > fa.NOALLOC_SCRATCH_BYTES
    x = synth.make_inputs(w)
    xd = G.to_gpu(x)
    o = torch.empty_like(xd["q"])
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device="cuda")
    fa.fa_fwd_splitkv_noalloc(xd["q"], xd["k"], xd["v"], o, lse, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    rows = G.sample_rows(w, n_random=24)
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, True, rows=rows)
    G.assert_o(G.f64(o).reshape(-1, w.d)[rows], o_ref, what="O (no-alloc, automatic splits)",
               o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, True, rows=rows))
    G.assert_lse(G.f64(lse).reshape(-1)[rows], lse_ref)


def test_noalloc_refuses_shapes_beyond_the_fixed_scratch():
    # 64 x 8 kv heads, 16 rows each, 64 splits: 268 MB of partials > 8 MiB
    need = fa.fa_fwd_splitkv_workspace_size(64, 32, 8, 4, 8192, 128, 64)
    assert need > fa.NOALLOC_SCRATCH_BYTES
    q = torch.empty((64, 32, 4, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.empty((64, 8, 8192, 128), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((64, 32, 4), dtype=torch.float32, device="cuda")
    st = fa.lib().fa_fwd_splitkv_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kv.data_ptr()),
        ctypes.c_void_p(kv.data_ptr()), ctypes.c_void_p(o.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()), 64, 32, 8, 4, 8192, 128, 0.0884, 1, 64, None)
    assert st == fa.FA_ERR_WORKSPACE
    assert "scratch" in fa.last_error_message()
