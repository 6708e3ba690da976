"""GPU test of fa_fwd_splitkv_noalloc, the split-KV forward that allocates no
device memory (for callers that may not allocate on their call path, such as
an inference runtime's plugin whose enqueue step must not allocate).

It must give the same result as fa_fwd_splitkv with a caller workspace, within
the parity tolerances of the other tests (|O| <= 1e-2, |LSE| <= 1e-3), on two
calls in a row with different shapes (the fixed scratch keeps the previous
call's contents, which must not leak into the next result), and it must refuse
a shape whose partials do not fit the fixed scratch.  This file is collected
last so that a stop at the first failure has run every other test already.
"""
import ctypes

import pytest
import torch

import exact_attention_114_b200 as fa
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


def test_noalloc_matches_workspace_entry_point_two_calls():
    for w, splits in CASES:
        assert 0 < fa.fa_fwd_splitkv_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, splits) \
            <= fa.NOALLOC_SCRATCH_BYTES
    inputs = [G.to_gpu(synth.make_inputs(w)) for w, _ in CASES]
    outs = []
    for (w, splits), xd in zip(CASES, inputs):   # two calls in a row
        o = torch.empty_like(xd["q"])
        lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device="cuda")
        fa.fa_fwd_splitkv_noalloc(xd["q"], xd["k"], xd["v"], o, lse, causal=w.causal,
                                  scale=w.scale, num_splits=splits)
        outs.append((o, lse))
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    for (w, splits), xd, (o, lse) in zip(CASES, inputs, outs):
        o_ref, lse_ref = _with_workspace(xd, w, splits)
        torch.cuda.synchronize()
        G.assert_o(G.f64(o), G.f64(o_ref), what="O (no-alloc vs workspace)")
        G.assert_lse(G.f64(lse), G.f64(lse_ref))


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
