"""GPU test of fa_fwd_splitkv_noalloc, the split-KV forward that allocates no
device memory (for callers that may not allocate on their call path, such as
an inference runtime's plugin whose enqueue step must not allocate).

On two calls in a row with different shapes (the fixed scratch keeps the
previous call's contents, which must not leak into the next result) its
output must match the fp64 oracle on the same inputs within the parity
tolerances of the other tests (|O - O_ref| <= 1e-2, |LSE - LSE_ref| <= 1e-3)
and agree with fa_fwd_splitkv given a caller workspace.  Captured into a CUDA
graph, the call must add no memory-allocation node (the allocating entry point,
captured the same way, adds one: the positive control); the automatic split
count must fit the fixed scratch, and an explicit split count that does not fit
must be refused.
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


def alloc_nodes(fn):
    """Memory-allocation nodes of a CUDA graph captured (relaxed mode) from the
    work fn enqueues on a fresh stream; the graph is never launched."""
    from cuda.bindings import runtime as rt
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        err, = rt.cudaStreamBeginCapture(stream.cuda_stream,
                                         rt.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
        assert err == rt.cudaError_t.cudaSuccess, err
        try:
            fn()
        finally:
            err, graph = rt.cudaStreamEndCapture(stream.cuda_stream)
    assert err == rt.cudaError_t.cudaSuccess, err
    try:
        err, _, n = rt.cudaGraphGetNodes(graph, 0)
        assert err == rt.cudaError_t.cudaSuccess, err
        err, nodes, n = rt.cudaGraphGetNodes(graph, n)
        assert err == rt.cudaError_t.cudaSuccess, err
        kinds = [rt.cudaGraphNodeGetType(nd)[1] for nd in nodes[:n]]
        return sum(1 for k in kinds if k == rt.cudaGraphNodeType.cudaGraphNodeTypeMemAlloc), len(kinds)
    finally:
        rt.cudaGraphDestroy(graph)


def test_noalloc_matches_oracle_and_workspace_entry_point_two_calls():
    for w, splits in CASES:
        assert 0 < fa.fa_fwd_splitkv_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, splits) \
            <= fa.NOALLOC_SCRATCH_BYTES
    hosts = [synth.make_inputs(w) for w, _ in CASES]
    inputs = [G.to_gpu(x) for x in hosts]
    outs = [(torch.empty_like(xd["q"]), torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device="cuda"))
            for (w, _), xd in zip(CASES, inputs)]
    torch.cuda.synchronize()
    for (w, splits), xd, (o, lse) in zip(CASES, inputs, outs):   # two calls in a row
        fa.fa_fwd_splitkv_noalloc(xd["q"], xd["k"], xd["v"], o, lse, causal=w.causal,
                                  scale=w.scale, num_splits=splits)
    torch.cuda.synchronize()
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
    # captured into a graph the no-allocation call adds no allocation node; the same
    # call without a workspace (the allocating entry point) adds one
    w, splits = CASES[0]
    xd = inputs[0]
    o, lse = outs[0]
    n_alloc, n_nodes = alloc_nodes(lambda: fa.fa_fwd_splitkv_noalloc(
        xd["q"], xd["k"], xd["v"], o, lse, causal=w.causal, scale=w.scale, num_splits=splits))
    assert n_nodes > 0 and n_alloc == 0, (n_alloc, n_nodes)
    n_alloc, n_nodes = alloc_nodes(lambda: fa.fa_fwd_splitkv(
        xd["q"], xd["k"], xd["v"], o, lse, causal=w.causal, scale=w.scale, num_splits=splits))
    assert n_alloc >= 1, "the allocating entry point added no allocation node"

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
