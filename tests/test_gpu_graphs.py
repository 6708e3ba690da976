"""The calls captured into a CUDA graph and replayed.  A call's later kernels are
programmatic dependents of the kernel before them, which stream capture records
as programmatic edges, and the split paths take their scratch stream-ordered
during capture (graph memory nodes).  Each case captures fa_fwd + fa_bwd once,
replays the graph on fresh inputs copied into the captured buffers, and compares
with the same calls run eagerly on those inputs: O, LSE, dK and dV bit for bit
(they repeat from call to call), dQ (an fp32 sum in hardware order) to a rounding
bound, and every output with the oracle."""
import pytest
import torch

import exact_attention_114_b200 as fa
import oracle
import synth
from tests import gpu_parity as G

pytestmark = pytest.mark.gpu

# B, Hq, Hkv, Nq, Nk, d, causal: key split (4 shares) and query split (8 CTAs per unit);
# plain tiles without the mask; the d = 256 forward and feature-split backward; a decode
# shape (split-KV kernels and their merge); a d = 256 decode shape (group rows, key split)
CASES = [
    (1, 4, 1, 2048, 2048, 128, True),
    (1, 8, 2, 1024, 1024, 128, False),
    (1, 2, 1, 640, 900, 256, True),
    (2, 8, 2, 1, 3000, 128, True),
    (2, 8, 2, 1, 3000, 256, False),
]


def _run(x, out, ws, causal, scale):
    fa.fa_fwd(x["q"], x["k"], x["v"], out["o"], out["lse"], causal=causal, scale=scale)
    fa.fa_bwd(x["q"], x["k"], x["v"], out["o"], x["dout"], out["lse"], out["dq"], out["dk"], out["dv"],
              causal=causal, scale=scale, workspace=ws)


def _outputs(x):
    B, Hq, Nq, _ = x["q"].shape
    return {"o": torch.empty_like(x["q"]), "lse": torch.empty(B, Hq, Nq, dtype=torch.float32, device="cuda"),
            "dq": torch.empty_like(x["q"]), "dk": torch.empty_like(x["k"]), "dv": torch.empty_like(x["v"])}


@pytest.mark.parametrize("shape", CASES, ids=[str(c) for c in CASES])
def test_graph_replay_matches_eager(shape):
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    i = CASES.index(shape)
    w_cap = synth.Workload("graph_capture", B, Hq, Hkv, Nq, Nk, d, causal, 9400 + 2 * i)
    w = synth.Workload("graph_replay", B, Hq, Hkv, Nq, Nk, d, causal, 9401 + 2 * i)
    x = {k: v.cuda() for k, v in synth.make_inputs(w_cap).items()}
    fresh = synth.make_inputs(w)
    out = _outputs(x)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, Hq, Hkv, Nq, Nk, d), dtype=torch.uint8, device="cuda")

    # one eager pass on a side stream first (library set-up happens outside the capture)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        _run(x, out, ws, causal, w.scale)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _run(x, out, ws, causal, w.scale)
    for k, v in fresh.items():
        x[k].copy_(v)
    g.replay()
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    got = {k: v.clone() for k, v in out.items()}
    g.replay()
    torch.cuda.synchronize()
    for k in ("o", "lse", "dk", "dv"):
        assert torch.equal(out[k], got[k]), f"{k}: two replays differ"

    eager = _outputs(x)
    _run(x, eager, ws, causal, w.scale)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    for k in ("o", "lse", "dk", "dv"):
        assert torch.equal(got[k], eager[k]), f"{k}: replay differs from the eager call"
    err = (got["dq"].float() - eager["dq"].float()).abs().max().item()
    assert err <= 1e-2 * eager["dq"].float().abs().max().item() + 1e-3, err
    del g

    xr = {k: v.double() for k, v in fresh.items()}
    o_ref, lse_ref = oracle.fwd(xr["q"], xr["k"], xr["v"], w.scale, causal)
    G.assert_o(G.f64(got["o"]), o_ref, o_abs=G.o_abs_ref(xr["q"], xr["k"], xr["v"], w.scale, causal))
    G.assert_lse(G.f64(got["lse"]), lse_ref)
    rq, rk, rv = oracle.bwd(xr["q"], xr["k"], xr["v"], xr["dout"], w.scale, causal)
    G.assert_grad(G.f64(got["dq"]), rq, "dQ")
    G.assert_grad(G.f64(got["dk"]), rk, "dK")
    G.assert_grad(G.f64(got["dv"]), rv, "dV")


def _programmatic_edges(fn):
    """A CUDA graph captured (relaxed mode) from the work fn enqueues on a fresh stream,
    never launched: (programmatic edges from a kernel node to a kernel node, kernel nodes,
    the node types at both ends of every programmatic edge)."""
    from cuda.bindings import runtime as rt
    ok = rt.cudaError_t.cudaSuccess
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        err, = rt.cudaStreamBeginCapture(stream.cuda_stream,
                                         rt.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
        assert err == ok, err
        try:
            fn()
        finally:
            err, graph = rt.cudaStreamEndCapture(stream.cuda_stream)
    assert err == ok, err
    try:
        res = rt.cudaGraphGetEdges_v2(graph, 0)
        assert res[0] == ok, res[0]
        err, src, dst, data, n = rt.cudaGraphGetEdges_v2(graph, res[-1])
        assert err == ok, err
        kernel = rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
        kind = lambda nd: rt.cudaGraphNodeGetType(nd)[1]
        # a programmatic edge: its type, or its source port (programmatic / launch completion)
        prog = [(kind(a), kind(b)) for a, b, e in zip(src[:n], dst[:n], data[:n])
                if int(e.type) == int(rt.cudaGraphDependencyType.cudaGraphDependencyTypeProgrammatic)
                or int(e.from_port) != int(rt.cudaGraphKernelNodePortDefault)]
        err, _, m = rt.cudaGraphGetNodes(graph, 0)
        err, nodes, m = rt.cudaGraphGetNodes(graph, m)
        kernels = sum(1 for nd in nodes[:m] if kind(nd) == kernel)
        return sum(1 for a, b in prog if a == kernel and b == kernel), kernels, prog
    finally:
        rt.cudaGraphDestroy(graph)


def test_capture_records_programmatic_edges():
    """A call's later kernels are programmatic dependents of the kernel before them:
    the backward's main and post passes (2 kernel-to-kernel edges), the merge of a
    key-split forward and of a split-KV decode (1 each), the e4m3 forward kernel after
    its V transpose (1); a plain forward has none."""
    w = synth.Workload("graph_edges", 1, 4, 1, 2048, 2048, 128, True, 9460)
    x = {k: v.cuda() for k, v in synth.make_inputs(w).items()}
    o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=True)
    ws = torch.empty(fa.fa_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d), dtype=torch.uint8,
                     device="cuda")
    g = [torch.empty_like(x[k]) for k in ("q", "k", "v")]
    torch.cuda.synchronize()
    prog, kern, edges = _programmatic_edges(
        lambda: fa.fa_bwd(x["q"], x["k"], x["v"], o, x["dout"], lse, *g, causal=True, workspace=ws))
    assert (prog, kern) == (2, 3), edges
    assert fa.fa_fwd_kv_split(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, True) > 1
    prog, kern, edges = _programmatic_edges(lambda: fa.fa_fwd(x["q"], x["k"], x["v"], o, lse, causal=True))
    assert (prog, kern) == (1, 2), edges
    w2 = synth.Workload("graph_edges_plain", 1, 32, 8, 2048, 2048, 128, True, 9461, backward=False)
    x2 = {k: v.cuda() for k, v in synth.make_inputs(w2, dout=False).items()}
    assert fa.fa_fwd_kv_split(w2.B, w2.Hq, w2.Hkv, w2.Nq, w2.Nk, w2.d, True) == 1
    o2, lse2 = fa.fa_fwd(x2["q"], x2["k"], x2["v"], causal=True)
    prog, kern, edges = _programmatic_edges(
        lambda: fa.fa_fwd(x2["q"], x2["k"], x2["v"], o2, lse2, causal=True))
    assert (prog, kern) == (0, 1), edges
    w3 = synth.Workload("graph_edges_decode", 2, 8, 2, 1, 3000, 128, True, 9462, backward=False)
    x3 = {k: v.cuda() for k, v in synth.make_inputs(w3, dout=False).items()}
    o3, lse3 = fa.fa_fwd_splitkv(x3["q"], x3["k"], x3["v"], causal=True, num_splits=4)
    torch.cuda.synchronize()
    prog, kern, edges = _programmatic_edges(
        lambda: fa.fa_fwd_splitkv(x3["q"], x3["k"], x3["v"], o3, lse3, causal=True, num_splits=4))
    assert (prog, kern) == (1, 2), edges
    # e4m3: the forward kernel after the V transpose (no key split at this size)
    w4 = synth.Workload("graph_edges_fp8", 1, 32, 8, 2048, 2048, 128, True, 9463, backward=False)
    assert fa.fa_fwd_kv_split(w4.B, w4.Hq, w4.Hkv, w4.Nq, w4.Nk, w4.d, True) == 1
    x4 = {k: v.cuda() for k, v in synth.make_inputs_fp8(w4).items()}
    ds = synth.FP8_DESCALE
    vt = torch.empty(fa.fa_fwd_fp8_workspace_size(w4.B, w4.Hkv, w4.Nk, w4.d), dtype=torch.uint8, device="cuda")
    o4, lse4 = fa.fa_fwd_fp8(x4["q"], x4["k"], x4["v"], ds["q"], ds["k"], ds["v"], causal=True, workspace=vt)
    torch.cuda.synchronize()
    prog, kern, edges = _programmatic_edges(
        lambda: fa.fa_fwd_fp8(x4["q"], x4["k"], x4["v"], ds["q"], ds["k"], ds["v"], o4, lse4, causal=True,
                              workspace=vt))
    assert (prog, kern) == (1, 2), edges
