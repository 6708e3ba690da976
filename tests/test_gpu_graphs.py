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
