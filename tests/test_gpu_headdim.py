"""GPU parity for head dims 32 and 96 (run on the 64 and 128 kernels with the
missing columns zero-filled by TMA) against the oracle: forward and backward,
tails around the tiles, GQA, causal and not."""
import pytest
import torch

import exact_attention_114_b200 as fa
import oracle
import synth
from tests import gpu_parity as G

pytestmark = pytest.mark.gpu

SHAPES = [
    # B, Hq, Hkv, Nq, Nk, d, causal
    (1, 2, 1, 1, 1, 32, False),
    (1, 2, 1, 63, 63, 32, True),
    (2, 4, 2, 257, 257, 32, True),
    (1, 2, 2, 200, 333, 32, False),
    (1, 2, 1, 65, 65, 96, True),
    (1, 4, 2, 300, 300, 96, True),
    (1, 2, 2, 333, 200, 96, True),
    (1, 8, 1, 70, 640, 96, False),
    (2, 2, 2, 513, 513, 96, True),
]
DTYPES = [torch.bfloat16, torch.float16]


@pytest.mark.parametrize("dtype", DTYPES, ids=["bf16", "fp16"])
@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_headdim_forward_backward(shape, dtype):
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    w = synth.Workload("headdim", B, Hq, Hkv, Nq, Nk, d, causal, 6300 + SHAPES.index(shape))
    x = synth.make_inputs(w, dtype=dtype)
    xd = {k: v.cuda() for k, v in x.items()}
    # guard the columns next to each row: a store past d would land in the next row
    o = torch.full_like(xd["q"], float("nan"))
    o, lse = fa.fa_fwd(xd["q"], xd["k"], xd["v"], o=o, causal=causal)
    dq = torch.full_like(xd["q"], float("nan"))
    dk = torch.full_like(xd["k"], float("nan"))
    dv = torch.full_like(xd["v"], float("nan"))
    dq, dk, dv = fa.fa_bwd(xd["q"], xd["k"], xd["v"], o, xd["dout"], lse, dq=dq, dk=dk, dv=dv,
                           causal=causal)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    xr = {k: v.double() for k, v in x.items()}
    o_ref, lse_ref = oracle.fwd(xr["q"], xr["k"], xr["v"], w.scale, causal)
    G.assert_o(G.f64(o), o_ref)
    G.assert_lse(G.f64(lse), lse_ref)
    rq, rk, rv = oracle.bwd(xr["q"], xr["k"], xr["v"], xr["dout"], w.scale, causal)
    G.assert_grad(G.f64(dq), rq, "dQ")
    G.assert_grad(G.f64(dk), rk, "dK")
    G.assert_grad(G.f64(dv), rv, "dV")
