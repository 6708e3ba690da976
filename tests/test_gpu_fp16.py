"""GPU parity for fp16 inputs (fa_fwd_ex / fa_bwd_ex with FA_DTYPE_FP16) against
the oracle, which reads the fp16 values exactly as doubles."""
import numpy as np
import pytest
import torch

import exact_attention_114_b200 as fa
import oracle
import synth
from tests import gpu_parity as G

pytestmark = pytest.mark.gpu

SHAPES = [
    # B, Hq, Hkv, Nq, Nk, d, causal
    (1, 2, 1, 63, 63, 64, True),
    (2, 2, 1, 65, 65, 128, True),
    (1, 4, 2, 300, 300, 128, True),
    (1, 2, 2, 333, 200, 128, True),
    (1, 8, 1, 70, 640, 64, False),
    (1, 4, 4, 513, 513, 128, False),
    (3, 32, 8, 1, 700, 128, False),     # decode shape: split-KV kernels
    (2, 8, 2, 4, 1000, 128, True),      # append shape: split-KV kernels
]


def _case(shape, seed):
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    w = synth.Workload("fp16", B, Hq, Hkv, Nq, Nk, d, causal, seed)
    x = synth.make_inputs(w, dtype=torch.float16)
    return w, x, {k: v.cuda() for k, v in x.items()}


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_fp16_forward_backward(shape):
    w, x, xd = _case(shape, 6100 + SHAPES.index(shape))
    assert xd["q"].dtype == torch.float16
    o, lse = fa.fa_fwd(xd["q"], xd["k"], xd["v"], causal=w.causal)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    assert o.dtype == torch.float16
    xr = {k: v.double() for k, v in x.items()}
    o_ref, lse_ref = oracle.fwd(xr["q"], xr["k"], xr["v"], w.scale, w.causal)
    G.assert_o(G.f64(o), o_ref, o_abs=G.o_abs_ref(xr["q"], xr["k"], xr["v"], w.scale, w.causal))
    G.assert_lse(G.f64(lse), lse_ref)
    if w.Nq * w.G <= 16 and w.d == 128:
        return  # decode shapes: forward only
    dq, dk, dv = fa.fa_bwd(xd["q"], xd["k"], xd["v"], o, xd["dout"], lse, causal=w.causal)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    rq, rk, rv = oracle.bwd(xr["q"], xr["k"], xr["v"], xr["dout"], w.scale, w.causal)
    G.assert_grad(G.f64(dq), rq, "dQ")
    G.assert_grad(G.f64(dk), rk, "dK")
    G.assert_grad(G.f64(dv), rv, "dV")


def test_fp16_gqa_config_sampled():
    """The GQA N=8192 workload in fp16, sampled rows of the forward."""
    w = synth.WORKLOADS["gqa_8k"]
    x = synth.make_inputs(w, dout=False, dtype=torch.float16)
    xd = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fa_fwd(xd["q"], xd["k"], xd["v"], causal=True)
    torch.cuda.synchronize()
    rows = G.sample_rows(w, n_random=32)
    o_ref, lse_ref = oracle.fwd(x["q"].double(), x["k"].double(), x["v"].double(), w.scale, True,
                                rows=rows)
    G.assert_o(G.f64(o).reshape(-1, w.d)[rows], o_ref,
               o_abs=G.o_abs_ref(x["q"].double(), x["k"].double(), x["v"].double(), w.scale, True, rows=rows))
    G.assert_lse(G.f64(lse).reshape(-1)[rows], lse_ref)


def test_bad_dtype_code_is_rejected():
    q = torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd_ex(7, q, q, q, torch.empty_like(q), None)
    assert e.value.status == fa.FA_ERR_INVALID_ARGUMENT
