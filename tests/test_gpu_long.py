"""GPU parity at long sequence lengths (the index arithmetic, the many-block
causal schedule and many-split decode): sampled outputs against the oracle."""
import numpy as np
import pytest
import torch

import exact_attention_114_b200 as fa
import oracle
import synth
from tests import gpu_parity as G

pytestmark = pytest.mark.gpu


def test_long_causal_forward_32k():
    w = synth.Workload("long32k", 1, 4, 1, 32768, 32768, 128, True, 9300, backward=False)
    x = synth.make_inputs(w)
    xd = G.to_gpu(x)
    o, lse = G.gpu_forward(xd, w)
    rows = G.sample_rows(w, n_random=16)
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, True, rows=rows)
    G.assert_o(G.f64(o).reshape(-1, w.d)[rows], o_ref,
               o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, True, rows=rows))
    G.assert_lse(G.f64(lse).reshape(-1)[rows], lse_ref)


def test_long_causal_backward_16k():
    w = synth.Workload("long16k", 1, 4, 2, 16384, 16384, 128, True, 9301)
    x = synth.make_inputs(w)
    xd = G.to_gpu(x)
    o, lse = G.gpu_forward(xd, w)
    dq, dk, dv = G.gpu_backward(xd, o, lse, w)
    rows = G.sample_rows(w, n_random=12)
    rq = oracle.bwd_dq_rows(x["q"], x["k"], x["v"], x["dout"], w.scale, True, rows)
    G.assert_grad(G.f64(dq).reshape(-1, w.d)[rows], rq, "dQ (sampled rows)")
    keys = G.sample_keys_cheap(w, kv_heads=(0, 1))
    rk, rv = oracle.bwd_dkv_rows(x["q"], x["k"], x["v"], x["dout"], w.scale, True, keys)
    G.assert_grad(G.f64(dk).reshape(-1, w.d)[keys], rk, "dK (sampled keys)")
    G.assert_grad(G.f64(dv).reshape(-1, w.d)[keys], rv, "dV (sampled keys)")


@pytest.mark.parametrize("splits", [0, 256])
def test_long_decode_128k(splits):
    """Nk = 131072 keys per sequence, GQA 8:1, through the split-KV kernels."""
    w = synth.Workload("dec128k", 2, 16, 2, 1, 131072, 128, False, 9302, backward=False)
    x = synth.make_inputs(w)
    xd = G.to_gpu(x)
    o, lse = fa.fa_fwd_splitkv(xd["q"], xd["k"], xd["v"], num_splits=splits)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, False)
    G.assert_o(G.f64(o), o_ref, o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, False))
    G.assert_lse(G.f64(lse), lse_ref)
