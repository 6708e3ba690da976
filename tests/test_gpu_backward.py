"""GPU parity: libfa backward (pre, key-stationary tcgen05 main kernel, post)
against the oracle's analytic backward on seeded inputs."""
import numpy as np
import pytest
import torch

import exact_attention_114_b200 as fa
import oracle
import synth
from tests import gpu_parity as G

pytestmark = pytest.mark.gpu

BWD_SHAPES = [
    (1, 1, 1, 1, 1, 64, False),
    (1, 2, 1, 63, 63, 64, True),
    (1, 2, 2, 64, 64, 128, False),
    (2, 2, 1, 65, 65, 128, True),
    (1, 4, 4, 128, 128, 128, True),
    (1, 2, 1, 129, 129, 64, True),
    (1, 4, 2, 300, 300, 128, True),
    (1, 2, 2, 513, 513, 64, False),
    (1, 4, 4, 200, 333, 128, True),
    (1, 2, 2, 333, 200, 128, True),
    (1, 8, 1, 70, 640, 128, False),
    (2, 8, 2, 256, 256, 64, True),
    (1, 4, 1, 1000, 1000, 128, True),
]


@pytest.mark.parametrize("shape", BWD_SHAPES, ids=[str(s) for s in BWD_SHAPES])
def test_backward_shapes(shape):
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    w = synth.Workload("case", B, Hq, Hkv, Nq, Nk, d, causal, 9000 + BWD_SHAPES.index(shape))
    _, _, (x, xd, o, lse) = G.check_forward_full(w)
    G.check_backward_full(w, x, xd, o, lse)


@pytest.mark.parametrize("name", ["tiny_mha", "mha_1k", "mha_1k_noncausal"])
def test_backward_config_full(name):
    w = synth.WORKLOADS[name]
    _, _, (x, xd, o, lse) = G.check_forward_full(w)
    G.check_backward_full(w, x, xd, o, lse)


@pytest.mark.parametrize("name", ["mha_4k_long", "gqa_8k"])
def test_backward_config_one_group_full(name):
    """One full kv group at a quarter of the sequence: every dQ/dK/dV element,
    many 64-row query blocks per key block, the GQA reduction over the group."""
    w = synth.WORKLOADS[name]
    w = w.with_(B=1, Hq=w.G, Hkv=1, Nq=w.Nq // 4, Nk=w.Nk // 4)
    _, _, (x, xd, o, lse) = G.check_forward_full(w)
    G.check_backward_full(w, x, xd, o, lse)


@pytest.mark.parametrize("name", ["mha_4k_long", "gqa_8k"])
def test_backward_config_sampled(name):
    """Full-size inputs and launch; dQ on sampled rows; dK/dV element by element
    on keys near the end (seen by few rows) and on the heaviest keys (seen by
    every row of the group: at gqa_8k the CTA of key block 0 accumulates dK/dV
    in tensor memory over 4 heads x 128 query blocks = 512 steps), on the first
    and last kv heads; plus the dV column-sum identity sum_j dV_j = sum of dO
    over the group's rows."""
    w = synth.WORKLOADS[name]
    x = synth.make_inputs(w)
    xd = G.to_gpu(x)
    o, lse = G.gpu_forward(xd, w)
    dq, dk, dv = G.gpu_backward(xd, o, lse, w)
    d = w.d
    rows = G.sample_rows(w, n_random=32)
    rq = oracle.bwd_dq_rows(x["q"], x["k"], x["v"], x["dout"], w.scale, w.causal, rows)
    dq_s = G.f64(dq).reshape(-1, d)[rows]
    # relative to the largest reference entry over the sampled rows
    G.assert_grad(dq_s, rq, "dQ (sampled rows)")
    for what, keys in (("keys near the end", G.sample_keys_cheap(w, kv_heads=(0, w.Hkv - 1))),
                       ("heaviest keys", G.sample_keys_heavy(w, kv_heads=(0, w.Hkv - 1)))):
        rk, rv = oracle.bwd_dkv_rows(x["q"], x["k"], x["v"], x["dout"], w.scale, w.causal, keys)
        G.assert_grad(G.f64(dk).reshape(-1, d)[keys], rk, f"dK ({what})")
        G.assert_grad(G.f64(dv).reshape(-1, d)[keys], rv, f"dV ({what})")
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()
    # dV column sums: every P row sums to one
    want = x["dout"].double().reshape(w.B, w.Hkv, w.G, w.Nq, d).sum(dim=(2, 3))
    got = dv.double().cpu().sum(dim=2)
    err = (got - want).abs().max().item()
    assert err <= 1e-2 * want.abs().max().item() + 0.05 * np.sqrt(w.Nk), err


def test_backward_with_caller_workspace_matches():
    w = synth.WORKLOADS["mha_1k"].with_(B=1, Hq=4, Hkv=2)
    x = synth.make_inputs(w)
    xd = G.to_gpu(x)
    o, lse = G.gpu_forward(xd, w)
    n = fa.fa_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    g1 = fa.fa_bwd(xd["q"], xd["k"], xd["v"], o, xd["dout"], lse, causal=True, workspace=ws)
    g2 = fa.fa_bwd(xd["q"], xd["k"], xd["v"], o, xd["dout"], lse, causal=True)
    torch.cuda.synchronize()
    # dK, dV have no atomics: identical; dQ sums in a different order at most
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
    assert (g1[0].float() - g2[0].float()).abs().max().item() <= 1e-2
