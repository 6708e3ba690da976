"""GPU parity of the backward's query split against the oracle.  Where there are
too few (key block, kv head) units to fill the SMs, or their count would leave a
last round of CTAs with most SMs idle, 2 to 8 CTAs share each unit's (query
head, query block) steps and the last of them adds the others' fp32 dK / dV
partials.  Each case checks every dQ / dK / dV element (sampled ones at the full
N = 8192 GQA size) and that dK / dV repeat bitwise from call to call (the
partials are added in a fixed order, whichever CTA finishes last)."""
import numpy as np
import pytest
import torch

import exact_attention_114_b200 as fa
import oracle
import synth
from tests import gpu_parity as G

pytestmark = pytest.mark.gpu

# B, Hq, Hkv, Nq, Nk, d, causal, the split a 148-SM device takes
SPLIT_SHAPES = [
    (1, 1, 1, 2048, 2048, 128, False, 2),
    (1, 1, 1, 2048, 2048, 64, True, 2),
    (1, 1, 1, 2048, 2048, 256, False, 2),
    (2, 4, 2, 1000, 1000, 128, True, 2),
    (1, 2, 1, 1536, 1536, 128, True, 3),
    (1, 4, 2, 1536, 1536, 64, False, 3),
    (1, 2, 1, 1536, 1536, 256, True, 3),
    (1, 2, 1, 2048, 2048, 128, False, 4),
    (1, 4, 1, 1000, 1000, 64, True, 4),
    (1, 2, 1, 2048, 2048, 256, True, 4),
    (1, 4, 1, 1000, 3000, 128, True, 4),   # bottom-right mask, Nq < Nk
    (1, 4, 1, 3000, 1000, 128, True, 4),   # Nq > Nk: the first rows see no key
    (1, 4, 1, 1536, 1536, 128, False, 6),
    (1, 4, 1, 1536, 1536, 256, True, 6),
    (1, 8, 1, 1000, 1000, 128, True, 8),
    (1, 4, 1, 2048, 2048, 64, False, 8),
    (1, 8, 1, 1000, 1000, 256, False, 8),
    (1, 4, 1, 3000, 1000, 128, False, 8),
]


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _run(w, x, dtype=torch.bfloat16, workspace=None):
    xd = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fa_fwd(xd["q"], xd["k"], xd["v"], causal=w.causal, scale=w.scale)
    g1 = fa.fa_bwd(xd["q"], xd["k"], xd["v"], o, xd["dout"], lse, causal=w.causal, scale=w.scale,
                   workspace=workspace)
    g2 = fa.fa_bwd(xd["q"], xd["k"], xd["v"], o, xd["dout"], lse, causal=w.causal, scale=w.scale,
                   workspace=workspace)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    return g1, g2


def _check_full(w, x, g):
    xr = {k: v.double() for k, v in x.items()}
    rq, rk, rv = oracle.bwd(xr["q"], xr["k"], xr["v"], xr["dout"], w.scale, w.causal)
    G.assert_grad(G.f64(g[0]), rq, "dQ")
    G.assert_grad(G.f64(g[1]), rk, "dK")
    G.assert_grad(G.f64(g[2]), rv, "dV")


@pytest.mark.parametrize("shape", SPLIT_SHAPES, ids=[str(s) for s in SPLIT_SHAPES])
def test_split_backward_full(shape):
    B, Hq, Hkv, Nq, Nk, d, causal, split = shape
    got = fa.fa_bwd_query_split(B, Hq, Hkv, Nq, Nk, d, causal)
    if _sms() == 148:
        assert got == split
    assert got >= 1
    w = synth.Workload("split", B, Hq, Hkv, Nq, Nk, d, causal, 9500 + SPLIT_SHAPES.index(shape))
    x = synth.make_inputs(w)
    g1, g2 = _run(w, x)
    _check_full(w, x, g1)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2]), "dK / dV not repeatable"


def test_split_backward_fp16():
    w = synth.Workload("split16", 1, 4, 1, 1536, 1536, 128, False, 9600)
    assert fa.fa_bwd_query_split(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal) > 1 or _sms() != 148
    x = synth.make_inputs(w, dtype=torch.float16)
    g1, g2 = _run(w, x)
    assert g1[1].dtype == torch.float16
    _check_full(w, x, g1)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])


def _unsplit_workspace_bytes(B, Hq, Nq, kd):
    """D and -LSE rows and the fp32 dQ accumulator, each 256-byte aligned: the
    workspace without room for the split's partials."""
    rows = B * Hq * ((Nq + 63) // 64 * 64)
    a = lambda n: (n + 255) // 256 * 256
    return 2 * a(rows * 4) + a(rows * kd * 4)


@pytest.mark.parametrize("causal", [False, True])
def test_small_workspace_runs_unsplit(causal):
    """A caller workspace with room for D, LSE and the accumulator but not for the
    partials runs the backward unsplit: still correct, and dK / dV differ from
    the split run only by the order of the fp32 sums."""
    w = synth.Workload("split_ws", 1, 4, 1, 2048, 2048, 128, causal, 9700 + int(causal))
    full = fa.fa_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d)
    small = _unsplit_workspace_bytes(w.B, w.Hq, w.Nq, 128)
    assert small < full
    x = synth.make_inputs(w)
    ws = torch.empty(small, dtype=torch.uint8, device="cuda")
    g_small, _ = _run(w, x, workspace=ws)
    _check_full(w, x, g_small)
    g_split, _ = _run(w, x)
    for a, b in zip(g_small, g_split):
        err = (a.float() - b.float()).abs().max().item()
        assert err <= 1e-2 * b.float().abs().max().item() + 1e-3, err


def test_split_gqa_8k_noncausal_sampled():
    """The N = 8192 GQA shape without a causal mask: 512 units split in two on a
    148-SM device.  dQ on sampled rows; dK / dV on the keys of the first two key
    blocks, the middle and the end of the first and last kv heads (every key sees
    all 4 x 8192 rows of its group); dV column sums; dK / dV repeat bitwise."""
    w = synth.WORKLOADS["gqa_8k"].with_(name="gqa_8k_noncausal", causal=False)
    if _sms() == 148:
        assert fa.fa_bwd_query_split(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal) == 2
    x = synth.make_inputs(w)
    (dq, dk, dv), g2 = _run(w, x)
    assert torch.equal(dk, g2[1]) and torch.equal(dv, g2[2])
    d = w.d
    rows = G.sample_rows(w, n_random=16)
    rq = oracle.bwd_dq_rows(x["q"], x["k"], x["v"], x["dout"], w.scale, w.causal, rows)
    G.assert_grad(G.f64(dq).reshape(-1, d)[rows], rq, "dQ (sampled rows)")
    keys = np.concatenate([G.sample_keys_heavy(w, kv_heads=(0, w.Hkv - 1)),
                           G.sample_keys_cheap(w, kv_heads=(w.Hkv - 1,))])
    rk, rv = oracle.bwd_dkv_rows(x["q"], x["k"], x["v"], x["dout"], w.scale, w.causal, keys)
    G.assert_grad(G.f64(dk).reshape(-1, d)[keys], rk, "dK (sampled keys)")
    G.assert_grad(G.f64(dv).reshape(-1, d)[keys], rv, "dV (sampled keys)")
    want = x["dout"].double().reshape(w.B, w.Hkv, w.G, w.Nq, d).sum(dim=(2, 3))
    got = dv.double().cpu().sum(dim=2)
    err = (got - want).abs().max().item()
    assert err <= 1e-2 * want.abs().max().item() + 0.05 * np.sqrt(w.Nk), err
