"""GPU parity for head dims other than 64 and 128 against the oracle: 32 and 96
(on the 64 and 128 kernels with the missing columns zero-filled by TMA) and
160 .. 256 (the one-tile forward kernel and the feature-split d = 256
backward, whose two CTAs per key block each own half of dK, dV and dQ);
forward and backward.  Tails around the tiles, GQA, causal and not."""
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
    (1, 2, 1, 1, 1, 32, False),
    (1, 2, 1, 63, 63, 32, True),
    (2, 4, 2, 257, 257, 32, True),
    (1, 2, 2, 200, 333, 32, False),
    (1, 2, 1, 65, 65, 96, True),
    (1, 4, 2, 300, 300, 96, True),
    (1, 2, 2, 333, 200, 96, True),
    (1, 8, 1, 70, 640, 96, False),
    (2, 2, 2, 513, 513, 96, True),
    (1, 2, 1, 1, 1, 256, False),
    (1, 2, 1, 63, 63, 256, True),
    (2, 2, 1, 129, 129, 256, True),
    (1, 4, 2, 300, 300, 256, True),
    (1, 2, 2, 333, 200, 256, True),     # rows that see no key
    (1, 2, 2, 200, 333, 256, False),
    (1, 8, 1, 70, 640, 256, False),
    (1, 4, 1, 257, 257, 192, True),
    (1, 2, 2, 130, 130, 160, False),
    (1, 4, 4, 128, 128, 224, True),
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
    G.assert_o(G.f64(o), o_ref, o_abs=G.o_abs_ref(xr["q"], xr["k"], xr["v"], w.scale, causal))
    G.assert_lse(G.f64(lse), lse_ref)
    rq, rk, rv = oracle.bwd(xr["q"], xr["k"], xr["v"], xr["dout"], w.scale, causal)
    G.assert_grad(G.f64(dq), rq, "dQ")
    G.assert_grad(G.f64(dk), rk, "dK")
    G.assert_grad(G.f64(dv), rv, "dV")


FWD_ONLY = [
    # B, Hq, Hkv, Nq, Nk, d, causal
    (1, 2, 1, 1, 1, 256, False),
    (1, 2, 1, 63, 63, 256, True),
    (2, 2, 1, 129, 129, 256, True),
    (1, 4, 2, 300, 300, 256, True),
    (1, 2, 2, 333, 200, 256, True),     # rows that see no key
    (1, 2, 2, 200, 333, 256, False),
    (1, 8, 1, 70, 640, 256, False),
    (1, 4, 1, 257, 257, 192, True),
    (1, 2, 2, 130, 130, 160, False),
]


@pytest.mark.parametrize("dtype", DTYPES, ids=["bf16", "fp16"])
@pytest.mark.parametrize("shape", FWD_ONLY, ids=[str(s) for s in FWD_ONLY])
def test_large_headdim_forward(shape, dtype):
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    w = synth.Workload("headdim_fwd", B, Hq, Hkv, Nq, Nk, d, causal, 6400 + FWD_ONLY.index(shape))
    x = synth.make_inputs(w, dtype=dtype, dout=False)
    xd = {k: v.cuda() for k, v in x.items()}
    o = torch.full_like(xd["q"], float("nan"))
    o, lse = fa.fa_fwd(xd["q"], xd["k"], xd["v"], o=o, causal=causal)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    xr = {k: v.double() for k, v in x.items()}
    o_ref, lse_ref = oracle.fwd(xr["q"], xr["k"], xr["v"], w.scale, causal)
    G.assert_o(G.f64(o), o_ref, o_abs=G.o_abs_ref(xr["q"], xr["k"], xr["v"], w.scale, causal))
    G.assert_lse(G.f64(lse), lse_ref)


def test_large_headdim_sampled_long():
    """d = 256, N = 4096 causal GQA: sampled rows of a multi-wave launch, and
    the backward on sampled query rows (dQ) and on the heaviest and the last
    keys (dK, dV) of the first and last kv heads."""
    w = synth.Workload("headdim_long", 1, 16, 4, 4096, 4096, 256, True, 6450)
    x = synth.make_inputs(w)
    xd = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fa_fwd(xd["q"], xd["k"], xd["v"], causal=True)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    rows = G.sample_rows(w, n_random=24)
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, True, rows=rows)
    G.assert_o(G.f64(o).reshape(-1, w.d)[rows], o_ref,
               o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, True, rows=rows))
    G.assert_lse(G.f64(lse).reshape(-1)[rows], lse_ref)
    dq, dk, dv = G.gpu_backward(xd, o, lse, w)
    rq = oracle.bwd_dq_rows(x["q"], x["k"], x["v"], x["dout"], w.scale, True, rows)
    G.assert_grad(G.f64(dq).reshape(-1, w.d)[rows], rq, "dQ (sampled rows)")
    keys = np.concatenate([G.sample_keys_heavy(w, kv_heads=(0, w.Hkv - 1)),
                           G.sample_keys_cheap(w, kv_heads=(0, w.Hkv - 1))])
    rk, rv = oracle.bwd_dkv_rows(x["q"], x["k"], x["v"], x["dout"], w.scale, True, keys)
    G.assert_grad(G.f64(dk).reshape(-1, w.d)[keys], rk, "dK (sampled keys)")
    G.assert_grad(G.f64(dv).reshape(-1, w.d)[keys], rv, "dV (sampled keys)")


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_forward_rescale_every_block(d, causal):
    """Scores that climb by 6 (natural-log units, 8.7 in log2) from each 128-key
    block to the next: every block's row max passes the lazy-rescale threshold,
    so O is rescaled at every block.  At d = 256 (two S buffers, S(j) issued
    ahead of P.V(j - 1)) each rescale first waits for the previous block's P.V;
    d = 128 (two query tiles) is the control."""
    B, Hq, Hkv, N = 1, 2, 1, 1024
    scale = 1.0 / d ** 0.5
    g = torch.Generator().manual_seed(20261203 + d + int(causal))
    q = 0.1 * torch.randn(B, Hq, N, d, generator=g)
    q[..., 0] = 1.0
    k = torch.randn(B, Hkv, N, d, generator=g)
    k[..., 0] = (6.0 / scale) * (torch.arange(N) // 128).float()   # s ~ 6 j on key block j
    v = torch.randn(B, Hkv, N, d, generator=g)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    o, lse = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    o_ref, lse_ref = oracle.fwd(q, k, v, scale, causal)
    G.assert_o(G.f64(o), o_ref, o_abs=G.o_abs_ref(q, k, v, scale, causal))
    G.assert_lse(G.f64(lse), lse_ref)


def test_large_headdim_bench_shape():
    """The step workload's shape at head size 256 as the benchmark times it (B=1,
    Hq=32, Hkv=8, N=8192, causal; the feature-split backward walks 512 steps per
    CTA of key block 0): forward on sampled rows, dQ on sampled rows, dK / dV on
    the heaviest and the last keys of the first and last kv heads, and the dV
    column-sum identity."""
    w = synth.WORKLOADS["gqa_8k"].with_(name="gqa_8k_d256", d=256)
    x = synth.make_inputs(w)
    xd = G.to_gpu(x)
    o, lse = G.gpu_forward(xd, w)
    rows = G.sample_rows(w, n_random=16)
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, True, rows=rows)
    G.assert_o(G.f64(o).reshape(-1, w.d)[rows], o_ref,
               o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, True, rows=rows))
    G.assert_lse(G.f64(lse).reshape(-1)[rows], lse_ref)
    dq, dk, dv = G.gpu_backward(xd, o, lse, w)
    rq = oracle.bwd_dq_rows(x["q"], x["k"], x["v"], x["dout"], w.scale, True, rows)
    G.assert_grad(G.f64(dq).reshape(-1, w.d)[rows], rq, "dQ (sampled rows)")
    keys = np.concatenate([G.sample_keys_heavy(w, kv_heads=(0, w.Hkv - 1)),
                           G.sample_keys_cheap(w, kv_heads=(0, w.Hkv - 1))])
    rk, rv = oracle.bwd_dkv_rows(x["q"], x["k"], x["v"], x["dout"], w.scale, True, keys)
    G.assert_grad(G.f64(dk).reshape(-1, w.d)[keys], rk, "dK (sampled keys)")
    G.assert_grad(G.f64(dv).reshape(-1, w.d)[keys], rv, "dV (sampled keys)")
    want = x["dout"].double().reshape(w.B, w.Hkv, w.G, w.Nq, w.d).sum(dim=(2, 3))
    got = dv.double().cpu().sum(dim=2)
    err = (got - want).abs().max().item()
    assert err <= 1e-2 * want.abs().max().item() + 0.05 * np.sqrt(w.Nk), err


LONG_256 = [
    # B, Hq, Hkv, Nq, Nk, causal, dtype
    (1, 8, 2, 2048, 2048, False, torch.bfloat16),   # every query block for every key block
    (1, 8, 4, 2048, 2048, True, torch.float16),
    (1, 4, 1, 1000, 3000, True, torch.bfloat16),     # bottom-right mask, Nq < Nk
    (1, 4, 2, 2500, 700, True, torch.bfloat16),      # Nq > Nk: early rows see no key
]


@pytest.mark.parametrize("shape", LONG_256, ids=[f"{s[:6]}-{'fp16' if s[6] == torch.float16 else 'bf16'}"
                                                 for s in LONG_256])
def test_large_headdim_long_variants(shape):
    """d = 256 forward and backward at multi-wave sizes beyond the causal,
    square bf16 cases: non-causal (every step slot and both feature halves
    over all query blocks), fp16, and Nq != Nk with the bottom-right mask.
    Sampled query rows (O, LSE, dQ) and the heaviest and last keys (dK, dV)."""
    B, Hq, Hkv, Nq, Nk, causal, dtype = shape
    w = synth.Workload("headdim_long_v", B, Hq, Hkv, Nq, Nk, 256, causal, 6460 + Nq + Nk)
    x = synth.make_inputs(w, dtype=dtype)
    xd = G.to_gpu(x)
    o, lse = G.gpu_forward(xd, w)
    rows = G.sample_rows(w, n_random=12)
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, causal, rows=rows)
    G.assert_o(G.f64(o).reshape(-1, w.d)[rows], o_ref,
               o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, causal, rows=rows))
    G.assert_lse(G.f64(lse).reshape(-1)[rows], lse_ref)
    dq, dk, dv = G.gpu_backward(xd, o, lse, w)
    rq = oracle.bwd_dq_rows(x["q"], x["k"], x["v"], x["dout"], w.scale, causal, rows)
    G.assert_grad(G.f64(dq).reshape(-1, w.d)[rows], rq, "dQ (sampled rows)")
    keys = np.concatenate([G.sample_keys_heavy(w, kv_heads=(0, w.Hkv - 1)),
                           G.sample_keys_cheap(w, kv_heads=(0, w.Hkv - 1))])
    rk, rv = oracle.bwd_dkv_rows(x["q"], x["k"], x["v"], x["dout"], w.scale, causal, keys)
    G.assert_grad(G.f64(dk).reshape(-1, w.d)[keys], rk, "dK (sampled keys)")
    G.assert_grad(G.f64(dv).reshape(-1, w.d)[keys], rv, "dV (sampled keys)")
