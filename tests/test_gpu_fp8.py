"""GPU checks of the e4m3 forward (fa_fwd_fp8) against the oracle run on the
dequantised inputs (code * descale, exact in fp64).

Tolerance, from the arithmetic of the kernel: S = Q K^T of e4m3 values is exact
in fp32 products with fp32 sums; P = 2^(x - m_ref) is rounded to e4m3 for the
P.V product while the row sum l keeps the fp32 P.  For a reference m_ref at
most 2^8 below the row max (the lazy rescale threshold) and P <= 2^8 < 448,
the rounding of one p is at most max(p / 16, 2^-10) on the scale where the row
max is 1, so per element
    |O - O_ref| <= sum_j max(p_j / 16, 2^-10) |v_j| / l   (+ bf16 rounding of O)
with p_j = exp(s_j - max s).  The test asserts this worst-case bound on every
element and, because a worst-case bound can hide a systematic mistake such as
a permuted P, also that the RMS error stays within twice the RMS of a model of
independent rounding errors: std(p rounding) <= max(p 2^-3, 2^-9) / sqrt(12).
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_114_b200 as fa
import oracle
import synth
from tests import gpu_parity as G

pytestmark = pytest.mark.gpu

DS = synth.FP8_DESCALE
SHAPES = [
    # B, Hq, Hkv, Nq, Nk, d, causal
    (1, 2, 1, 63, 63, 128, True),
    (2, 2, 1, 65, 65, 128, True),
    (1, 2, 2, 100, 37, 128, True),      # Nk not a multiple of 16: padded V^T rows
    (1, 4, 2, 300, 300, 128, True),
    (1, 2, 2, 333, 200, 128, True),     # rows that see no key
    (1, 4, 4, 200, 333, 128, True),
    (1, 8, 1, 70, 640, 128, False),
    (1, 2, 2, 513, 513, 128, False),
    (1, 4, 1, 1, 1000, 128, False),     # one query row: still the tiled kernel
    (2, 4, 2, 1000, 1000, 128, True),
    (1, 32, 8, 64, 4096, 128, True),    # group rows (a kv head's 4 query heads share tiles), key split
    (4, 32, 8, 1, 4096, 128, False),    # decode shape on the tiled kernel: group rows, key split
]


def dequant(x8, name):
    return oracle.e4m3_to_f64(x8) * DS[name]


def error_model(qd, kd, vd, scale, causal, rows):
    """Per sampled row: worst-case bound and independent-rounding variance of
    each output element (see the module docstring)."""
    B, Hq, Nq, d = qd.shape
    Hkv, Nk = kd.shape[1], kd.shape[2]
    G_ = Hq // Hkv
    worst = np.zeros((len(rows), d))
    var = np.zeros((len(rows), d))
    for n, r in enumerate(rows):
        b, h, i = r // (Hq * Nq), (r // Nq) % Hq, r % Nq
        g = h // G_
        s = scale * (kd[b, g] @ qd[b, h, i])
        if causal:
            s[np.arange(Nk) > i + (Nk - Nq)] = -np.inf
        if np.isneginf(s).all():
            continue
        p = np.exp(s - s.max())
        l = p.sum()
        vis = p > 0
        err = np.where(vis, np.maximum(p / 16, 2.0 ** -10), 0.0)
        sig = np.where(vis, np.maximum(p * 2.0 ** -3, 2.0 ** -9), 0.0) / math.sqrt(12)
        worst[n] = err @ np.abs(vd[b, g]) / l
        var[n] = (sig ** 2) @ (vd[b, g] ** 2) / l ** 2
    return worst, var


def check(o_gpu, lse_gpu, o_ref, lse_ref, worst, var, vmax):
    assert np.isfinite(o_gpu).all()
    G.assert_lse(lse_gpu, lse_ref)
    err = np.abs(o_gpu - o_ref)
    lim = worst + 2.0 ** -8 * np.abs(o_ref) + 1e-4 * vmax
    bad = err > lim
    assert not bad.any(), f"{bad.sum()} elements over the bound; worst excess {np.max(err - lim):.3e}"
    rms = math.sqrt(np.mean(err ** 2))
    rms_model = math.sqrt(np.mean(var + (2.0 ** -9 * o_ref) ** 2 / 3))
    assert rms <= 2 * rms_model + 1e-7, f"RMS error {rms:.3e} > 2 x model {rms_model:.3e}"
    return rms, rms_model


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_fp8_forward(shape):
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    w = synth.Workload("fp8", B, Hq, Hkv, Nq, Nk, d, causal, 6500 + SHAPES.index(shape))
    x = synth.make_inputs_fp8(w)
    xd = {k: v.cuda() for k, v in x.items()}
    o = torch.full((B, Hq, Nq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    o, lse = fa.fa_fwd_fp8(xd["q"], xd["k"], xd["v"], DS["q"], DS["k"], DS["v"], o=o, causal=causal)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    qd, kd, vd = dequant(x["q"], "q"), dequant(x["k"], "k"), dequant(x["v"], "v")
    o_ref, lse_ref = oracle.fwd(qd, kd, vd, w.scale, causal)
    rows = np.arange(B * Hq * Nq)
    worst, var = error_model(qd, kd, vd, w.scale, causal, rows)
    check(G.f64(o).reshape(-1, d), G.f64(lse).reshape(-1), o_ref.reshape(-1, d), lse_ref.reshape(-1),
          worst, var, np.abs(vd).max())


def test_fp8_gqa_config_sampled():
    """The GQA N=8192 causal workload in e4m3, sampled rows, with a caller-owned
    workspace."""
    w = synth.WORKLOADS["gqa_8k"]
    x = synth.make_inputs_fp8(w)
    xd = {k: v.cuda() for k, v in x.items()}
    ws = torch.empty(fa.fa_fwd_fp8_workspace_size(w.B, w.Hkv, w.Nk, w.d), dtype=torch.uint8,
                     device="cuda")
    o, lse = fa.fa_fwd_fp8(xd["q"], xd["k"], xd["v"], DS["q"], DS["k"], DS["v"], causal=True,
                           workspace=ws)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    qd, kd, vd = dequant(x["q"], "q"), dequant(x["k"], "k"), dequant(x["v"], "v")
    rows = G.sample_rows(w, n_random=24)
    o_ref, lse_ref = oracle.fwd(qd, kd, vd, w.scale, True, rows=rows)
    worst, var = error_model(qd, kd, vd, w.scale, True, rows)
    check(G.f64(o).reshape(-1, w.d)[rows], G.f64(lse).reshape(-1)[rows], o_ref, lse_ref, worst, var,
          np.abs(vd).max())


def test_fp8_matches_bf16_path_closely():
    """Cross-check: the dequantised inputs rounded to bf16 through the bf16
    kernel give nearly the same O (RMS difference far below the output scale)."""
    w = synth.Workload("fp8_vs_bf16", 1, 4, 2, 384, 384, 128, True, 6600)
    x = synth.make_inputs_fp8(w)
    xd = {k: v.cuda() for k, v in x.items()}
    o8, _ = fa.fa_fwd_fp8(xd["q"], xd["k"], xd["v"], DS["q"], DS["k"], DS["v"], causal=True)
    qd, kd, vd = dequant(x["q"], "q"), dequant(x["k"], "k"), dequant(x["v"], "v")
    tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (qd, kd, vd))
    o16, _ = fa.fa_fwd(tq, tk, tv, causal=True)
    torch.cuda.synchronize()
    diff = np.abs(G.f64(o8) - G.f64(o16))
    assert np.sqrt(np.mean(diff ** 2)) < 2e-2
