"""GPU parity: split-KV decode (split pass + LSE combine) against the oracle."""
import numpy as np
import pytest
import torch

import exact_attention_114_b200 as fa
import oracle
import synth
from tests import gpu_parity as G

pytestmark = pytest.mark.gpu

# B, Hq, Hkv, Nq, Nk, causal -- d = 128; R = Nq * Hq / Hkv rows per kv head <= 16
DEC_SHAPES = [
    (1, 1, 1, 1, 1, False),
    (2, 4, 1, 1, 63, False),
    (3, 32, 8, 1, 700, False),
    (2, 8, 8, 2, 517, True),
    (1, 4, 1, 4, 1000, True),     # R = 16
    (2, 16, 2, 2, 4099, True),    # R = 16, ragged tail
    (1, 2, 1, 3, 2, True),        # Nq > Nk: a row that sees no key
]


@pytest.mark.parametrize("shape", DEC_SHAPES, ids=[str(s) for s in DEC_SHAPES])
@pytest.mark.parametrize("splits", [0, 1, 3, 16])
def test_splitkv_shapes(shape, splits):
    B, Hq, Hkv, Nq, Nk, causal = shape
    w = synth.Workload("dec", B, Hq, Hkv, Nq, Nk, 128, causal, 8100 + DEC_SHAPES.index(shape),
                       backward=False)
    x = synth.make_inputs(w)
    xd = G.to_gpu(x)
    nbytes = fa.fa_fwd_splitkv_workspace_size(B, Hq, Hkv, Nq, Nk, 128, splits)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")
    o, lse = fa.fa_fwd_splitkv(xd["q"], xd["k"], xd["v"], causal=causal, num_splits=splits,
                               workspace=ws if nbytes else None)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, causal)
    G.assert_o(G.f64(o), o_ref, o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, causal))
    G.assert_lse(G.f64(lse), lse_ref)


def test_splitkv_allocating_path_matches_workspace_path():
    w = synth.WORKLOADS["gqa_decode"].with_(B=4)
    xd = G.to_gpu(synth.make_inputs(w))
    o1, l1 = fa.fa_fwd_splitkv(xd["q"], xd["k"], xd["v"], num_splits=4)
    n = fa.fa_fwd_splitkv_workspace_size(4, 32, 8, 1, 8192, 128, 4)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    o2, l2 = fa.fa_fwd_splitkv(xd["q"], xd["k"], xd["v"], num_splits=4, workspace=ws)
    o3, l3 = fa.fa_fwd(xd["q"], xd["k"], xd["v"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.allclose(o1.float(), o3.float(), atol=1e-2)


def test_decode_config_sampled():
    """The full decode workload (B=64, Hq=32, Hkv=8, Nk=8192) through fa_fwd,
    as the benchmark launches it; sampled rows against the oracle."""
    w = synth.WORKLOADS["gqa_decode"]
    x = synth.make_inputs(w)
    xd = G.to_gpu(x)
    o, lse = G.gpu_forward(xd, w)
    rows = G.sample_rows(w, n_random=200)
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, w.causal, rows=rows)
    G.assert_o(G.f64(o).reshape(-1, w.d)[rows], o_ref,
               o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, w.causal, rows=rows))
    G.assert_lse(G.f64(lse).reshape(-1)[rows], lse_ref)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


def test_decode_config_full_small_batch():
    w = synth.WORKLOADS["gqa_decode"].with_(B=2)
    G.check_forward_full(w)


# head dims below 128 on the split-KV kernels (columns past d are TMA zero fill and skipped)
NARROW = [
    # B, Hq, Hkv, Nq, Nk, d, causal
    (2, 8, 2, 1, 700, 64, False),
    (1, 4, 1, 4, 1000, 32, True),
    (2, 16, 2, 2, 517, 96, True),
    (1, 2, 1, 3, 2, 64, True),        # a row that sees no key
]


@pytest.mark.parametrize("shape", NARROW, ids=[str(s) for s in NARROW])
@pytest.mark.parametrize("splits", [0, 1, 5])
def test_splitkv_narrow_heads(shape, splits):
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    w = synth.Workload("dec_narrow", B, Hq, Hkv, Nq, Nk, d, causal, 8200 + NARROW.index(shape),
                       backward=False)
    x = synth.make_inputs(w)
    xd = G.to_gpu(x)
    o = torch.full_like(xd["q"], float("nan"))
    o, lse = fa.fa_fwd_splitkv(xd["q"], xd["k"], xd["v"], o=o, causal=causal, num_splits=splits)
    o2, lse2 = fa.fa_fwd(xd["q"], xd["k"], xd["v"], causal=causal)   # the same kernels via fa_fwd
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, causal)
    G.assert_o(G.f64(o), o_ref, o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, causal))
    G.assert_lse(G.f64(lse), lse_ref)
    G.assert_o(G.f64(o2), o_ref, o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, causal))
