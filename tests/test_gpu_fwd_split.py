"""GPU parity of the forward's key split against the oracle.  Where a tiled
forward has fewer work tiles (pairs of 128-row query tiles of one head) than the
GPU has SMs, each tile's key blocks are cut into contiguous shares that run as
separate tiles, and a second kernel merges their fp32 partials by their LSE.
Each case checks O and LSE (every row, or sampled rows at the long append
shapes) and that O repeats bitwise from call to call."""
import functools

import numpy as np
import pytest
import torch

import exact_attention_114_b200 as fa
import oracle
import synth
from tests import gpu_parity as G

pytestmark = pytest.mark.gpu

# B, Hq, Hkv, Nq, Nk, d, causal, the key shares a 148-SM device takes
FWD_SPLIT_SHAPES = [
    (1, 4, 1, 2048, 2048, 128, True, 4),
    (1, 4, 1, 2048, 2048, 128, False, 4),
    (1, 8, 2, 1000, 3000, 128, True, 4),     # bottom-right mask, Nq < Nk
    (1, 2, 1, 3000, 2000, 128, True, 6),     # Nq > Nk: the first rows see no key
    (2, 2, 1, 600, 4000, 128, True, 12),
    (1, 2, 1, 1000, 2000, 256, False, 8),    # one query tile per work tile
    (1, 2, 1, 1024, 8192, 256, True, 8),
    (1, 2, 1, 300, 5000, 64, True, 16),
    (1, 4, 1, 200, 4096, 128, False, 16),
    # decode shapes at d = 256 (beyond the split-KV decode kernels' 128) take the tiled path
    (1, 8, 2, 1, 8192, 256, True, 16),
    (2, 16, 4, 4, 16384, 256, True, 16),
    (2, 4, 4, 1, 5000, 256, False, 16),     # MHA decode at d = 256: one row per tile head, key split only
]


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _forward_twice(w, xd):
    o1, l1 = fa.fa_fwd(xd["q"], xd["k"], xd["v"], causal=w.causal, scale=w.scale)
    o2, l2 = fa.fa_fwd(xd["q"], xd["k"], xd["v"], causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    return o1, l1, o2, l2


@pytest.mark.parametrize("shape", FWD_SPLIT_SHAPES, ids=[str(s) for s in FWD_SPLIT_SHAPES])
def test_fwd_split_full(shape):
    B, Hq, Hkv, Nq, Nk, d, causal, shares = shape
    got = fa.fa_fwd_kv_split(B, Hq, Hkv, Nq, Nk, d, causal)
    if _sms() == 148:
        assert got == shares
    w = synth.Workload("fwd_split", B, Hq, Hkv, Nq, Nk, d, causal, 9800 + FWD_SPLIT_SHAPES.index(shape))
    x = synth.make_inputs(w, dout=False)
    xd = {k: v.cuda() for k, v in x.items()}
    o, lse, o2, l2 = _forward_twice(w, xd)
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, w.causal)
    G.assert_o(G.f64(o), o_ref, o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, w.causal))
    G.assert_lse(G.f64(lse), lse_ref)
    assert torch.equal(o, o2) and torch.equal(lse, l2), "O / LSE not repeatable"


def test_fwd_split_fp16_with_backward():
    """fp16 inputs through the split forward, and the backward on its O / LSE."""
    w = synth.Workload("fwd_split16", 1, 4, 1, 2048, 2048, 128, True, 9900)
    x = synth.make_inputs(w, dtype=torch.float16)
    xd = {k: v.cuda() for k, v in x.items()}
    o, lse, _, _ = _forward_twice(w, xd)
    assert o.dtype == torch.float16
    xr = {k: v.double() for k, v in x.items()}
    o_ref, lse_ref = oracle.fwd(xr["q"], xr["k"], xr["v"], w.scale, w.causal)
    G.assert_o(G.f64(o), o_ref, o_abs=G.o_abs_ref(xr["q"], xr["k"], xr["v"], w.scale, w.causal))
    G.assert_lse(G.f64(lse), lse_ref)
    dq, dk, dv = fa.fa_bwd(xd["q"], xd["k"], xd["v"], o, xd["dout"], lse, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    rq, rk, rv = oracle.bwd(xr["q"], xr["k"], xr["v"], xr["dout"], w.scale, w.causal)
    G.assert_grad(G.f64(dq), rq, "dQ")
    G.assert_grad(G.f64(dk), rk, "dK")
    G.assert_grad(G.f64(dv), rv, "dV")


APPEND_SHAPES = [
    # a 512-row chunk appended to a 32K context, and a 64-row one (GQA 32 / 8)
    (1, 32, 8, 512, 32768, 128, True, 2),
    (1, 32, 8, 64, 32768, 128, True, 16),
    # a 4096-row chunk: 512 equal units; the 68 after the last full round of 148 run in two
    # shares (a tail split), the others whole.  (A 2048-row one stays whole: with K and V
    # beyond L2 its 4-share tail gained nothing.)
    (1, 32, 8, 2048, 32768, 128, True, 1),
    (1, 32, 8, 4096, 32768, 128, True, 2),
]


@pytest.mark.parametrize("shape", APPEND_SHAPES, ids=[str(s) for s in APPEND_SHAPES])
def test_fwd_split_append_sampled(shape):
    B, Hq, Hkv, Nq, Nk, d, causal, shares = shape
    if _sms() == 148:
        assert fa.fa_fwd_kv_split(B, Hq, Hkv, Nq, Nk, d, causal) == shares
    w = synth.Workload("append", B, Hq, Hkv, Nq, Nk, d, causal, 9950 + APPEND_SHAPES.index(shape))
    x = synth.make_inputs(w, dout=False)
    xd = {k: v.cuda() for k, v in x.items()}
    o, lse, o2, _ = _forward_twice(w, xd)
    assert torch.equal(o, o2)
    rows = G.sample_rows(w, n_random=24)
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, w.causal, rows=rows)
    G.assert_o(G.f64(o).reshape(-1, d)[rows], o_ref,
               o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, w.causal, rows=rows))
    G.assert_lse(G.f64(lse).reshape(-1)[rows], lse_ref)


# Tail split: more units than SMs, with a last round that would leave most SMs idle; the
# first 148 units (claimed first, heaviest first) run whole and write o / lse directly, the
# rest run in shares merged by the merge kernel, which leaves the whole units' rows alone.
TAIL_SHAPES = [
    (1, 20, 4, 2048, 2048, 64, False, 8),
    (1, 40, 8, 1024, 3000, 64, True, 4),
    (2, 40, 8, 512, 3000, 64, True, 8),
    (1, 20, 4, 2048, 2048, 128, False, 8),
    (2, 20, 4, 1024, 3000, 128, True, 4),
    (1, 20, 4, 1024, 3000, 256, False, 12),
]


@pytest.mark.parametrize("shape", TAIL_SHAPES, ids=[str(s) for s in TAIL_SHAPES])
def test_fwd_tail_split_full(shape):
    B, Hq, Hkv, Nq, Nk, d, causal, shares = shape
    if _sms() == 148:
        assert fa.fa_fwd_kv_split(B, Hq, Hkv, Nq, Nk, d, causal) == shares
    w = synth.Workload("tail_split", B, Hq, Hkv, Nq, Nk, d, causal, 9850 + TAIL_SHAPES.index(shape))
    x = synth.make_inputs(w, dout=False)
    xd = {k: v.cuda() for k, v in x.items()}
    o, lse, o2, l2 = _forward_twice(w, xd)
    assert torch.equal(o, o2) and torch.equal(lse, l2)
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, w.causal)
    G.assert_o(G.f64(o), o_ref, o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, w.causal))
    G.assert_lse(G.f64(lse), lse_ref)


# Seeded random shapes on which the planner splits the keys: units (query-tile pairs x heads,
# Nq >= 300 so no group rows) at most the SM count, where every unit runs in shares, or beyond
# it, where the units after the last full round do (a tail split).  Drawn at run time (the
# plan depends on the device's SM count), within a budget the oracle finishes in about a
# second; every O and LSE element is compared.
@functools.lru_cache(maxsize=None)
def _draw_split_shapes(tail, n=6, seed=20261205):
    rng = np.random.default_rng(seed + int(tail))
    sms, out = _sms(), []
    for _ in range(20000):
        if len(out) == n:
            break
        d = int(rng.choice([64, 128]))
        Hkv = int(rng.choice([2, 4, 8] if tail else [1, 2, 4, 8]))
        G_ = int(rng.choice([2, 3, 4, 8] if tail else [1, 2, 4]))
        B = int(rng.integers(1, 3))
        Hq = Hkv * G_
        Nq = int(rng.integers(300, 2200 if tail else 2600))
        Nk = int(rng.integers(300, 3000 if tail else 4000))
        causal = bool(rng.integers(0, 2))
        units = B * Hq * ((Nq + 255) // 256)
        pairs = B * Hq * Nq * Nk * (0.5 if causal else 1.0)
        if (units > sms) != tail or pairs * d > 6e9:
            continue
        shares = fa.fa_fwd_kv_split(B, Hq, Hkv, Nq, Nk, d, causal)
        if shares > 1:
            out.append((B, Hq, Hkv, Nq, Nk, d, causal, shares))
    return tuple(out)


@pytest.mark.parametrize("tail", [False, True], ids=["every_unit", "tail"])
@pytest.mark.parametrize("i", range(6))
def test_fwd_split_random(tail, i):
    shapes = _draw_split_shapes(tail)
    if i >= len(shapes):
        pytest.skip(f"only {len(shapes)} split shapes drawn on this device")
    B, Hq, Hkv, Nq, Nk, d, causal, shares = shapes[i]
    w = synth.Workload("fwd_split_random", B, Hq, Hkv, Nq, Nk, d, causal, 9870 + 10 * int(tail) + i)
    dtype = torch.float16 if i % 3 == 2 else torch.bfloat16
    x = synth.make_inputs(w, dout=False, dtype=dtype)
    xd = {k: v.cuda() for k, v in x.items()}
    o, lse, o2, l2 = _forward_twice(w, xd)
    assert torch.equal(o, o2) and torch.equal(lse, l2)
    xr = {k: v.double() for k, v in x.items()}
    o_ref, lse_ref = oracle.fwd(xr["q"], xr["k"], xr["v"], w.scale, w.causal)
    G.assert_o(G.f64(o), o_ref, o_abs=G.o_abs_ref(xr["q"], xr["k"], xr["v"], w.scale, w.causal))
    G.assert_lse(G.f64(lse), lse_ref)


# Group rows: where a query head has fewer rows than a work tile (Nq < 256, or < 128 at
# d = 256) and a kv head serves G > 1 query heads, the G * Nq rows of its heads share
# the kv head's tiles (row r at query position r % Nq).  B, Hq, Hkv, Nq, Nk, d, causal
GROUP_ROW_SHAPES = [
    (64, 32, 8, 1, 8192, 256, False),    # d = 256 decode: 512 tiles, one per (batch, kv head)
    (2, 12, 4, 37, 500, 128, True),      # G = 3, bottom-right mask with Nq < Nk
    (1, 8, 2, 100, 100, 64, True),       # causal Nq = Nk: one tile mixes every query position
    (2, 6, 2, 90, 260, 256, True),
    (1, 4, 2, 200, 100, 128, True),      # Nq > Nk: positions below Nq - Nk see no key
    (2, 8, 4, 130, 60, 64, True),
    (3, 6, 2, 6, 700, 128, False),       # 18 rows per kv head: just past the decode kernels' 16
]


@pytest.mark.parametrize("shape", GROUP_ROW_SHAPES, ids=[str(s) for s in GROUP_ROW_SHAPES])
def test_group_rows_full(shape):
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    w = synth.Workload("group_rows", B, Hq, Hkv, Nq, Nk, d, causal, 9700 + GROUP_ROW_SHAPES.index(shape))
    x = synth.make_inputs(w, dout=False)
    xd = {k: v.cuda() for k, v in x.items()}
    o, lse, o2, _ = _forward_twice(w, xd)
    assert torch.equal(o, o2)
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, w.causal)
    G.assert_o(G.f64(o), o_ref, o_abs=G.o_abs_ref(x["q"], x["k"], x["v"], w.scale, w.causal))
    G.assert_lse(G.f64(lse), lse_ref)


def test_group_rows_fp16():
    w = synth.Workload("group_rows16", 1, 8, 2, 33, 2000, 128, False, 9790)
    x = synth.make_inputs(w, dout=False, dtype=torch.float16)
    xd = {k: v.cuda() for k, v in x.items()}
    o, lse, _, _ = _forward_twice(w, xd)
    xr = {k: v.double() for k, v in x.items()}
    o_ref, lse_ref = oracle.fwd(xr["q"], xr["k"], xr["v"], w.scale, w.causal)
    G.assert_o(G.f64(o), o_ref, o_abs=G.o_abs_ref(xr["q"], xr["k"], xr["v"], w.scale, w.causal))
    G.assert_lse(G.f64(lse), lse_ref)
