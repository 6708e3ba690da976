"""CPU checks of the per-element O bound the GPU parity tests use,
max(1e-2, half a bf16 ulp of O_ref + 2^-9 sum_j P_j |v_j| + 2e-3).

The kernels round P to bf16 as the operand of the P.V product and divide by the
row sum of the unrounded P, then round O to bf16.  Modelled here in fp64 on
small rows: that arithmetic can miss 1e-2 for |O| in [2, 4), and it always stays
inside the bound; and the bound's sum_j P_j |v_j| is the oracle's forward with
|V| in place of V."""
import numpy as np
import torch

import oracle
from tests import gpu_parity as G


def bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def kernel_like_row(s, v):
    """O of one row as the kernels form it: p = exp(s - max s); numerator with p
    rounded to bf16, denominator with p unrounded; the result rounded to bf16."""
    p = np.exp(s - s.max())
    return bf16((bf16(p)[:, None] * v).sum(0) / p.sum())


def exact_row(s, v):
    p = np.exp(s - s.max())
    return (p[:, None] * v).sum(0) / p.sum(), (p[:, None] * np.abs(v)).sum(0) / p.sum()


def test_one_percent_alone_can_be_missed_and_the_bound_holds():
    # rows of one to three keys whose values all lie in 2.5 .. 4 in magnitude
    # (|O| in [2, 4), where a bf16 ulp is 2^-6): the operand rounding (2^-9
    # relative per term) and the output rounding (half an ulp) add up past 1e-2
    # on some rows of this seeded draw
    worst = 0.0
    rng = np.random.default_rng(5)
    for _ in range(20000):
        n = int(rng.integers(1, 4))
        s = rng.normal(0.0, 1.0, n)
        v = rng.uniform(2.5, 3.99, (n, 4)) * rng.choice([-1.0, 1.0])
        o_gpu = kernel_like_row(s, v)
        o_ref, o_abs = exact_row(s, v)
        diff = np.abs(o_gpu - o_ref)
        bound = np.maximum(G.O_TOL, G.half_ulp_bf16(o_ref) + G.P_OPERAND_REL * o_abs + 2e-3)
        assert (diff <= bound).all()
        worst = max(worst, diff.max())
    assert worst > G.O_TOL, worst   # 1e-2 on its own is not attainable for this arithmetic


def test_abs_value_forward_is_the_weighted_absolute_sum():
    # sum_j P_j |v_j| from the oracle's forward with |V|: at least |O| everywhere,
    # and equal to O where every v_j >= 0
    rng = np.random.default_rng(11)
    q = torch.from_numpy(rng.normal(size=(1, 2, 7, 16))).to(torch.bfloat16)
    k = torch.from_numpy(rng.normal(size=(1, 1, 9, 16))).to(torch.bfloat16)
    v = torch.from_numpy(rng.normal(size=(1, 1, 9, 16))).to(torch.bfloat16)
    o_ref, _ = oracle.fwd(q, k, v, 0.25, True)
    o_abs = G.o_abs_ref(q, k, v, 0.25, True)()
    assert (o_abs >= np.abs(o_ref) - 1e-12).all()
    o_pos, _ = oracle.fwd(q, k, v.abs(), 0.25, True)
    assert np.array_equal(o_abs, o_pos)
