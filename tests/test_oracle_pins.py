"""CPU tests: the oracle against the pages' worked example, closed forms,
invariants and finite differences (see ``oracle_pins.py``), plus the fp32
two-block check on the tiny workload's rows."""
import math

import numpy as np
import pytest

import oracle
import synth
from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_fp32_two_block_check_tiny_workload():
    """For each of the 128 rows of the tiny workload (B=1, H=1, N=128, d=64),
    the fp32 online recurrence with two blocks of 64 matches the fp32 whole-row
    softmax to 1e-6 of the row's largest |O| entry, and both match fp64 (the
    oracle)."""
    w = synth.WORKLOADS["tiny_mha"]
    x = synth.make_inputs(w)
    q = x["q"][0, 0].double().numpy()
    k = x["k"][0, 0].double().numpy()
    v = x["v"][0, 0].double().numpy()
    o64, lse64 = oracle.fwd(x["q"], x["k"], x["v"], w.scale, w.causal)
    for i in range(w.Nq):
        s = w.scale * (k @ q[i])  # the row of scores fed to both recurrences
        ob, mb, lb = oracle.online_row(s, v, 64, precision="f32")
        of, mf, lf = oracle.full_row_f32(s, v)
        # relative to the row's largest output entry (entries near zero are sums
        # with cancellation, where an element-wise ratio says nothing)
        assert np.max(np.abs(ob - of)) <= 1e-6 * np.max(np.abs(of)), i
        assert abs((mb + math.log(lb)) - (mf + math.log(lf))) <= 1e-6
        assert np.max(np.abs(ob - o64[0, 0, i])) <= 1e-5
        assert abs(mb + math.log(lb) - lse64[0, 0, i]) <= 1e-5


def test_oracle_threads_do_not_change_results():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((2, 4, 33, 8))
    k = rng.standard_normal((2, 2, 41, 8))
    v = rng.standard_normal((2, 2, 41, 8))
    do = rng.standard_normal((2, 4, 33, 8))
    a = oracle.bwd(q, k, v, do, 0.4, True, nthreads=1)
    b = oracle.bwd(q, k, v, do, 0.4, True, nthreads=7)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    o1, l1 = oracle.fwd(q, k, v, 0.4, True, nthreads=1)
    o2, l2 = oracle.fwd(q, k, v, 0.4, True, nthreads=5)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
