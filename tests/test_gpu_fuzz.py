"""GPU parity on seeded random shapes: batch, heads, GQA ratio, query and key
lengths (Nq != Nk included, so some rows see no key), head dim, mask and 16-bit
type are drawn from a fixed generator, and every draw runs forward and
backward against the oracle.  Small sizes keep the oracle fast; the draws
include decode shapes (Nq x G <= 16, the split-KV kernels) and d > 128 (the
one-tile forward and the feature-split backward)."""
import numpy as np
import pytest
import torch

import exact_attention_114_b200 as fa
import oracle
import synth
from tests import gpu_parity as G

pytestmark = pytest.mark.gpu


def draw_cases(n=64, seed=20261202, max_len=600, seed0=7000):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        Hkv = int(rng.choice([1, 2, 4]))
        G_ = int(rng.choice([1, 2, 4, 8]))
        B = int(rng.integers(1, 3))
        d = int(rng.choice([32, 64, 96, 128, 128, 160, 256]))
        causal = bool(rng.integers(0, 2))
        if rng.random() < 0.25:            # decode / append shape
            Nq = int(rng.integers(1, max(2, 16 // G_) + 1))
        else:
            Nq = int(rng.integers(1, max_len))
        Nk = int(rng.integers(1, max_len + 100)) if rng.random() < 0.5 else Nq
        dtype = "fp16" if rng.random() < 0.3 else "bf16"
        cases.append((B, Hkv * G_, Hkv, Nq, Nk, d, causal, dtype, seed0 + i))
    return cases


# a first set of short shapes, and a second, independent set reaching further
# (several 64-row query blocks and 128-key blocks per CTA, head sizes up to 256
# in the backward too)
CASES = draw_cases() + draw_cases(n=64, seed=20261203, max_len=1100, seed0=7100)


@pytest.mark.parametrize("case", CASES, ids=[str(c[:8]) for c in CASES])
def test_fuzz_shape(case):
    B, Hq, Hkv, Nq, Nk, d, causal, dtype, seed = case
    w = synth.Workload("fuzz", B, Hq, Hkv, Nq, Nk, d, causal, seed)
    tdt = torch.float16 if dtype == "fp16" else torch.bfloat16
    x = synth.make_inputs(w, dtype=tdt)
    xd = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fa_fwd(xd["q"], xd["k"], xd["v"], causal=causal)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    xr = {k: v.double() for k, v in x.items()}
    o_ref, lse_ref = oracle.fwd(xr["q"], xr["k"], xr["v"], w.scale, causal)
    G.assert_o(G.f64(o), o_ref, o_abs=G.o_abs_ref(xr["q"], xr["k"], xr["v"], w.scale, causal))
    G.assert_lse(G.f64(lse), lse_ref)
    dq, dk, dv = fa.fa_bwd(xd["q"], xd["k"], xd["v"], o, xd["dout"], lse, causal=causal)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    rq, rk, rv = oracle.bwd(xr["q"], xr["k"], xr["v"], xr["dout"], w.scale, causal)
    G.assert_grad(G.f64(dq), rq, "dQ")
    G.assert_grad(G.f64(dk), rk, "dK")
    G.assert_grad(G.f64(dv), rv, "dV")
