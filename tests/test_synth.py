"""CPU tests for the seeded input generator (no attention arithmetic here)."""
import numpy as np
import torch

import synth


def test_splitmix64_published_outputs():
    # SplitMix64 from state 0: the first outputs quoted with the reference
    # implementation of the generator (Vigna's splitmix64.c test values).
    assert synth.splitmix64_at(0, 0) == 0xE220A8397B1DCDAF
    assert synth.splitmix64_at(0, 1) == 0x6E789E6AA1B965F4
    assert synth.splitmix64_at(0, 2) == 0x06C45D188009454F


def test_counter_based_and_thread_independent():
    a = synth.normal_bf16_bits(7, 3, 300_001, nthreads=1)
    b = synth.normal_bf16_bits(7, 3, 300_001, nthreads=6)
    assert np.array_equal(a, b)
    c = synth.normal_bf16_bits(7, 3, 1000, nthreads=1)
    assert np.array_equal(a[:1000], c)
    assert not np.array_equal(a[:1000], synth.normal_bf16_bits(7, 4, 1000))


def test_bf16_is_round_to_nearest_even_of_f32():
    f = synth.normal_f32(11, 1, 100_000)
    b = synth.normal_bf16_bits(11, 1, 100_000)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(b, ref)


def test_moments_are_standard_normal():
    f = synth.normal_f32(5, 2, 2_000_000).astype(np.float64)
    assert abs(f.mean()) < 5e-3
    assert abs(f.var() - 1) < 5e-3
    assert abs(np.mean(f ** 4) - 3) < 3e-2  # kurtosis of N(0,1)


def test_workload_shapes_and_scaled_rows():
    w = synth.WORKLOADS["mha_4k_long"].with_(B=1, Hq=2, Hkv=2, Nq=130, Nk=130)
    x = synth.make_inputs(w)
    assert x["q"].shape == (1, 2, 130, 128) and x["k"].shape == (1, 2, 130, 128)
    plain = synth.make_inputs(w.with_(scaled_q_rows=False))
    rows = torch.arange(130) % 64 == 0
    assert torch.equal(x["q"][:, :, rows], plain["q"][:, :, rows] * 8)
    assert torch.equal(x["q"][:, :, ~rows], plain["q"][:, :, ~rows])
    assert torch.equal(x["k"], plain["k"])


def test_flop_rule():
    w = synth.WORKLOADS["gqa_8k"]
    assert w.fwd_flops() == 4 * 1 * 32 * 8192 * 8192 * 128 / 2
    assert w.bwd_flops() == 2.5 * w.fwd_flops()
