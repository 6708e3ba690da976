"""Forward calls in flight together on several streams.  The forward kernel is
persistent and its blocks claim tiles from a per-launch counter slot, which
the launch's last block sets back to zero; concurrent launches take different
slots.  A wrong slot, a missed reset or a shared counter would skip or repeat
tiles, so every output here is compared bit for bit with the same call run
alone (the forward is bitwise repeatable)."""
import pytest
import torch

import exact_attention_114_b200 as fa
import synth

pytestmark = pytest.mark.gpu

# (name, B, Hq, Hkv, Nq, Nk, d, causal, dtype): GQA, MHA, Nq != Nk, d = 64 / 256, fp16
CASES = [
    ("gqa_causal", 1, 16, 4, 1536, 1536, 128, True, torch.bfloat16),
    ("mha_noncausal", 2, 8, 8, 1000, 1000, 128, False, torch.bfloat16),
    ("append", 1, 8, 2, 300, 2100, 128, True, torch.bfloat16),
    ("d64", 2, 12, 4, 2048, 2048, 64, True, torch.bfloat16),
    ("d256", 1, 4, 4, 777, 777, 256, True, torch.bfloat16),
    ("fp16", 1, 16, 16, 1024, 1024, 128, True, torch.float16),
    ("group_rows", 2, 16, 4, 40, 3000, 128, True, torch.bfloat16),    # kv heads' rows share tiles, key split
    ("decode_d256", 4, 16, 4, 1, 4096, 256, False, torch.bfloat16),
]


def _inputs(i, case):
    name, B, Hq, Hkv, Nq, Nk, d, causal, dt = case
    w = synth.Workload(name, B, Hq, Hkv, Nq, Nk, d, causal, 7300 + i, backward=False)
    x = {k: v.cuda() for k, v in synth.make_inputs(w, dtype=dt, dout=False).items()}
    return w, x


def test_concurrent_streams_match_serial():
    probs = [_inputs(i, c) for i, c in enumerate(CASES)]
    ref = []
    for w, x in probs:
        o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=w.causal)
        torch.cuda.synchronize()
        ref.append((o.clone(), lse.clone()))
    streams = [torch.cuda.Stream() for _ in range(4)]
    rounds = 3
    # every (round, problem) call writes its own buffers, allocated up front
    outs = [[(torch.empty_like(x["q"]), torch.empty_like(ref[j][1])) for j, (w, x) in enumerate(probs)]
            for _ in range(rounds)]
    torch.cuda.synchronize()
    for r in range(rounds):
        for j, (w, x) in enumerate(probs):
            s = streams[(r + j) % len(streams)]
            o, lse = outs[r][j]
            fa.fa_fwd(x["q"], x["k"], x["v"], o, lse, causal=w.causal, stream=s)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    for r in range(rounds):
        for j, (w, _) in enumerate(probs):
            o, lse = outs[r][j]
            assert torch.equal(o, ref[j][0]), (w.name, r)
            assert torch.equal(lse, ref[j][1]), (w.name, r)


def test_many_launches_keep_counter_slots_consistent():
    """More launches than counter slots (256), alternating two shapes whose
    tile counts differ, then a check against the single-call result."""
    (w1, x1), (w2, x2) = _inputs(0, CASES[0]), _inputs(3, CASES[3])
    o1, l1 = fa.fa_fwd(x1["q"], x1["k"], x1["v"], causal=True)
    o2, l2 = fa.fa_fwd(x2["q"], x2["k"], x2["v"], causal=True)
    torch.cuda.synchronize()
    r1, r2 = o1.clone(), o2.clone()
    for _ in range(150):
        fa.fa_fwd(x1["q"], x1["k"], x1["v"], o1, l1, causal=True)
        fa.fa_fwd(x2["q"], x2["k"], x2["v"], o2, l2, causal=True)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    assert torch.equal(o1, r1) and torch.equal(o2, r2)


def test_slot_held_by_another_launch_is_reported_not_silent():
    """A launch whose counter slot is held by another launch (simulated by
    presetting the slot's owner tag through the test hook) must end in
    FA_ERR_SLOT_CONFLICT from fa_check_device_status, never FA_OK with skipped
    tiles; the check clears every slot, after which the same call, pinned to
    the same slot, again matches the result of a normal launch bit for bit."""
    # 16 tile pairs x 16 heads = 256 tiles > 148 SMs: blocks must claim tiles
    w = synth.Workload("slot", 1, 16, 4, 4096, 4096, 128, True, 7400, backward=False)
    x = {k: v.cuda() for k, v in synth.make_inputs(w, dout=False).items()}
    o_ref, l_ref = fa.fa_fwd(x["q"], x["k"], x["v"], causal=True)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    slot = 7
    try:
        fa.fa_testhook_tile_slot(slot, preset_owner=0xDEADBEEF)
        fa.fa_fwd(x["q"], x["k"], x["v"], causal=True)
        torch.cuda.synchronize()
        with pytest.raises(fa.FaError) as err:
            fa.fa_check_device_status()
        assert err.value.status == fa.FA_ERR_SLOT_CONFLICT
        # the check cleared the slots: a launch pinned to the same slot runs whole
        o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=True)
        torch.cuda.synchronize()
        fa.fa_check_device_status()
    finally:
        fa.fa_testhook_tile_slot(-1)
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    o2, l2 = fa.fa_fwd(x["q"], x["k"], x["v"], causal=True)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    assert torch.equal(o2, o_ref) and torch.equal(l2, l_ref)


# backward shapes whose units are shared by several CTAs (query split): each call's
# counters and fp32 partials live in its own workspace
BWD_CASES = [
    ("split8", 1, 4, 1, 2048, 2048, 128, True),
    ("split4_d256", 1, 2, 1, 2048, 2048, 256, True),
    ("split2_noncausal", 1, 1, 1, 2048, 2048, 64, False),
]


def test_concurrent_backward_streams_match_serial():
    probs = []
    for i, (name, B, Hq, Hkv, Nq, Nk, d, causal) in enumerate(BWD_CASES):
        w = synth.Workload(name, B, Hq, Hkv, Nq, Nk, d, causal, 7400 + i)
        x = {k: v.cuda() for k, v in synth.make_inputs(w).items()}
        o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=causal)
        probs.append((w, x, o, lse))
    ref = []
    for w, x, o, lse in probs:
        g = fa.fa_bwd(x["q"], x["k"], x["v"], o, x["dout"], lse, causal=w.causal)
        torch.cuda.synchronize()
        ref.append([t.clone() for t in g])
    streams = [torch.cuda.Stream() for _ in range(3)]
    rounds = 2
    outs = [[[torch.empty_like(t) for t in ref[j]] for j in range(len(probs))] for _ in range(rounds)]
    torch.cuda.synchronize()
    for r in range(rounds):
        for j, (w, x, o, lse) in enumerate(probs):
            fa.fa_bwd(x["q"], x["k"], x["v"], o, x["dout"], lse, *outs[r][j], causal=w.causal,
                      stream=streams[(r + j) % len(streams)])
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    for r in range(rounds):
        for j, (w, *_rest) in enumerate(probs):
            dq, dk, dv = outs[r][j]
            # dK / dV: fixed-order sums, bitwise; dQ: fp32 reductions in any order
            assert torch.equal(dk, ref[j][1]) and torch.equal(dv, ref[j][2]), (w.name, r)
            err = (dq.float() - ref[j][0].float()).abs().max().item()
            assert err <= 1e-2 * ref[j][0].float().abs().max().item(), (w.name, r, err)
