"""Pins for the fp64 oracle: checks that tie it to something other than itself.

Each ``pin_*`` function raises AssertionError when the oracle in use disagrees
with a value the pages print, a closed form, an invariant of the mathematics or
central finite differences.  ``tests/test_oracle_pins.py`` runs them against the
built oracle, and ``tests/test_oracle_mutants.py`` runs them against copies with
a planted mistake to show each such mistake is caught.

Sources: "FlashAttention：为什么少搬数据，反而算得更快" §02 (the S/P/O table,
scale and causal mask present), §04 (worked example, recurrence, initial state),
§05 (backward by recomputation); "AI infra. 一层全看懂(五)Flash Attention" §四
(safe softmax); "FlashAttention技术原理详解" (MHA / MQA / GQA).
"""
from __future__ import annotations

import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            nums = [float(x) for x in val.split()]
            vals[key] = nums if len(nums) > 1 else nums[0]
    return vals


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, rtol=1e-12, atol=1e-12):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    ok = np.isclose(a, b, rtol=rtol, atol=atol) | ((a == b) & np.isinf(a))
    assert ok.all(), f"max diff {np.nanmax(np.abs(a - b))}"


# ----------------------------------------------------------------------------
# the worked example printed on the page (§04)
# ----------------------------------------------------------------------------
def pin_worked_example_recurrence():
    g = read_golden("online_softmax_worked_example.txt")
    s = np.log(np.array(g["exp_scores"]))
    v = np.array(g["values"])
    o, m, l, tr = oracle.online_row(s, v, int(g["block"]), trace=True)
    assert len(tr) == 2
    _close(tr[0]["l"], g["block1_l"])
    _close(tr[0]["U"][0], g["block1_U"])
    _close(tr[1]["l_rescaled"], g["block2_l_rescaled"])
    _close(tr[1]["U_rescaled"][0], g["block2_U_rescaled"])
    _close(math.exp(tr[0]["m"] - tr[1]["m"]), g["rescale_factor"])
    _close(tr[1]["l"], g["block2_l"])
    _close(tr[1]["U"][0], g["block2_U"])
    _close(o[0], g["output"])
    # whole row at once: one block of four
    o1, _, l1 = oracle.online_row(s, v, 4)
    _close(o1[0], g["output"])
    _close(l1, 2.5)  # exp(s - max) summed with max = ln 4: (1 + 2 + 4 + 3) / 4


def pin_worked_example_fp32():
    """fp32 recurrence reproduces the example within 4 ulp at every step."""
    g = read_golden("online_softmax_worked_example.txt")
    s = np.log(np.array(g["exp_scores"]))
    v = np.array(g["values"])
    o, m, l, tr = oracle.online_row(s, v, int(g["block"]), precision="f32", trace=True)

    def ulps(x, ref):
        return abs(np.float32(x) - np.float32(ref)) / np.spacing(np.float32(ref))

    for got, key in [(tr[0]["l"], "block1_l"), (tr[0]["U"][0], "block1_U"),
                     (tr[1]["l_rescaled"], "block2_l_rescaled"),
                     (tr[1]["U_rescaled"][0], "block2_U_rescaled"),
                     (tr[1]["l"], "block2_l"), (tr[1]["U"][0], "block2_U"), (o[0], "output")]:
        assert ulps(got, g[key]) <= 4, (key, got, g[key])


def pin_worked_example_attention():
    """The same row through the attention oracle: d = 4, q = e0, k_j = ln(x_j) e0,
    scale 1, one-hot values give the weights; scalar values give 29."""
    g = read_golden("online_softmax_worked_example.txt")
    x = np.array(g["exp_scores"])
    q = np.zeros((1, 1, 1, 4))
    q[..., 0] = 1.0
    k = np.zeros((1, 1, 4, 4))
    k[0, 0, :, 0] = np.log(x)
    v = np.eye(4).reshape(1, 1, 4, 4)
    o, lse = oracle.fwd(q, k, v, 1.0, False)
    _close(o[0, 0, 0], g["weights"])
    _close(lse[0, 0, 0], math.log(x.sum()))
    v2 = np.zeros((1, 1, 4, 4))
    v2[0, 0, :, 0] = g["values"]
    o2, _ = oracle.fwd(q, k, v2, 1.0, False)
    _close(o2[0, 0, 0, 0], g["output"])


# ----------------------------------------------------------------------------
# closed forms
# ----------------------------------------------------------------------------
def pin_equal_scores_mean():
    """Q = 0: every visible score is 0, so O_i is the mean of the visible V rows
    and LSE_i = ln(#visible).  With V_j = j the mean is (last visible)/2, which
    also pins the bottom-right causal boundary j <= i + Nk - Nq."""
    for Nq, Nk, causal in [(6, 6, True), (4, 9, True), (5, 5, False), (3, 8, False)]:
        q = np.zeros((1, 1, Nq, 2))
        k = _rng(1).standard_normal((1, 1, Nk, 2))
        v = np.zeros((1, 1, Nk, 2))
        v[0, 0, :, 0] = np.arange(Nk)
        v[0, 0, :, 1] = 1.0
        o, lse = oracle.fwd(q, k, v, 0.7, causal)
        for i in range(Nq):
            last = i + Nk - Nq if causal else Nk - 1
            n = last + 1
            _close(o[0, 0, i, 0], last / 2.0)
            _close(o[0, 0, i, 1], 1.0)
            _close(lse[0, 0, i], math.log(n))


def pin_single_key():
    rng = _rng(2)
    q = rng.standard_normal((2, 3, 5, 4))
    k = rng.standard_normal((2, 3, 1, 4))
    v = rng.standard_normal((2, 3, 1, 4))
    sc = 0.37
    o, lse = oracle.fwd(q, k, v, sc, False)
    for b in range(2):
        for h in range(3):
            for i in range(5):
                _close(o[b, h, i], v[b, h, 0])
                _close(lse[b, h, i], sc * float(q[b, h, i] @ k[b, h, 0]))


def pin_causal_row0():
    rng = _rng(3)
    q = rng.standard_normal((1, 2, 7, 5))
    k = rng.standard_normal((1, 2, 7, 5))
    v = rng.standard_normal((1, 2, 7, 5))
    o, lse = oracle.fwd(q, k, v, 0.5, True)
    for h in range(2):
        _close(o[0, h, 0], v[0, h, 0])
        _close(lse[0, h, 0], 0.5 * float(q[0, h, 0] @ k[0, h, 0]))


def pin_two_key_logistic():
    """q = (1, 0), k = (2, 0), (0, 0), scale 1/2: scores (1, 0), so the weights are
    e/(1+e) and 1/(1+e) and LSE = ln(1 + e)."""
    q = np.array([1.0, 0.0]).reshape(1, 1, 1, 2)
    k = np.array([[2.0, 0.0], [0.0, 0.0]]).reshape(1, 1, 2, 2)
    v = np.array([[3.0, -1.0], [5.0, 7.0]]).reshape(1, 1, 2, 2)
    o, lse = oracle.fwd(q, k, v, 0.5, False)
    e = math.e
    w0, w1 = e / (1 + e), 1 / (1 + e)
    _close(o[0, 0, 0], [3 * w0 + 5 * w1, -1 * w0 + 7 * w1])
    _close(lse[0, 0, 0], math.log(1 + e))


def pin_shift_keys():
    """Adding one vector c to every key leaves O unchanged and adds scale q_i.c
    to LSE_i (non-causal and causal)."""
    rng = _rng(4)
    q = rng.standard_normal((1, 2, 6, 3))
    k = rng.standard_normal((1, 2, 8, 3))
    v = rng.standard_normal((1, 2, 8, 3))
    c = np.array([0.3, -1.1, 0.8])
    for causal in (False, True):
        o1, l1 = oracle.fwd(q, k, v, 0.6, causal)
        o2, l2 = oracle.fwd(q, k + c, v, 0.6, causal)
        _close(o1, o2, rtol=1e-11, atol=1e-12)
        _close(l2 - l1, 0.6 * (q @ c))


def pin_permutation():
    rng = _rng(5)
    q = rng.standard_normal((1, 1, 4, 3))
    k = rng.standard_normal((1, 1, 9, 3))
    v = rng.standard_normal((1, 1, 9, 3))
    perm = rng.permutation(9)
    o1, l1 = oracle.fwd(q, k, v, 0.8, False)
    o2, l2 = oracle.fwd(q, k[:, :, perm], v[:, :, perm], 0.8, False)
    _close(o1, o2, rtol=1e-11, atol=1e-12)
    _close(l1, l2, rtol=1e-12, atol=1e-12)


def pin_gqa_grouping():
    """Hq = 4, Hkv = 2: query heads 0, 1 use kv head 0 and heads 2, 3 use kv head 1
    (contiguous groups).  Constant V rows make the head mapping visible."""
    rng = _rng(6)
    q = rng.standard_normal((1, 4, 3, 2))
    k = rng.standard_normal((1, 2, 5, 2))
    v = np.zeros((1, 2, 5, 2))
    v[0, 0] = 1.0
    v[0, 1] = -1.0
    o, _ = oracle.fwd(q, k, v, 1.0, False)
    _close(o[0, 0], np.ones((3, 2)))
    _close(o[0, 1], np.ones((3, 2)))
    _close(o[0, 2], -np.ones((3, 2)))
    _close(o[0, 3], -np.ones((3, 2)))


def pin_fully_masked_rows():
    """Causal with Nq > Nk: rows i < Nq - Nk see no key; O = 0, LSE = -inf and
    their gradients are 0; no NaN anywhere."""
    rng = _rng(7)
    q = rng.standard_normal((1, 1, 7, 3))
    k = rng.standard_normal((1, 1, 4, 3))
    v = rng.standard_normal((1, 1, 4, 3))
    do = rng.standard_normal((1, 1, 7, 3))
    o, lse = oracle.fwd(q, k, v, 0.5, True)
    assert np.all(o[0, 0, :3] == 0.0)
    assert np.all(np.isneginf(lse[0, 0, :3]))
    assert np.all(np.isfinite(lse[0, 0, 3:]))
    _close(o[0, 0, 3], v[0, 0, 0])  # first row with a visible key sees key 0 only
    dq, dk, dv = oracle.bwd(q, k, v, do, 0.5, True)
    assert np.all(dq[0, 0, :3] == 0.0)
    assert np.isfinite(dq).all() and np.isfinite(dk).all() and np.isfinite(dv).all()


# ----------------------------------------------------------------------------
# invariant: blocked online softmax equals the full softmax (§04, §08)
# ----------------------------------------------------------------------------
def pin_blocked_equals_full():
    rng = _rng(8)
    n, dv = 23, 5
    s = rng.standard_normal(n) * 3.0
    s[[2, 9]] = -np.inf  # masked positions
    v = rng.standard_normal((n, dv))
    # the full answer from the attention oracle: q = e0 and k_j = s_j e0 give the
    # scores s_j; a masked position gets a huge negative score (its exp is 0)
    q = np.zeros((1, 1, 1, dv))
    q[..., 0] = 1.0
    k = np.zeros((1, 1, n, dv))
    k[0, 0, :, 0] = np.where(np.isinf(s), -1e300, s)
    o_full, lse_full = oracle.fwd(q, k, v.reshape(1, 1, n, dv), 1.0, False)
    for block in range(1, n + 1):
        o, m, l = oracle.online_row(s, v, block)
        _close(o, o_full[0, 0, 0], rtol=1e-12, atol=1e-13)
        _close(m + math.log(l), lse_full[0, 0, 0], rtol=1e-13, atol=1e-13)


def pin_lse_merge():
    """Merging per-part (O_s, lse_s) over a partition of the keys reproduces the
    whole row (the rescale-and-add rule of §04 in log form)."""
    rng = _rng(9)
    Nk, d = 29, 4
    q = rng.standard_normal((1, 1, 1, d))
    k = rng.standard_normal((1, 1, Nk, d)) * 2
    v = rng.standard_normal((1, 1, Nk, d))
    o_full, lse_full = oracle.fwd(q, k, v, 0.9, False)
    for cuts in ([0, 29], [0, 10, 29], [0, 1, 2, 17, 29], [0, 7, 14, 21, 28, 29]):
        parts_o, parts_l = [], []
        for a, b in zip(cuts[:-1], cuts[1:]):
            o_s, l_s = oracle.fwd(q, k[:, :, a:b], v[:, :, a:b], 0.9, False)
            parts_o.append(o_s[0, 0, 0])
            parts_l.append(l_s[0, 0, 0])
        o, lse = oracle.lse_merge(np.array(parts_o), np.array(parts_l))
        _close(o, o_full[0, 0, 0], rtol=1e-12, atol=1e-13)
        _close(lse, lse_full[0, 0, 0])
    # a part with no visible key (lse = -inf) contributes nothing
    o, lse = oracle.lse_merge(np.vstack([o_full[0, 0, 0], np.full(d, 123.0)]),
                              np.array([lse_full[0, 0, 0], -np.inf]))
    _close(o, o_full[0, 0, 0])
    _close(lse, lse_full[0, 0, 0])


# ----------------------------------------------------------------------------
# backward: central finite differences and invariants
# ----------------------------------------------------------------------------
def _loss(q, k, v, do, scale, causal):
    o, _ = oracle.fwd(q, k, v, scale, causal)
    return float(np.sum(o * do))


def _fd_grad(x, f, h=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        old = x[idx]
        x[idx] = old + h
        fp = f()
        x[idx] = old - h
        fm = f()
        x[idx] = old
        g[idx] = (fp - fm) / (2 * h)
    return g


FD_CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal
    (1, 1, 1, 4, 4, 3, False),
    (1, 2, 1, 5, 7, 3, True),
    (2, 4, 2, 3, 3, 2, True),
    (1, 2, 2, 6, 3, 2, True),   # Nq > Nk: fully masked rows
    (1, 1, 1, 9, 9, 8, True),
]


def pin_backward_finite_differences(cases=FD_CASES):
    for ci, (B, Hq, Hkv, Nq, Nk, d, causal) in enumerate(cases):
        rng = _rng(100 + ci)
        q = rng.standard_normal((B, Hq, Nq, d))
        k = rng.standard_normal((B, Hkv, Nk, d))
        v = rng.standard_normal((B, Hkv, Nk, d))
        do = rng.standard_normal((B, Hq, Nq, d))
        sc = 0.6
        dq, dk, dv = oracle.bwd(q, k, v, do, sc, causal)
        f = lambda: _loss(q, k, v, do, sc, causal)  # noqa: E731
        for name, x, g in (("dq", q, dq), ("dk", k, dk), ("dv", v, dv)):
            num = _fd_grad(x, f)
            err = np.max(np.abs(num - g)) / max(1.0, np.max(np.abs(g)))
            assert err <= 1e-6, (ci, name, err)


def pin_backward_invariants():
    """Every P row sums to 1 and every dS row to 0, so per (b, kv head):
    sum_j dK_j = 0 and sum_j dV_j = sum of dO over the group's rows that see at
    least one key."""
    rng = _rng(11)
    for causal, Nq, Nk in ((False, 6, 9), (True, 8, 8), (True, 9, 5)):
        B, Hq, Hkv, d = 2, 4, 2, 3
        q = rng.standard_normal((B, Hq, Nq, d))
        k = rng.standard_normal((B, Hkv, Nk, d))
        v = rng.standard_normal((B, Hkv, Nk, d))
        do = rng.standard_normal((B, Hq, Nq, d))
        dq, dk, dv = oracle.bwd(q, k, v, do, 0.45, causal)
        _close(dk.sum(axis=2), np.zeros((B, Hkv, d)), atol=1e-12)
        G = Hq // Hkv
        seen = np.ones(Nq, bool)
        if causal:
            seen = np.arange(Nq) + (Nk - Nq) >= 0
        want = do[:, :, seen].sum(axis=2).reshape(B, Hkv, G, d).sum(axis=2)
        _close(dv.sum(axis=2), want, rtol=1e-12, atol=1e-12)


def pin_sampled_backward_matches_full():
    rng = _rng(12)
    B, Hq, Hkv, Nq, Nk, d = 2, 4, 2, 7, 10, 3
    for causal in (False, True):
        q = rng.standard_normal((B, Hq, Nq, d))
        k = rng.standard_normal((B, Hkv, Nk, d))
        v = rng.standard_normal((B, Hkv, Nk, d))
        do = rng.standard_normal((B, Hq, Nq, d))
        dq, dk, dv = oracle.bwd(q, k, v, do, 0.3, causal)
        rows = np.array([0, 5, 13, 27, B * Hq * Nq - 1])
        _close(oracle.bwd_dq_rows(q, k, v, do, 0.3, causal, rows), dq.reshape(-1, d)[rows],
               rtol=1e-12, atol=1e-13)
        keys = np.array([0, 3, 9, 11, B * Hkv * Nk - 1])
        dks, dvs = oracle.bwd_dkv_rows(q, k, v, do, 0.3, causal, keys)
        _close(dks, dk.reshape(-1, d)[keys], rtol=1e-11, atol=1e-13)
        _close(dvs, dv.reshape(-1, d)[keys], rtol=1e-11, atol=1e-13)
        o, lse = oracle.fwd(q, k, v, 0.3, causal)
        o_r, lse_r = oracle.fwd(q, k, v, 0.3, causal, rows=rows)
        _close(o_r, o.reshape(-1, d)[rows])
        _close(lse_r, lse.reshape(-1)[rows])


def pin_bf16_input_path():
    """bf16 bit patterns and their exact double values give identical results."""
    import torch
    rng = _rng(13)
    x = [torch.tensor(rng.standard_normal(s)).to(torch.bfloat16)
         for s in ((1, 2, 5, 4), (1, 1, 6, 4), (1, 1, 6, 4))]
    o1, l1 = oracle.fwd(*x, 0.5, True)
    o2, l2 = oracle.fwd(*[t.double() for t in x], 0.5, True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


# Values fixed by the definition of OCP FP8 E4M3 (bias 7, 3 mantissa bits,
# exponent field 0 subnormal with step 2^-9, 0x7F / 0xFF NaN, no infinities).
E4M3_TABLE = {
    0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x0F: 1.875 * 2.0 ** -6,
    0x30: 0.5, 0x38: 1.0, 0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x54: 12.0, 0x77: 240.0,
    0x78: 256.0, 0x7E: 448.0, 0x81: -(2.0 ** -9), 0xB8: -1.0, 0xC4: -3.0, 0xFE: -448.0,
}


def pin_e4m3_table():
    v = oracle.e4m3_to_f64(np.arange(256, dtype=np.uint8))
    for code, want in E4M3_TABLE.items():
        assert v[code] == want, (hex(code), v[code], want)
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert v[0x80] == 0.0 and np.signbit(v[0x80])
    assert np.isfinite(np.delete(v, [0x7F, 0xFF])).all()


def pin_e4m3_library_and_order():
    """All 256 codes agree with torch's float8_e4m3fn, the positive codes are
    strictly increasing and the negative ones mirror them."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    v = oracle.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    same = (v == ref) | (np.isnan(v) & np.isnan(ref))
    assert same.all(), np.nonzero(~same)[0][:8]
    pos = v[:0x7F]
    assert (np.diff(pos) > 0).all()
    assert np.array_equal(v[0x80:0xFF], -pos)


ALL_PINS = [
    pin_worked_example_recurrence,
    pin_worked_example_fp32,
    pin_worked_example_attention,
    pin_equal_scores_mean,
    pin_single_key,
    pin_causal_row0,
    pin_two_key_logistic,
    pin_shift_keys,
    pin_permutation,
    pin_gqa_grouping,
    pin_fully_masked_rows,
    pin_blocked_equals_full,
    pin_lse_merge,
    pin_backward_finite_differences,
    pin_backward_invariants,
    pin_sampled_backward_matches_full,
    pin_bf16_input_path,
    pin_e4m3_table,
    pin_e4m3_library_and_order,
]
