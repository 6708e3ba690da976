"""GPU parity: decode over a paged KV cache (fa_fwd_paged) against the oracle.

The pool of pages is filled with seeded N(0,1) bf16 values and handed out to
the sequences in a random order; the test gathers each sequence's K/V back
into contiguous form (pure indexing) for the oracle."""
import numpy as np
import pytest
import torch

import exact_attention_114_b200 as fa
import oracle
import synth
from tests import gpu_parity as G

pytestmark = pytest.mark.gpu


def make_paged(B, Hq, Hkv, Nq, page_size, seq_lens, seed, extra_pages=3, d=128, fp16=False):
    rng = np.random.default_rng(seed)
    pages_per_seq = [max(1, -(-L // page_size)) for L in seq_lens]
    max_pages = max(pages_per_seq)
    num_pages = sum(pages_per_seq) + extra_pages
    perm = rng.permutation(num_pages)
    table = np.zeros((B, max_pages), np.int32)
    pos = 0
    for b, n in enumerate(pages_per_seq):
        table[b, :n] = perm[pos:pos + n]
        table[b, n:] = perm[pos]            # unused entries: any valid page
        pos += n
    n_pool = num_pages * page_size * Hkv * d

    def draw(tid, n, shape):
        if fp16:
            return torch.from_numpy(synth.normal_f32(seed, tid, n).astype(np.float16)).reshape(shape)
        bits = synth.normal_bf16_bits(seed, tid, n)
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).reshape(shape)

    k_pool = draw(synth.TENSOR_K, n_pool, (num_pages, page_size, Hkv, d))
    v_pool = draw(synth.TENSOR_V, n_pool, (num_pages, page_size, Hkv, d))
    q = draw(synth.TENSOR_Q, B * Hq * Nq * d, (B, Hq, Nq, d))
    return q, k_pool, v_pool, table, np.array(seq_lens, np.int32)


def gather(pool, table_row, L, page_size):
    """Keys 0..L-1 of one sequence as [1, Hkv, L, d]."""
    rows = [pool[table_row[j // page_size], j % page_size] for j in range(L)]
    return torch.stack(rows, 0).permute(1, 0, 2).unsqueeze(0).contiguous()


def run_case(B, Hq, Hkv, Nq, page_size, seq_lens, causal, splits, seed, d=128, fp16=False):
    q, kp, vp, table, lens = make_paged(B, Hq, Hkv, Nq, page_size, seq_lens, seed, d=d, fp16=fp16)
    dq, dk, dv = q.cuda(), kp.cuda(), vp.cuda()
    dt, dl = torch.from_numpy(table).cuda(), torch.from_numpy(lens).cuda()
    o, lse = fa.fa_fwd_paged(dq, dk, dv, dt, dl, causal=causal, num_splits=splits)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    scale = 1.0 / np.sqrt(d)
    for b, L in enumerate(seq_lens):
        og, lg = G.f64(o[b:b + 1]), G.f64(lse[b:b + 1])
        if L == 0:
            assert np.all(og == 0.0) and np.all(np.isneginf(lg))
            continue
        kb, vb = gather(kp, table[b], L, page_size), gather(vp, table[b], L, page_size)
        o_ref, lse_ref = oracle.fwd(q[b:b + 1], kb, vb, scale, causal)
        G.assert_o(og, o_ref, what=f"O (sequence {b}, {L} keys)",
                   o_abs=G.o_abs_ref(q[b:b + 1], kb, vb, scale, causal))
        G.assert_lse(lg, lse_ref)


PAGED_CASES = [
    # B, Hq, Hkv, Nq, page_size, seq_lens, causal
    (3, 32, 8, 1, 64, [1, 700, 4099], False),
    (4, 8, 2, 2, 128, [130, 64, 1, 2048], True),
    (2, 16, 4, 4, 64, [65, 300], True),
    (3, 4, 1, 4, 256, [0, 257, 1000], True),
    (2, 8, 8, 1, 64, [8192, 8191], False),
]


@pytest.mark.parametrize("case", PAGED_CASES, ids=[str(c) for c in PAGED_CASES])
@pytest.mark.parametrize("splits", [0, 1, 5])
def test_paged_decode(case, splits):
    B, Hq, Hkv, Nq, ps, lens, causal = case
    run_case(B, Hq, Hkv, Nq, ps, lens, causal, splits, 5100 + PAGED_CASES.index(case))


def test_paged_matches_contiguous_cache():
    """Pages laid out in order (page n of sequence b = b * pages + n) describe
    exactly the contiguous cache of fa_fwd; both entry points must agree."""
    w = synth.WORKLOADS["gqa_decode"].with_(B=4)
    x = synth.make_inputs(w)
    ps = 64
    pages = w.Nk // ps
    # [B, Hkv, Nk, d] -> pool [B * pages, ps, Hkv, d]
    pool_k = x["k"].permute(0, 2, 1, 3).reshape(w.B * pages, ps, w.Hkv, w.d).contiguous()
    pool_v = x["v"].permute(0, 2, 1, 3).reshape(w.B * pages, ps, w.Hkv, w.d).contiguous()
    table = torch.arange(w.B * pages, dtype=torch.int32).reshape(w.B, pages)
    lens = torch.full((w.B,), w.Nk, dtype=torch.int32)
    xd = G.to_gpu(x)
    o1, l1 = fa.fa_fwd_splitkv(xd["q"], xd["k"], xd["v"], num_splits=4)
    o2, l2 = fa.fa_fwd_paged(xd["q"], pool_k.cuda(), pool_v.cuda(), table.cuda(), lens.cuda(),
                             num_splits=4)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("d", [32, 64, 96])
def test_paged_decode_narrow_heads(d):
    run_case(3, 8, 2, 2, 64, [1, 700, 2049], True, 0, 8300 + d, d=d)


@pytest.mark.parametrize("d", [64, 128])
def test_paged_decode_fp16(d):
    run_case(2, 16, 4, 2, 128, [300, 4099], True, 0, 8400 + d, d=d, fp16=True)
