"""Guard bands in place of a memory checker: every output buffer and workspace
is the middle of a larger allocation whose head and tail hold a canary bit
pattern; after the call the canaries must be intact, so no kernel writes
outside the extent it was given (ragged tails, padded head dims, split
partials, the e4m3 V^T workspace, paged decode)."""
import math

import pytest
import torch

import exact_attention_114_b200 as fa
import synth

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side (keeps the middle 16-byte aligned)
CANARY = 0x5A         # byte value of the guard bands


class Guarded:
    def __init__(self, shape, dtype):
        self.n_bytes = math.prod(shape) * torch.tensor([], dtype=dtype).element_size()
        self.buf = torch.full((self.n_bytes + 2 * GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        self.t = self.buf[GUARD:GUARD + self.n_bytes].view(dtype).view(shape)

    def intact(self):
        return bool((self.buf[:GUARD] == CANARY).all()) and bool((self.buf[GUARD + self.n_bytes:] == CANARY).all())


def _inputs(w, dtype=torch.bfloat16):
    return {k: v.cuda() for k, v in synth.make_inputs(w, dtype=dtype).items()}


@pytest.mark.parametrize("shape", [
    (1, 4, 2, 333, 200, 128, True), (2, 2, 1, 65, 129, 64, False), (1, 2, 2, 77, 77, 96, True),
    (1, 4, 1, 100, 300, 32, True), (1, 2, 1, 130, 130, 256, True), (1, 2, 1, 70, 70, 192, False),
])
def test_forward_backward_stay_inside(shape):
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    w = synth.Workload("guard", B, Hq, Hkv, Nq, Nk, d, causal, 9500 + d)
    x = _inputs(w)
    o, lse = Guarded((B, Hq, Nq, d), torch.bfloat16), Guarded((B, Hq, Nq), torch.float32)
    fa.fa_fwd(x["q"], x["k"], x["v"], o.t, lse.t, causal=causal)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    assert o.intact() and lse.intact()
    g = [Guarded(tuple(x[n].shape), torch.bfloat16) for n in ("q", "k", "v")]
    ws = Guarded((fa.fa_bwd_workspace_size(B, Hq, Hkv, Nq, Nk, d),), torch.uint8)
    fa.fa_bwd(x["q"], x["k"], x["v"], o.t, x["dout"], lse.t, g[0].t, g[1].t, g[2].t, causal=causal,
              workspace=ws.t)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    assert all(t.intact() for t in g) and ws.intact()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("splits", [1, 7])
def test_splitkv_stays_inside(d, splits):
    w = synth.Workload("guard_dec", 3, 8, 2, 2, 1000, d, True, 9600, backward=False)
    x = _inputs(w)
    o, lse = Guarded((3, 8, 2, d), torch.bfloat16), Guarded((3, 8, 2), torch.float32)
    ws = Guarded((max(fa.fa_fwd_splitkv_workspace_size(3, 8, 2, 2, 1000, d, splits), 16),), torch.uint8)
    fa.fa_fwd_splitkv(x["q"], x["k"], x["v"], o.t, lse.t, causal=True, num_splits=splits, workspace=ws.t)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    assert o.intact() and lse.intact() and ws.intact()


def test_paged_decode_stays_inside():
    B, Hq, Hkv, d, ps = 2, 8, 2, 128, 64
    lens = [100, 700]
    pages = [math.ceil(L / ps) for L in lens]
    num_pages = sum(pages) + 2
    g = torch.Generator().manual_seed(9700)
    perm = torch.randperm(num_pages, generator=g)
    table = torch.zeros((B, max(pages)), dtype=torch.int32)
    pos = 0
    for b, n in enumerate(pages):
        table[b, :n] = perm[pos:pos + n]
        pos += n
    kp = torch.randn((num_pages, ps, Hkv, d), generator=g).to(torch.bfloat16).cuda()
    vp = torch.randn((num_pages, ps, Hkv, d), generator=g).to(torch.bfloat16).cuda()
    q = torch.randn((B, Hq, 1, d), generator=g).to(torch.bfloat16).cuda()
    o, lse = Guarded((B, Hq, 1, d), torch.bfloat16), Guarded((B, Hq, 1), torch.float32)
    fa.fa_fwd_paged(q, kp, vp, table.cuda(), torch.tensor(lens, dtype=torch.int32).cuda(), o.t, lse.t,
                    num_splits=3)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    assert o.intact() and lse.intact()


def test_fp8_forward_stays_inside():
    w = synth.Workload("guard_fp8", 1, 4, 2, 300, 37, 128, True, 9800)
    x = {k: v.cuda() for k, v in synth.make_inputs_fp8(w).items()}
    ds = synth.FP8_DESCALE
    o, lse = Guarded((1, 4, 300, 128), torch.bfloat16), Guarded((1, 4, 300), torch.float32)
    ws = Guarded((fa.fa_fwd_fp8_workspace_size(1, 2, 37, 128),), torch.uint8)
    fa.fa_fwd_fp8(x["q"], x["k"], x["v"], ds["q"], ds["k"], ds["v"], o.t, lse.t, causal=True,
                  workspace=ws.t)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    assert o.intact() and lse.intact() and ws.intact()
