"""GPU tests of the boundary: error paths that need a device, the bounded-wait
machinery (a wait that nothing satisfies runs out and is reported, and the
device stays usable), and the stream contract."""
import pytest
import torch

import exact_attention_114_b200 as fa
import synth
from tests import gpu_parity as G

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_device_survives():
    assert fa.fa_selftest_wait_timeout(2000) == fa.FA_ERR_TIMEOUT
    # the status word was cleared by the check and the context still works
    fa.fa_check_device_status()
    G.check_forward_full(synth.WORKLOADS["tiny_mha"])


def test_runs_on_a_side_stream():
    w = synth.WORKLOADS["mha_1k"].with_(B=1, Hq=2, Hkv=2)
    x = synth.make_inputs(w, dout=False)
    xd = G.to_gpu(x)
    o_ref, _ = G.gpu_forward(xd, w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o, _ = fa.fa_fwd(xd["q"], xd["k"], xd["v"], causal=True)
    s.synchronize()
    assert torch.equal(o, o_ref)


def test_too_small_workspace_on_device():
    w = synth.WORKLOADS["tiny_mha"]
    xd = G.to_gpu(synth.make_inputs(w))
    o, lse = G.gpu_forward(xd, w)
    n = fa.fa_bwd_workspace_size(1, 1, 1, 128, 128, 64)
    ws = torch.empty(n - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.fa_bwd(xd["q"], xd["k"], xd["v"], o, xd["dout"], lse, workspace=ws)
    assert e.value.status == fa.FA_ERR_WORKSPACE
