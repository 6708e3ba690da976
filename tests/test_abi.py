"""CPU tests of the C ABI boundary: the library loads, exports every function
declared in include/fa.h, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

import exact_attention_114_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")

# a plausible, 16-byte aligned address; never dereferenced because every call
# below fails validation first
FAKE = ctypes.c_void_p(0x10000)
MISALIGNED = ctypes.c_void_p(0x10008)


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 10, names
    L = fa.lib()
    for n in names:
        assert hasattr(L, n), f"{n} declared in fa.h but not exported by libfa.so"


def test_abi_version_and_status_strings():
    assert fa.abi_version() == 1
    for code, name in [(0, "FA_OK"), (1, "FA_ERR_INVALID_ARGUMENT"), (2, "FA_ERR_UNSUPPORTED"),
                       (3, "FA_ERR_WORKSPACE"), (4, "FA_ERR_CUDA"), (5, "FA_ERR_TIMEOUT"),
                       (6, "FA_ERR_SLOT_CONFLICT")]:
        assert fa.status_string(code) == name
        # the enum values in the header match
        assert re.search(rf"\b{name}\s*=\s*{code}\b", open(HEADER, encoding="utf-8").read())


def _fwd(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, Hq=2, Hkv=1, Nq=8, Nk=8, d=64,
         scale=0.125, causal=0):
    return fa.lib().fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(o=None), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(k=MISALIGNED), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(lse=ctypes.c_void_p(0x10002)), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(B=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(Nq=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(Nk=-3), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(Hq=3, Hkv=2), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(causal=2), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(d=80), fa.FA_ERR_UNSUPPORTED),
    (dict(d=48), fa.FA_ERR_UNSUPPORTED),
    (dict(d=16), fa.FA_ERR_UNSUPPORTED),
    (dict(d=288), fa.FA_ERR_UNSUPPORTED),
    (dict(d=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(B=1 << 20, Hq=1 << 10, Hkv=1 << 10), fa.FA_ERR_UNSUPPORTED),
])
def test_fwd_rejects_bad_arguments(kw, status):
    assert _fwd(**kw) == status
    assert fa.last_error_message() != ""


def test_bwd_rejects_bad_arguments():
    L = fa.lib()
    args = [FAKE] * 5 + [FAKE] + [FAKE] * 3
    base = dict(B=1, Hq=2, Hkv=1, Nq=8, Nk=8, d=128, scale=0.1, causal=1)

    def call(ptrs, ws=None, ws_bytes=0, **over):
        p = dict(base, **over)
        return L.fa_bwd(*ptrs, p["B"], p["Hq"], p["Hkv"], p["Nq"], p["Nk"], p["d"], p["scale"],
                        p["causal"], ws, ws_bytes, None)

    for i in range(9):
        bad = list(args)
        bad[i] = None
        assert call(bad) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(args, d=80) == fa.FA_ERR_UNSUPPORTED
    assert call(args, d=288) == fa.FA_ERR_UNSUPPORTED    # head sizes stop at 256
    assert fa.fa_bwd_workspace_size(1, 2, 1, 8, 8, 288) == 0
    # d = 256: D and -LSE rows (64 padded rows each) and the fp32 accumulator, 256 wide
    assert fa.fa_bwd_workspace_size(1, 2, 1, 8, 8, 256) == 2 * 512 + 2 * 64 * 256 * 4
    # a workspace that is too small is refused before any launch
    need = fa.fa_bwd_workspace_size(1, 2, 1, 8, 8, 128)
    assert call(args, ws=ctypes.c_void_p(0x100000), ws_bytes=need - 1) == fa.FA_ERR_WORKSPACE
    assert call(args, ws=ctypes.c_void_p(0x100010), ws_bytes=need) == fa.FA_ERR_INVALID_ARGUMENT


def test_splitkv_rejects_bad_arguments():
    L = fa.lib()

    def call(Hq=32, Hkv=8, Nq=1, d=128, splits=0, ws=None, ws_bytes=0):
        return L.fa_fwd_splitkv(FAKE, FAKE, FAKE, FAKE, None, 2, Hq, Hkv, Nq, 4096, d, 0.1, 0,
                                splits, ws, ws_bytes, None)

    assert call(splits=-1) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(splits=257) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(Nq=8) == fa.FA_ERR_UNSUPPORTED       # 8 * 4 rows per kv head > 16
    assert call(d=160) == fa.FA_ERR_UNSUPPORTED
    need = fa.fa_fwd_splitkv_workspace_size(2, 32, 8, 1, 4096, 128, 4)
    assert need > 0
    assert call(splits=4, ws=ctypes.c_void_p(0x100000), ws_bytes=need - 16) == fa.FA_ERR_WORKSPACE
    assert call(splits=4, ws=ctypes.c_void_p(0x100080), ws_bytes=need) == fa.FA_ERR_INVALID_ARGUMENT


def test_splitkv_noalloc_rejects_before_touching_cuda():
    # explicit split counts keep the plan off the device query, so every
    # refusal below happens before the first CUDA call
    L = fa.lib()

    def call(B=2, Hq=32, Hkv=8, Nq=1, Nk=4096, d=128, splits=4, q=FAKE):
        return L.fa_fwd_splitkv_noalloc(q, FAKE, FAKE, FAKE, None, B, Hq, Hkv, Nq, Nk, d, 0.1, 0,
                                        splits, None)

    assert call(q=None) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(q=MISALIGNED) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(splits=-1) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(splits=257) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(Nq=8) == fa.FA_ERR_UNSUPPORTED
    assert call(d=160) == fa.FA_ERR_UNSUPPORTED
    # partials larger than the fixed scratch are refused, naming the sizes
    need = fa.fa_fwd_splitkv_workspace_size(64, 32, 8, 4, 8192, 128, 64)
    assert need > fa.NOALLOC_SCRATCH_BYTES
    assert call(B=64, Nq=4, Nk=8192, splits=64) == fa.FA_ERR_WORKSPACE
    msg = fa.last_error_message()
    assert str(need) in msg and str(fa.NOALLOC_SCRATCH_BYTES) in msg
    # the limit is the header's
    text = open(HEADER, encoding="utf-8").read()
    m = re.search(r"FA_SPLITKV_NOALLOC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", text)
    assert m and int(m[1]) * int(m[2]) * int(m[3]) == fa.NOALLOC_SCRATCH_BYTES


def _sm_count():
    import torch
    return torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 148


def test_workspace_sizes():
    # backward: D and LSE rows (fp32) + fp32 dQ accumulator, rows padded to 64
    n = fa.fa_bwd_workspace_size(1, 32, 8, 8192, 8192, 128)
    rows = 32 * 8192
    base = rows * 4 * 2 + rows * 128 * 4
    if _sm_count() == 148:
        # without a causal mask the 512 (key block, kv head) units split in two: one
        # fp32 dK | dV partial per unit (2 x 128 keys x 128 x 4 B) and two counters
        assert n == base + 512 * 2 * 128 * 128 * 4 + 512 * 2 * 4
    else:
        assert n >= base
    assert fa.fa_bwd_workspace_size(1, 1, 1, 65, 65, 64) == 512 * 2 + 128 * 64 * 4  # 65 -> 128 rows
    assert fa.fa_bwd_workspace_size(0, 1, 1, 1, 1, 64) == 0
    # split-KV: one partial (O_s, lse_s) per (b, kv head, split, row); one split needs none
    assert fa.fa_fwd_splitkv_workspace_size(4, 8, 2, 1, 4096, 128, 1) == 0
    n4 = fa.fa_fwd_splitkv_workspace_size(4, 8, 2, 1, 4096, 128, 4)
    part_rows = 4 * 2 * 4 * 4
    assert n4 == part_rows * 128 * 4 + ((part_rows * 4 + 255) // 256) * 256


def test_no_gpu_reports_cuda_error_without_crashing():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = _fwd(B=1, Hq=1, Hkv=1, Nq=128, Nk=128, d=64)
    assert st == fa.FA_ERR_CUDA
    assert fa.last_error_message()


def test_paged_rejects_bad_arguments():
    L = fa.lib()

    def call(page_size=64, num_pages=8, max_pages=4, table=FAKE, lens=FAKE, d=128, Nq=1, splits=0):
        return L.fa_fwd_paged(FAKE, FAKE, FAKE, table, lens, FAKE, None, 2, 8, 2, Nq, d, page_size,
                              num_pages, max_pages, 0.1, 0, splits, None, 0, None)

    assert call(table=None) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(lens=ctypes.c_void_p(0x10002)) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(page_size=48) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(page_size=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(num_pages=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(max_pages=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(d=160) == fa.FA_ERR_UNSUPPORTED
    assert call(Nq=5) == fa.FA_ERR_UNSUPPORTED      # 5 * 4 rows per kv head > 16
    assert call(splits=300) == fa.FA_ERR_INVALID_ARGUMENT
    assert fa.fa_fwd_paged_workspace_size(2, 8, 2, 1, 64, 4, 128, 2) > 0


def test_dtype_codes_are_checked_first():
    """fa_fwd_ex / fa_bwd_ex refuse a dtype code outside fa_dtype_t before any
    other check, and accept both codes up to the pointer checks."""
    L = fa.lib()
    for bad in (-1, 2, 7):
        st = L.fa_fwd_ex(bad, FAKE, FAKE, FAKE, FAKE, None, 1, 2, 1, 8, 8, 64, 0.1, 0, None)
        assert st == fa.FA_ERR_INVALID_ARGUMENT
        assert "dtype" in fa.last_error_message()
        st = L.fa_bwd_ex(bad, *([FAKE] * 9), 1, 2, 1, 8, 8, 64, 0.1, 1, None, 0, None)
        assert st == fa.FA_ERR_INVALID_ARGUMENT
    for good in (fa.FA_DTYPE_BF16, fa.FA_DTYPE_FP16):
        st = L.fa_fwd_ex(good, None, FAKE, FAKE, FAKE, None, 1, 2, 1, 8, 8, 64, 0.1, 0, None)
        assert st == fa.FA_ERR_INVALID_ARGUMENT and "q" in fa.last_error_message()


def test_padded_head_dims_share_the_kernel_workspace():
    """d = 32 and 96 run on the 64 and 128 kernels, whose dQ accumulator rows
    have the kernel width."""
    ws = fa.fa_bwd_workspace_size
    assert ws(1, 4, 2, 100, 100, 32) == ws(1, 4, 2, 100, 100, 64)
    assert ws(1, 4, 2, 100, 100, 96) == ws(1, 4, 2, 100, 100, 128)
    assert ws(1, 4, 2, 100, 100, 64) < ws(1, 4, 2, 100, 100, 128)


def test_fp8_rejects_bad_arguments():
    L = fa.lib()
    base = dict(B=1, Hq=2, Hkv=1, Nq=8, Nk=8, d=128, scale=0.1, causal=1, ds=(0.5, 0.5, 0.5))

    def call(q=FAKE, ws=None, ws_bytes=0, **over):
        p = dict(base, **over)
        return L.fa_fwd_fp8(q, FAKE, FAKE, *p["ds"], FAKE, None, p["B"], p["Hq"], p["Hkv"], p["Nq"],
                            p["Nk"], p["d"], p["scale"], p["causal"], ws, ws_bytes, None)

    assert call(q=None) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(d=64) == fa.FA_ERR_UNSUPPORTED
    assert call(ds=(0.5, 0.0, 0.5)) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(ds=(0.5, 0.5, float("inf"))) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(ds=(1e30, 1e30, 1.0)) == fa.FA_ERR_INVALID_ARGUMENT   # scale * dq * dk overflows
    need = fa.fa_fwd_fp8_workspace_size(1, 1, 8, 128)
    assert need == 2048                     # 128 d rows x 16 padded keys
    assert fa.fa_fwd_fp8_workspace_size(1, 1, 8, 64) == 0
    assert call(ws=ctypes.c_void_p(0x100000), ws_bytes=need - 1) == fa.FA_ERR_WORKSPACE
    assert call(ws=ctypes.c_void_p(0x100010), ws_bytes=need) == fa.FA_ERR_INVALID_ARGUMENT
    assert fa.fa_fwd_fp8_workspace_size(2, 8, 8192, 128) == 2 * 8 * 128 * 8192


def test_tile_slot_hook_checks_its_slot_before_any_cuda_call():
    """The test hook refuses a slot outside -1..255; pinning and releasing
    without a preset owner makes no CUDA call at all."""
    L = fa.lib()
    for bad in (-2, 256, 10_000):
        assert L.fa_testhook_tile_slot(bad, 0) == fa.FA_ERR_INVALID_ARGUMENT
        assert "slot" in fa.last_error_message()
    assert L.fa_testhook_tile_slot(3, 0) == fa.FA_OK
    assert L.fa_testhook_tile_slot(-1, 0) == fa.FA_OK


def test_backward_query_split_rule():
    """The split fa_bwd takes on a 148-SM device: none where the units fill
    the SMs in whole rounds (the causal step workloads), two where 512 equal
    units would leave a last round of 68 CTAs, and up to eight where a few
    units would leave most SMs idle; 0 for sizes fa_bwd refuses."""
    if _sm_count() != 148:
        pytest.skip("the expected splits are for 148 SMs")
    qs = fa.fa_bwd_query_split
    assert qs(1, 32, 8, 8192, 8192, 128, 1) == 1      # gqa_8k causal
    assert qs(1, 32, 8, 8192, 8192, 128, 0) == 2      # gqa_8k without the mask
    assert qs(2, 32, 32, 4096, 4096, 128, 1) == 1     # mha_4k_long
    assert qs(4, 16, 16, 1024, 1024, 64, 0) == 1      # mha_1k: 16 steps per unit
    assert qs(1, 32, 8, 8192, 8192, 256, 1) == 1
    assert qs(1, 4, 1, 2048, 2048, 128, 1) == 8       # 16 units
    assert qs(1, 4, 1, 2048, 2048, 128, 0) == 8
    assert qs(1, 2, 1, 1536, 1536, 128, 1) == 3
    assert qs(1, 2, 1, 2048, 2048, 128, 0) == 4
    assert qs(1, 4, 1, 1536, 1536, 128, 0) == 6
    assert qs(1, 4, 1, 1000, 3000, 128, 1) == 4       # bottom-right mask, Nq < Nk
    assert qs(1, 1, 1, 64, 64, 64, 0) == 1
    assert qs(1, 3, 2, 64, 64, 64, 0) == 0            # Hq not a multiple of Hkv
    assert qs(1, 2, 1, 64, 64, 288, 0) == 0
    assert fa.lib().fa_bwd_query_split(1, 2, 1, 64, 64, 64, 2) == 0   # causal flag not 0 / 1


def test_forward_key_split_rule():
    """The key shares fa_fwd takes on a 148-SM device: none where the work tiles
    fill the SMs (the step workloads) or for the decode shapes (split-KV decode
    kernels), up to 16 where a few long tiles would leave most SMs idle (a short
    chunk appended to a long context); 0 for sizes fa_fwd refuses."""
    if _sm_count() != 148:
        pytest.skip("the expected shares are for 148 SMs")
    ks = fa.fa_fwd_kv_split
    assert ks(1, 32, 8, 8192, 8192, 128, 1) == 1      # gqa_8k: 1024 work tiles
    assert ks(2, 32, 32, 4096, 4096, 128, 1) == 1     # mha_4k_long
    assert ks(4, 16, 16, 1024, 1024, 64, 0) == 1      # mha_1k: 256 work tiles
    assert ks(1, 32, 8, 8192, 8192, 256, 1) == 1
    assert ks(64, 32, 8, 1, 8192, 128, 0) == 1        # decode shape
    assert ks(1, 32, 8, 512, 32768, 128, 1) == 2      # 64 work tiles of 254-256 key blocks
    assert ks(1, 32, 8, 64, 32768, 128, 1) == 16      # group rows: 8 work tiles (one per kv head)
    assert ks(1, 4, 1, 2048, 2048, 128, 1) == 4
    assert ks(1, 4, 1, 2048, 2048, 128, 0) == 4
    assert ks(1, 2, 1, 300, 5000, 64, 1) == 16
    assert ks(1, 2, 1, 1000, 2000, 256, 0) == 8
    assert ks(1, 4, 1, 1000, 1000, 128, 1) == 1       # 16 tiles of at most 8 blocks: too little to gain
    assert ks(1, 8, 2, 1, 8192, 256, 1) == 16         # a d = 256 decode shape runs the tiled kernel
    assert ks(1, 32, 8, 1024, 32768, 128, 1) == 1     # 128 equal units: one round, splitting costs more
    assert ks(1, 32, 8, 2048, 32768, 128, 1) == 1     # 256 units: 4-share tail, but K / V beyond L2 (no gain)
    assert ks(1, 32, 8, 4096, 32768, 128, 1) == 2     # 512 units: the last 68 in 2 shares
    assert ks(1, 3, 2, 64, 64, 64, 0) == 0            # Hq not a multiple of Hkv
    assert ks(1, 2, 1, 64, 64, 80, 0) == 0            # head size not a multiple of 32
    assert fa.lib().fa_fwd_kv_split(1, 2, 1, 64, 64, 64, 2) == 0


def test_forward_key_split_plan_cache():
    """The planner's cache: a context that grows by one key at a time (a new shape
    per call, more than the cache keeps) gives the same plans as the first calls
    on those shapes, and the known plans still hold after the cache started over."""
    if _sm_count() != 148:
        pytest.skip("the expected shares are for 148 SMs")
    ks = fa.fa_fwd_kv_split
    first = [ks(1, 32, 8, 512, nk, 128, 1) for nk in range(100, 6000)]
    for i in range(5000):   # 5000 different key-block counts
        ks(1, 8, 2, 300 + 7 * i, 1000 + 128 * i, 64, 1)
    again = [ks(1, 32, 8, 512, nk, 128, 1) for nk in range(100, 6000)]
    assert first == again
    assert ks(1, 32, 8, 512, 32768, 128, 1) == 2
    assert ks(1, 32, 8, 4096, 32768, 128, 1) == 2
    assert ks(1, 2, 1, 300, 5000, 64, 1) == 16
