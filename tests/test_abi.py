"""Host-side checks of the C ABI (no GPU needed, no kernel launched): the
library builds for sm_100a and loads, exports every entry point that
include/fp8attn.h declares, agrees on the parameter-struct layout, and
rejects invalid arguments before touching the device."""
import ctypes
import os
import re

import pytest

from online_softmax_tcgen05_b200 import _binding
from online_softmax_tcgen05_b200._binding import EINVAL, EUNSUPPORTED, OK, Params

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "fp8attn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    pat = r"^\s*(?:const\s+)?(?:unsigned\s+)?(?:int|char|size_t|void|float)\s*\**\s*(\w+)\s*\("
    return sorted(set(re.findall(pat, text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    return _binding.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "fp8_attn_fwd" in names and "fp8_attn_fwd_ex" in names and "fp8_e4m3_scale_cast" in names
    for n in names:
        assert hasattr(lib, n), n
        assert n in _binding.SIGNATURES, n


def test_params_layout(lib):
    assert lib.fp8attn_params_sizeof() == ctypes.sizeof(Params)
    assert lib.fp8attn_version() == 104


def test_status_strings(lib):
    for s in (0, -1, -2, -3, -4):
        assert _binding.status_string(s)
    assert _binding.device_status_string(0) == ""
    assert "timeout" in _binding.device_status_string(0x107)


FAKE = 0x10000   # never dereferenced: every case below fails validation first


def base_params(**kw):
    p = dict(Q=FAKE, K=FAKE, V=FAKE, O=FAKE, B=1, H=2, H_kv=1, N=256, d=128, causal=0,
             scale=0.088, S=256.0, kv_order=1, n_sink=4, o_dtype=0, block_n=0,
             collapse_ctr=None, collapse_sink_ctr=None, collapse_rows=None, status_word=None,
             timeout_ns=0, debug_skip_kv_step=0)
    p.update(kw)
    return Params(**p)


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), EUNSUPPORTED), (dict(d=256), EUNSUPPORTED), (dict(block_n=32), EUNSUPPORTED),
    (dict(H=3, H_kv=2), EINVAL), (dict(H_kv=0), EINVAL), (dict(N=-1), EINVAL),
    (dict(S=0.0), EINVAL), (dict(S=-1.0), EINVAL), (dict(S=float("nan")), EINVAL),
    (dict(S=float("inf")), EINVAL), (dict(scale=float("nan")), EINVAL), (dict(scale=0.0), EINVAL),
    (dict(kv_order=2), EINVAL), (dict(causal=2), EINVAL), (dict(n_sink=-1), EINVAL),
    (dict(n_sink=257), EINVAL), (dict(o_dtype=5), EINVAL), (dict(Q=None), EINVAL),
    (dict(O=FAKE + 8), EINVAL), (dict(K=FAKE + 1), EINVAL),
    (dict(collapse_rows=FAKE), EINVAL), (dict(collapse_ctr=FAKE + 4), EINVAL),
    (dict(debug_skip_kv_step=-1), EINVAL), (dict(debug_skip_kv_step=2), EINVAL),
    (dict(timeout_ns=1), EINVAL), (dict(timeout_ns=999_999), EINVAL),
    (dict(denominator=2), EINVAL), (dict(denominator=1, S=0.001), EINVAL),
    (dict(qk_dtype=2), EINVAL),
    (dict(q_begin=64, q_end=256), EINVAL), (dict(q_begin=0, q_end=257), EINVAL),
    (dict(q_begin=128, q_end=128), EINVAL), (dict(q_begin=-128, q_end=128), EINVAL),
    (dict(q_begin=0, q_end=200), EINVAL), (dict(q_begin=256, q_end=256), EINVAL),
    (dict(B=65536, H=1, H_kv=1), EINVAL), (dict(B=256, H=256, H_kv=256), EINVAL),
])
def test_invalid_arguments_rejected_before_launch(lib, kw, status):
    p = base_params(**kw)
    assert lib.fp8_attn_fwd_ex(ctypes.byref(p), None) == status
    assert _binding.last_error() != ""


def test_empty_problem_is_a_noop(lib):
    for kw in (dict(B=0), dict(H=0), dict(N=0, n_sink=0)):
        p = base_params(Q=None, K=None, V=None, O=None, **kw)
        assert lib.fp8_attn_fwd_ex(ctypes.byref(p), None) == OK


def test_null_params_and_short_form_validation(lib):
    assert lib.fp8_attn_fwd_ex(None, None) == EINVAL
    assert lib.fp8_attn_fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 96, 0, 0.1, 256.0, 0, 0, None,
                            None) == EUNSUPPORTED
    assert lib.fp8_attn_fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 128, 0, 0.1, 256.0, 3, 0, None,
                            None) == EINVAL


def test_cast_validation(lib):
    assert lib.fp8_e4m3_scale_cast(None, None, 0, 1.0, None) == OK
    assert lib.fp8_e4m3_scale_cast(None, FAKE, 16, 1.0, None) == EINVAL
    assert lib.fp8_e4m3_scale_cast(FAKE, FAKE, 16, float("nan"), None) == EINVAL
    assert lib.fp8_e4m3_scale_cast(FAKE + 4, FAKE, 16, 1.0, None) == EINVAL


# ------------------------------------------------- host-buffer entry (no GPU) --
def test_host_workspace_bytes(lib):
    # prefill, 16 chunks -> 8 pieces of one kv head: 3 sets of Q (4 heads), K, V, O (BF16)
    plane = 32768 * 128
    assert _binding.host_workspace_bytes(B=1, H=32, H_kv=8, N=32768, d=128) == \
        3 * (4 * plane + plane + plane + 4 * plane * 2)
    # one chunk: the whole problem is one piece
    assert _binding.host_workspace_bytes(B=1, H=32, H_kv=8, N=32768, d=128, host_chunks=1) == \
        3 * 8 * (4 * plane + plane + plane + 4 * plane * 2)
    # BF16 Q/K, FP32 O, sizes rounded up to 256 bytes
    n, d = 100, 64
    r = lambda x: (x + 255) // 256 * 256
    assert _binding.host_workspace_bytes(B=2, H=4, H_kv=2, N=n, d=d, qk_dtype=1, o_dtype=1,
                                         host_chunks=4) == \
        3 * (r(2 * n * d * 2) + r(n * d * 2) + r(n * d) + r(2 * n * d * 4))
    for bad in (dict(B=0), dict(N=0), dict(H=3), dict(H_kv=0)):
        kw = dict(B=1, H=4, H_kv=2, N=256, d=64)
        kw.update(bad)
        assert _binding.host_workspace_bytes(**kw) == 0
    assert _binding.host_workspace_bytes(B=1, H=4, H_kv=2, N=256, d=64, host_chunks=0) == 0


@pytest.mark.parametrize("kw,plan,ws,nbytes,chunks", [
    (dict(q_begin=128, q_end=256), FAKE, 0x100000, 1 << 40, 4),   # row ranges: device entry only
    (dict(d=96), FAKE, 0x100000, 1 << 40, 4),
    (dict(), None, 0x100000, 1 << 40, 4),                          # no plan
    (dict(), FAKE, 0x100000, 1 << 40, 0),                          # host_chunks < 1
    (dict(), FAKE, None, 1 << 40, 4),                              # no workspace
    (dict(), FAKE, 0x100080, 1 << 40, 4),                          # workspace not 256-aligned
    (dict(), FAKE, 0x100000, 1024, 4),                             # workspace too small
    (dict(Q=None), FAKE, 0x100000, 1 << 40, 4),
])
def test_host_entry_rejects_before_any_cuda_call(lib, kw, plan, ws, nbytes, chunks):
    p = base_params(**kw)
    st = lib.fp8_attn_fwd_host(ctypes.byref(p), plan, ws, nbytes, chunks, None)
    assert st in (EINVAL, EUNSUPPORTED)
    assert _binding.last_error() != ""


@pytest.mark.parametrize("bad", ["shape", "dtype", "layout", "device"])
def test_attention_rejects_unusable_out(bad):
    # checked before any copy or launch, so host tensors suffice (no GPU)
    import torch
    from online_softmax_tcgen05_b200 import attention
    B, H, N, d = 1, 2, 128, 64
    q = torch.zeros((B, H, N, d), dtype=torch.uint8)
    out = {"shape": torch.empty((B, H, N + 1, d), dtype=torch.bfloat16),
           "dtype": torch.empty((B, H, N, d), dtype=torch.float32),
           "layout": torch.empty((B, H, d, N), dtype=torch.bfloat16).transpose(2, 3),
           "device": torch.empty((B, H, N, d), dtype=torch.bfloat16, device="meta")}[bad]
    with pytest.raises(ValueError):
        attention(q, q, q, out=out)


def test_schedule_switch(lib):
    """fp8attn_set_schedule returns the previous schedule and refuses unknown ones."""
    from online_softmax_tcgen05_b200 import SCHEDULE_ONE_TILE, SCHEDULE_TWO_TILES
    assert lib.fp8attn_set_schedule(SCHEDULE_TWO_TILES) == SCHEDULE_ONE_TILE
    assert lib.fp8attn_set_schedule(SCHEDULE_ONE_TILE) == SCHEDULE_TWO_TILES
    assert lib.fp8attn_set_schedule(7) == EINVAL
    assert lib.fp8attn_set_schedule(SCHEDULE_ONE_TILE) == SCHEDULE_ONE_TILE
