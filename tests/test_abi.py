"""The C-ABI library loads, exports every entry point include/moba.h declares, and
rejects bad arguments on the host before touching a device (CPU only)."""
import ctypes
import os
import re

import pytest
import torch

import block_sparse_long_prefill_b200 as moba

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moba.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_abi():
    assert _declared() == sorted(moba.ABI_FUNCTIONS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(moba.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings():
    assert moba.status_string(0) == "ok"
    for code in range(-9, 0):
        assert moba.status_string(code) != "unknown status"


def test_workspace_size_is_host_only_and_grows_with_topk():
    a = moba.workspace_size(1, 32, 8, 32768, 128, 512, 3)
    b = moba.workspace_size(1, 32, 8, 32768, 128, 512, 4)
    assert 0 < a < b
    # k = 1 keeps only the own block: no partials, no entries.
    c = moba.workspace_size(1, 32, 8, 32768, 128, 512, 1)
    assert c < a


@pytest.mark.parametrize("args,code", [
    ((1, 32, 8, 32768, 128, 500, 3), -1),   # block not a multiple of 128
    ((1, 30, 8, 32768, 128, 512, 3), -1),   # hq not a multiple of hkv
    ((1, 32, 8, 32768, 96, 512, 3), -2),    # unsupported d
    ((1, 32, 8, 32768, 128, 512, 0), -4),   # topk < 1
    ((1, 32, 8, 32768, 128, 512, 33), -4),  # topk > 32
])
def test_workspace_size_rejects_bad_shapes(args, code):
    out = ctypes.c_size_t(0)
    assert moba.library().moba_workspace_size(*args, ctypes.byref(out)) == code


def test_block_need_not_divide_n():
    """N = 250 * 128 with blocks of 512: 63 blocks, the last one partial."""
    a = moba.workspace_size(1, 32, 8, 32000, 128, 512, 3)
    b = moba.workspace_size(1, 32, 8, 32256, 128, 512, 3)  # 63 full blocks
    assert 0 < a <= b


def test_bad_arguments_are_rejected_before_any_launch():
    lib = moba.library()
    T = moba.MobaTensor
    null = T(None, 0, 0, 0)
    ok = T(1 << 20, 8 * 1024, 8 * 1024, 128)
    mis = T((1 << 20) + 2, 8 * 1024, 8 * 1024, 128)
    odd = T(1 << 20, 8 * 1024, 8 * 1024, 100)
    # pool: null tensor, misaligned pointer, misaligned stride, empty sequence, no block
    assert lib.moba_pool_keys(null, 1, 1, 1024, 128, 128, 1 << 20, 1 << 20, None) == -4
    assert lib.moba_pool_keys(mis, 1, 1, 1024, 128, 128, 1 << 20, 1 << 20, None) == -3
    assert lib.moba_pool_keys(odd, 1, 1, 1024, 128, 128, 1 << 20, 1 << 20, None) == -3
    assert lib.moba_pool_keys(ok, 1, 1, 0, 128, 128, 1 << 20, 1 << 20, None) == -1
    assert lib.moba_pool_keys(ok, 1, 1, 1000, 128, 0, 1 << 20, 1 << 20, None) == -1
    # select: a block that is not a multiple of 128 (any N is taken)
    assert lib.moba_select_topk(ok, 1 << 20, 1, 1, 1, 1000, 128, 100, 3, 1 << 20, 1 << 20,
                                1 << 30, None) == -1
    # select: workspace too small
    assert lib.moba_select_topk(ok, 1 << 20, 1, 1, 1, 1024, 128, 128, 3, 1 << 20, 1 << 20, 16,
                                None) == -5
    # attention: negative window, unsupported d
    assert lib.moba_attn_fwd(ok, ok, ok, 1 << 20, 1, 1, 1, 1024, 128, 128, 3, -1, 0.0, ok,
                             1 << 20, 1 << 20, 1 << 30, None) == -4
    assert lib.swa_attn_fwd(ok, ok, ok, 1, 1, 1, 1024, 96, 64, 0.0, ok, 1 << 20, None) == -2
    assert lib.swa_attn_fwd(ok, ok, ok, 1, 1, 1, 1024, 128, 0, 0.0, ok, 1 << 20, None) == -4


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_a_device_reports_no_device():
    lib = moba.library()
    ok = moba.MobaTensor(1 << 20, 8 * 1024, 8 * 1024, 128)
    rc = lib.swa_attn_fwd(ok, ok, ok, 1, 1, 1, 1024, 128, 64, 0.0, ok, 1 << 20, None)
    assert rc == -8


def test_chunk_workspace_and_offset_checks():
    """Chunked prefill (N query rows, the last N of Nk positions): the workspace of the
    last 8K rows of a 32K context is smaller than the whole prefill's; the query offset
    Nk - N may be any non-negative number."""
    whole = moba.workspace_size(1, 32, 8, 32768, 128, 512, 3)
    chunk = moba.workspace_size_chunk(1, 32, 8, 8192, 32768, 128, 512, 3)
    assert 0 < chunk < whole
    assert moba.workspace_size_chunk(1, 32, 8, 32768, 32768, 128, 512, 3) == whole
    lib = moba.library()
    out = ctypes.c_size_t(0)
    assert lib.moba_workspace_size_chunk(1, 32, 8, 8192, 8192 + 64, 128, 512, 3, ctypes.byref(out)) == 0
    assert lib.moba_workspace_size_chunk(1, 32, 8, 8192, 4096, 128, 512, 3, ctypes.byref(out)) == -1
    ok = moba.MobaTensor(1 << 20, 8 * 1024, 8 * 1024, 128)
    assert lib.swa_attn_fwd_chunk(ok, ok, ok, 1, 1, 1, 1000, 900, 128, 64, 0.0, ok, 1 << 20, None) == -1


def test_static_gate_rejects_a_sink_beyond_the_list():
    lib = moba.library()
    assert lib.moba_select_static(1, 2, 1, 1024, 1024, 128, 128, 3, 3, 1 << 20, 1 << 20, 1 << 30,
                                  None) == -4
    assert lib.moba_select_static(1, 2, 1, 1024, 1024, 128, 128, 3, -1, 1 << 20, 1 << 20, 1 << 30,
                                  None) == -4


def test_minmax_entries_check_arguments():
    lib = moba.library()
    ok = moba.MobaTensor(1 << 20, 8 * 1024, 8 * 1024, 128)
    assert lib.moba_pool_keys_minmax(ok, 1, 1, 1024, 128, 0, 1 << 20, None) == -1
    assert lib.moba_pool_keys_minmax(ok, 1, 1, 1024, 128, 128, None, None) == -4
    assert lib.moba_select_topk_minmax(ok, 1 << 20, 1, 2, 1, 1024, 1000, 128, 128, 3, 1 << 20,
                                       1 << 20, 1 << 30, None) == -1  # fewer keys than queries


@pytest.mark.parametrize("cu", [[1, 256], [0, 128, 64], [0, 100], []])
def test_varlen_rejects_bad_offsets_before_any_launch(cu):
    q = torch.empty(256, 2, 64, dtype=torch.bfloat16)
    k = torch.empty(256, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        moba.moba_prefill_varlen(q, k, k, cu, 128, 2)


def test_host_pipeline_needs_groups_that_divide_the_kv_heads():
    with pytest.raises(ValueError):
        moba.MobaPrefillHost(1, 8, 4, 1024, 128, 512, 3, groups=3)


def test_backward_checks_arguments_on_the_host():
    lib = moba.library()
    ok = moba.MobaTensor(1 << 20, 8 * 1024, 8 * 1024, 128)
    out = ctypes.c_size_t(0)
    assert lib.moba_bwd_workspace_size(1, 2, 1, 1024, 128, 128, 3, ctypes.byref(out)) == 0
    assert out.value > 0
    assert lib.moba_bwd_workspace_size(1, 2, 1, 1024, 80, 128, 3, ctypes.byref(out)) == -2
    args = lambda window, d, ws: (ok, ok, ok, ok, ok, 1 << 20, 1 << 20, 1 << 20, 1 << 30, 1, 2, 1,
                                 1024, d, 128, 3, window, 0.0, ok, ok, ok, 1 << 20, ws, None)
    assert lib.moba_attn_bwd(*args(5, 128, 1 << 30)) == -4     # a window: not supported
    assert lib.moba_attn_bwd(*args(0, 80, 1 << 30)) == -2      # d = 80: not supported
    assert lib.moba_attn_bwd(*args(0, 128, 16)) == -5          # backward workspace too small
