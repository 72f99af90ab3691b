"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point that include/moba.h declares, sizes workspaces and rejects
invalid arguments before launching anything."""
import ctypes
import os
import re

import pytest

import long_context_prefill_block_b200 as moba

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols(headers=None):
    """Entry points declared in include/*.h (all headers but the trace build's
    by default)."""
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h") and (fn in headers if headers else fn != "moba_trace.h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"MOBA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return names


def test_header_declares_the_boundary():
    names = set(declared_symbols())
    for need in ("moba_meanpool", "moba_gate_topk", "moba_forward", "moba_forward_with_indices",
                 "dense_causal_forward", "moba_workspace_size"):
        assert need in names


def test_library_exports_every_declared_symbol():
    lib = moba.lib()
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_checked_build_exports_the_same_entry_points():
    from long_context_prefill_block_b200 import build

    if not os.path.exists(build.LIB_CHECKED):
        pytest.skip("checked build absent")
    checked = ctypes.CDLL(build.LIB_CHECKED)
    for name in declared_symbols():
        assert hasattr(checked, name), name
    checked.moba_status_string.argtypes = [ctypes.c_int]
    checked.moba_status_string.restype = ctypes.c_char_p
    assert b"check" in checked.moba_status_string(moba.MOBA_ERR_CHECK)


def test_trace_entry_points_only_in_the_trace_build():
    from long_context_prefill_block_b200 import build

    names = declared_symbols(["moba_trace.h"])
    assert set(names) == {"moba_trace_arm", "moba_trace_disarm"}
    lib = moba.lib()
    for name in names:
        assert not hasattr(lib, name), name
    if not os.path.exists(build.LIB_TRACE):
        pytest.skip("trace build absent")
    traced = ctypes.CDLL(build.LIB_TRACE)
    for name in declared_symbols(["moba_trace.h"]) + declared_symbols():
        assert hasattr(traced, name), name


def params(**kw):
    base = dict(batch=1, total_tokens=32768, max_seqlen=32768, num_q_heads=32, num_kv_heads=32,
                head_dim=128, block_size=512, topk=3, dtype=moba.MOBA_BF16)
    base.update(kw)
    return moba.MobaParams(**base)


def test_workspace_sizes():
    assert moba.moba_workspace_size(params()) > 0


def test_prefix_mean_gate_workspace():
    # the prefix-mean gate keeps one fp32 own-block score per (token, q head)
    # and up to k history entries per row instead of k - 1
    base, pref = params(), params(own_block=1)
    extra = moba.moba_workspace_size(pref) - moba.moba_workspace_size(base)
    assert extra >= 32768 * 32 * 4
    # the allocation-free gate has no room for those scores: refused before any launch
    fn = moba.lib().moba_gate_topk_noalloc
    fn.argtypes = [ctypes.POINTER(moba.MobaParams)] + [ctypes.c_void_p] * 5
    fn.restype = ctypes.c_int
    assert fn(ctypes.byref(pref), None, None, None, None, None) == moba.MOBA_ERR_UNSUPPORTED
    # million-token GQA shape: partial results are kept one kv-head group at a time
    big = params(total_tokens=1 << 20, max_seqlen=1 << 20, num_kv_heads=8, block_size=4096, topk=12)
    assert 0 < moba.moba_workspace_size(big) < 48 * (1 << 30)
    assert moba.moba_num_blocks(big) == 256


@pytest.mark.parametrize("bad", [
    dict(num_q_heads=3, num_kv_heads=2), dict(block_size=0), dict(topk=0), dict(batch=-1),
    dict(routing=2), dict(routing=-1), dict(own_block=2), dict(own_block=-1),
    dict(num_kv_heads=0)])
def test_invalid_params_rejected(bad):
    p = params(**bad)
    assert moba.moba_workspace_size(p) == 0
    rc = moba.lib().moba_forward(ctypes.byref(p), None, None, None, None, None, None, None, 0, None)
    assert rc == moba.MOBA_ERR_INVALID_ARG


@pytest.mark.parametrize("bad", [dict(head_dim=96), dict(topk=33), dict(dtype=7)])
def test_unsupported_params(bad):
    p = params(**bad)
    rc = moba.lib().moba_forward(ctypes.byref(p), None, None, None, None, None, None, None, 0, None)
    assert rc == moba.MOBA_ERR_UNSUPPORTED


def test_null_and_misaligned_pointers_rejected_before_launch():
    p = params()
    lib = moba.lib()
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 2)
    assert lib.moba_forward(ctypes.byref(p), None, fake, fake, fake, fake, None, fake, 1 << 40,
                            None) == moba.MOBA_ERR_INVALID_ARG
    assert lib.moba_forward(ctypes.byref(p), odd, fake, fake, fake, fake, None, fake, 1 << 40,
                            None) == moba.MOBA_ERR_INVALID_ARG
    # workspace too small
    assert lib.moba_forward(ctypes.byref(p), fake, fake, fake, fake, fake, None, fake, 16,
                            None) == moba.MOBA_ERR_WORKSPACE
    # 16-byte but not 32-byte aligned: the kernels move rows in 32-byte pieces
    half = ctypes.c_void_p((1 << 20) + 16)
    assert lib.moba_forward(ctypes.byref(p), half, fake, fake, fake, fake, None, fake, 1 << 40,
                            None) == moba.MOBA_ERR_INVALID_ARG
    assert lib.moba_forward(ctypes.byref(p), fake, fake, fake, fake, half, None, fake, 1 << 40,
                            None) == moba.MOBA_ERR_INVALID_ARG
    assert lib.moba_forward(ctypes.byref(p), fake, fake, fake, fake, fake, None, half, 1 << 40,
                            None) == moba.MOBA_ERR_WORKSPACE
    assert lib.dense_causal_forward(ctypes.byref(p), fake, None, fake, fake, fake, None,
                                    None) == moba.MOBA_ERR_INVALID_ARG


def test_empty_input_is_a_no_op():
    p = params(total_tokens=0, batch=0, max_seqlen=0)
    assert moba.lib().moba_forward(ctypes.byref(p), None, None, None, None, None, None, None, 0,
                                   None) == moba.MOBA_OK


def test_status_strings():
    lib = moba.lib()
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert lib.moba_status_string(code)


def test_decode_argument_checks():
    # validated on the host before any launch: no GPU needed
    L = moba.lib()
    L.moba_decode_workspace_size.argtypes = [ctypes.POINTER(moba.MobaParams), ctypes.c_int]
    L.moba_decode_workspace_size.restype = ctypes.c_size_t
    assert L.moba_decode_workspace_size(ctypes.byref(params()), 4) > 0
    assert L.moba_decode_workspace_size(ctypes.byref(params()), -1) == 0
    fn = L.moba_decode
    V = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(moba.MobaParams), V, V, V, V, V, ctypes.c_int, V, V, V, V, V,
                   ctypes.c_size_t, V]
    fn.restype = ctypes.c_int
    args = [None] * 5
    assert fn(ctypes.byref(params()), *args, -1, None, None, None, None, None, 0, None) \
        == moba.MOBA_ERR_INVALID_ARG
    assert fn(ctypes.byref(params(own_block=1)), *args, 1, None, None, None, None, None, 0, None) \
        == moba.MOBA_ERR_UNSUPPORTED
    assert fn(ctypes.byref(params()), *args, 0, None, None, None, None, None, 0, None) == moba.MOBA_OK
    up = L.moba_meanpool_update
    up.argtypes = [ctypes.POINTER(moba.MobaParams), V, V, V, ctypes.c_int, V, V]
    up.restype = ctypes.c_int
    assert up(ctypes.byref(params()), None, None, None, -1, None, None) == moba.MOBA_ERR_INVALID_ARG
    assert up(ctypes.byref(params()), None, None, None, 0, None, None) == moba.MOBA_OK

