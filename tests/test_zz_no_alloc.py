"""The allocation-free gate entry point (moba_gate_topk_noalloc), for
callers that cannot allocate device memory: it must give the same block
indices as moba_gate_topk, call after call, although every call reuses the
same built-in scratch array. Collected last on purpose."""
import ctypes

import pytest
import torch

import long_context_prefill_block_b200 as moba
from moba_inputs import small_case

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_noalloc_gate_matches_gate_topk_on_consecutive_calls():
    shapes = [
        ((1000, 333, 0, 2048), 4, 2, 128, 128, 3, torch.bfloat16, 501),
        ((4096, 777), 8, 2, 128, 256, 5, torch.bfloat16, 502),   # larger table, different layout
        ((300, 95), 2, 2, 64, 20, 3, torch.float32, 503),        # small table after a large one
    ]
    for lengths, Hq, Hkv, d, B, topk, dtype, seed in shapes:
        q, k, _, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=seed)
        qd, kd = q.to(DEV), k.to(DEV)
        ref = moba.moba_gate_topk(qd, kd, cu, B, topk)
        first = moba.moba_gate_topk_noalloc(qd, kd, cu, B, topk)
        second = moba.moba_gate_topk_noalloc(qd, kd, cu, B, topk)
        torch.cuda.synchronize()
        assert torch.equal(first, ref)
        assert torch.equal(second, ref)


def test_noalloc_gate_rejects_tables_beyond_its_limit():
    # 2 sequences x 4096 blocks x 8 kv heads x d=128 x 4 B = 32 MiB > 4 MiB
    p = moba.MobaParams(2, 2 * 65536, 65536, 8, 8, 128, 16, 3, moba.MOBA_BF16)
    fn = moba.lib().moba_gate_topk_noalloc
    fn.argtypes = [ctypes.POINTER(moba.MobaParams)] + [ctypes.c_void_p] * 5
    fake = ctypes.c_void_p(1 << 20)
    assert fn(ctypes.byref(p), fake, fake, fake, fake, None) == moba.MOBA_ERR_WORKSPACE
