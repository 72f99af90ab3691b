"""The allocation-free gate entry point (moba_gate_topk_noalloc), for
callers that cannot allocate device memory (a runtime that owns all device
memory, or a path that cannot take cudaMalloc's device-wide
synchronisation). It must give the same block indices as moba_gate_topk,
and the oracle's up to near-ties, call after call, although every call
reuses the same built-in 4 MiB scratch array. Collected last on purpose.

Every pointer handed to the library here comes from the allocator; the
refusal tests pass null pointers, which the entry point can never launch
on, and rely on its size check coming first."""
import ctypes

import pytest
import torch

import long_context_prefill_block_b200 as moba
import oracle
from moba_inputs import small_case
from parity import index_mismatches

pytestmark = pytest.mark.gpu
DEV = "cuda"
LIMIT_FLOATS = (4 << 20) // 4  # the built-in table holds 1,048,576 floats


def _compare(lengths, Hq, Hkv, d, B, topk, dtype, seed, shared=False, max_seqlen=None):
    q, k, _, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=seed)
    qd, kd = q.to(DEV), k.to(DEV)
    kw = dict(max_seqlen=max_seqlen, shared_routing=shared)
    ref = moba.moba_gate_topk(qd, kd, cu, B, topk, **kw)
    first = moba.moba_gate_topk_noalloc(qd, kd, cu, B, topk, **kw)
    second = moba.moba_gate_topk_noalloc(qd, kd, cu, B, topk, **kw)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    assert torch.equal(first, ref)
    assert torch.equal(second, ref)
    ref_idx, gap = oracle.gate_topk(q, k, cu, B, topk, shared_routing=shared)
    index_mismatches(second.cpu().numpy(), ref_idx, gap)


@pytest.mark.parametrize("case", [
    ((1000, 333, 0, 2048), 4, 2, 128, 128, 3, torch.bfloat16, 501, False),
    ((4096, 777), 8, 2, 128, 256, 5, torch.bfloat16, 502, False),   # larger table
    ((300, 95), 2, 2, 64, 20, 3, torch.float32, 503, False),        # small table after a large one
    ((2048, 1500), 8, 2, 128, 128, 4, torch.bfloat16, 504, True),   # shared routing, tensor cores
    ((700, 64), 6, 2, 64, 32, 3, torch.float32, 505, True),         # shared routing, SIMT gate
])
def test_noalloc_gate_matches_gate_topk_and_oracle_on_consecutive_calls(case):
    *shape, shared = case
    _compare(*shape, shared=shared)


def test_noalloc_gate_at_the_table_limit():
    # 4 sequences x ceil(32768 / 128) = 256 blocks x 8 kv heads x d = 128:
    # exactly 1,048,576 floats, the whole array (max_seqlen above the longest
    # sequence only reserves block slots)
    lengths, Hkv, d, B = (1000, 333, 2048, 77), 8, 128, 128
    assert len(lengths) * (32768 // B) * Hkv * d == LIMIT_FLOATS
    _compare(lengths, 8, Hkv, d, B, 3, torch.bfloat16, 506, max_seqlen=32768)


def _raw_call(p):
    fn = moba.lib().moba_gate_topk_noalloc
    fn.argtypes = [ctypes.POINTER(moba.MobaParams)] + [ctypes.c_void_p] * 5
    fn.restype = ctypes.c_int
    return fn(ctypes.byref(p), None, None, None, None, None)


def test_noalloc_gate_rejects_tables_beyond_its_limit():
    # the first table size over the limit: one more block slot than the
    # limit shape above (4 x 257 x 8 x 128 floats)
    p = moba.MobaParams(4, 4 * 32769, 32769, 8, 8, 128, 128, 3, moba.MOBA_BF16)
    assert 4 * ((32769 + 127) // 128) * 8 * 128 > LIMIT_FLOATS
    assert _raw_call(p) == moba.MOBA_ERR_WORKSPACE
    # 2 sequences x 4096 blocks x 8 kv heads x d=128 x 4 B = 32 MiB > 4 MiB
    p = moba.MobaParams(2, 2 * 65536, 65536, 8, 8, 128, 16, 3, moba.MOBA_BF16)
    assert _raw_call(p) == moba.MOBA_ERR_WORKSPACE
    # within the limit, the null pointers are refused before any launch
    p = moba.MobaParams(4, 4 * 32768, 32768, 8, 8, 128, 128, 3, moba.MOBA_BF16)
    assert _raw_call(p) == moba.MOBA_ERR_INVALID_ARG
    # the prefix-mean gate needs workspace for its scores
    p = moba.MobaParams(1, 1024, 1024, 2, 2, 128, 128, 3, moba.MOBA_BF16, 0, 1)
    assert _raw_call(p) == moba.MOBA_ERR_UNSUPPORTED
