"""Host-side argument checks of the Python binding: shapes and element types
that the C ABI takes on trust (a mismatch would make a kernel read or write
past a buffer) are refused before anything reaches the library. Runs on CPU:
every case fails before a device pointer is needed."""
import pytest
import torch

import long_context_prefill_block_b200 as moba

T, HQ, HKV, D = 64, 4, 2, 128


def _qkv(dtype=torch.bfloat16, t=T, hq=HQ, hkv=HKV, d=D):
    return (torch.zeros(t, hq, d, dtype=dtype), torch.zeros(t, hkv, d, dtype=dtype),
            torch.zeros(t, hkv, d, dtype=dtype))


CU = torch.tensor([0, 40, 64], dtype=torch.int32)


def test_mixed_dtypes_are_refused():
    q, k, v = _qkv()
    with pytest.raises(TypeError, match="dtype"):
        moba.moba_forward(q, k.float(), v, CU, 32, 2)
    with pytest.raises(TypeError, match="dtype"):
        moba.moba_forward(q, k, v.float(), CU, 32, 2)
    with pytest.raises(TypeError, match="dtype"):
        moba.moba_gate_topk(q.float(), k, CU, 32, 2)


@pytest.mark.parametrize("bad", ["k_tokens", "k_dim", "heads", "v_shape", "out_shape"])
def test_shape_mismatches_are_refused(bad):
    q, k, v = _qkv()
    out = None
    if bad == "k_tokens":
        k = torch.zeros(T - 1, HKV, D, dtype=q.dtype)
    elif bad == "k_dim":
        k = torch.zeros(T, HKV, 64, dtype=q.dtype)
    elif bad == "heads":
        k = torch.zeros(T, 3, D, dtype=q.dtype)
        v = torch.zeros(T, 3, D, dtype=q.dtype)
    elif bad == "v_shape":
        v = torch.zeros(T, HKV + 2, D, dtype=q.dtype)
    else:
        out = torch.zeros(T, HQ, 64, dtype=q.dtype)
    with pytest.raises(ValueError):
        moba.moba_forward(q, k, v, CU, 32, 2, out=out)


@pytest.mark.parametrize("cu", [[0, 40, 63], [1, 40, 64], [0, 50, 40, 64], [[0, 64]]])
def test_inconsistent_cu_seqlens_are_refused(cu):
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="cu_seqlens"):
        moba.moba_forward(q, k, v, torch.tensor(cu, dtype=torch.int32), 32, 2)


def test_index_rows_of_the_wrong_shape_are_refused():
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="idx"):
        moba.moba_forward_with_indices(q, k, v, CU, torch.zeros(T, HQ + 1, 2, dtype=torch.int32), 32)
    with pytest.raises(ValueError, match="idx"):
        moba.moba_forward_with_indices(q, k, v, CU, torch.zeros(T, HQ, 2, dtype=torch.int64), 32)


def test_backward_operands_are_checked():
    q, k, v = _qkv()
    out = torch.zeros_like(q)
    lse = torch.zeros(T, HQ, dtype=torch.float32)
    with pytest.raises(ValueError, match="dout"):
        moba.moba_backward(q, k, v, CU, out, lse, torch.zeros(T, HQ, D), 32, 2)
    with pytest.raises(ValueError, match="lse"):
        moba.moba_backward(q, k, v, CU, out, lse[:, :1], torch.zeros_like(q), 32, 2)


def test_consistent_cpu_arguments_reach_the_device_check():
    # well-formed arguments pass the shape checks and stop only at the
    # requirement for CUDA tensors
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="CUDA"):
        moba.moba_forward(q, k, v, CU, 32, 2)


def test_decode_and_meanpool_arguments_are_checked():
    _, k, v = _qkv()
    q = torch.zeros(2, HQ, D, dtype=torch.bfloat16)
    kbar = torch.zeros(2, 2, HKV, D)
    cu_q = torch.tensor([0, 1, 2], dtype=torch.int32)
    with pytest.raises(ValueError):   # q head dim differs from the cache's
        moba.moba_decode(torch.zeros(2, HQ, 64, dtype=torch.bfloat16), k, v, CU, cu_q, kbar, 32, 2)
    with pytest.raises(TypeError):    # cache K and V of different dtypes
        moba.moba_decode(q, k, v.float(), CU, cu_q, kbar, 32, 2)
    with pytest.raises(ValueError, match="cu_seqlens"):
        moba.moba_meanpool(k, torch.tensor([0, 10], dtype=torch.int32), 32)
    with pytest.raises(ValueError, match="cu_seqlens"):
        moba.moba_meanpool_update(k, torch.tensor([0, 70], dtype=torch.int32),
                                  torch.tensor([0, 1], dtype=torch.int32), kbar, 32, 1)
