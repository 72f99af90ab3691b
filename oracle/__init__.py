"""fp64 CPU oracle for the MoBA prefill forward pass (ctypes binding).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
bench's CPU-baseline leg. The CUDA path never imports it and shares no code
with it. The arithmetic lives in moba_oracle.cpp; this module only marshals
arrays. Inputs are passed as stored (bf16 bit patterns or fp32), and the
oracle widens them exactly to double.

Citations (page title, section, equation) are in moba_oracle.cpp. Every
function here has at least one pin in tests/test_oracle_pins.py.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None
BF16, F32 = 0, 1


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P, I, L = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        sig = {
            "oracle_num_threads": [],
            "oracle_meanpool": [P, I, P, I, I, I, I, I, P],
            "oracle_gate_topk": [P, P, I, P, I, I, I, I, I, I, P, P],
            "oracle_forward": [P, P, P, I, P, I, I, I, I, I, I, P, P, P, P, P],
            "oracle_forward_rows": [P, P, P, I, P, I, I, I, I, I, I, P, L, P, P, P, P, P, P],
            "oracle_forward_mask": [P, P, P, I, P, I, I, I, I, I, I, P, P],
            "oracle_forward_two_branch": [P, P, P, I, P, I, I, I, I, I, I, I, P],
            "oracle_dense_causal": [P, P, P, I, P, I, I, I, I, P, P],
            "oracle_gate_topk_routed": [P, P, I, P, I, I, I, I, I, I, I, P, P],
            "oracle_forward_routed": [P, P, P, I, P, I, I, I, I, I, I, I, P, P, P, P, P],
            "oracle_forward_rows_routed": [P, P, P, I, P, I, I, I, I, I, I, I, P, L, P, P, P, P, P,
                                           P],
            "oracle_backward_routed": [P, P, P, P, I, P, I, I, I, I, I, I, I, P, P, P, P],
            "oracle_forward_mask_routed": [P, P, P, I, P, I, I, I, I, I, I, I, P, P],
        }
        for name, args in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def _raw(x):
    """(contiguous numpy array of stored bits, dtype code) for a torch tensor or array."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().contiguous().cpu()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), F32
            if x.dtype == torch.float64:
                return x.to(torch.float32).numpy(), F32
            raise TypeError(f"unsupported dtype {x.dtype}")
    except ImportError:
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.float64:
        return x.astype(np.float32), F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"unsupported dtype {x.dtype}")


def _i32(x):
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _routing(shared_routing, prefix_mean):
    """Routing flags of the *_routed entry points: bit 0 = one choice per kv
    head's group (the group's mean score), bit 1 = the own block scored by the
    mean of its keys up to the query instead of forced."""
    return int(bool(shared_routing)) | (int(bool(prefix_mean)) << 1)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _qkv(q, k, v):
    qr, dt = _raw(q)
    kr, dk = _raw(k)
    vr, dv = (None, dt) if v is None else _raw(v)
    if not (dt == dk == dv):
        raise TypeError("q, k, v must share one dtype")
    return qr, kr, vr, dt


def num_threads() -> int:
    return _lib().oracle_num_threads()


def meanpool(k, cu_seqlens, block_size):
    """Block means [batch, nb_max, Hkv, d] (float64)."""
    kr, dt = _raw(k)
    cu = _i32(cu_seqlens)
    T, Hkv, d = kr.shape
    batch = len(cu) - 1
    lens = np.diff(cu)
    nb_max = int(((lens + block_size - 1) // block_size).max()) if batch else 0
    out = np.zeros((batch, nb_max, Hkv, d), dtype=np.float64)
    rc = _lib().oracle_meanpool(_ptr(kr), dt, _ptr(cu), batch, Hkv, d, block_size, nb_max, _ptr(out))
    if rc:
        raise ValueError("oracle_meanpool: invalid arguments")
    return out


def gate_topk(q, k, cu_seqlens, block_size, topk, shared_routing=False, prefix_mean=False):
    """(idx [T, Hq, topk] int32, gap [T, Hq] float64). shared_routing: every
    query head of a kv head's group takes the blocks chosen by the group's
    mean score. prefix_mean: the own block is scored by the mean of its keys
    up to the query and competes for the k slots instead of being forced."""
    qr, kr, _, dt = _qkv(q, k, None)
    cu = _i32(cu_seqlens)
    T, Hq, d = qr.shape
    Hkv = kr.shape[1]
    idx = np.full((T, Hq, topk), -1, dtype=np.int32)
    gap = np.zeros((T, Hq), dtype=np.float64)
    rc = _lib().oracle_gate_topk_routed(_ptr(qr), _ptr(kr), dt, _ptr(cu), len(cu) - 1, Hq, Hkv, d,
                                        block_size, topk, _routing(shared_routing, prefix_mean),
                                        _ptr(idx),
                                        _ptr(gap))
    if rc:
        raise ValueError("oracle_gate_topk: invalid arguments")
    return idx, gap


def forward(q, k, v, cu_seqlens, block_size, topk, indices=None, shared_routing=False,
            prefix_mean=False):
    """Full forward by definition: (out [T,Hq,d], lse [T,Hq], idx [T,Hq,topk], nkeys [T,Hq])."""
    qr, kr, vr, dt = _qkv(q, k, v)
    cu = _i32(cu_seqlens)
    T, Hq, d = qr.shape
    Hkv = kr.shape[1]
    idx_in = None if indices is None else _i32(indices)
    out = np.zeros((T, Hq, d), dtype=np.float64)
    lse = np.zeros((T, Hq), dtype=np.float64)
    idx = np.full((T, Hq, topk), -1, dtype=np.int32)
    nkeys = np.zeros((T, Hq), dtype=np.int64)
    rc = _lib().oracle_forward_routed(_ptr(qr), _ptr(kr), _ptr(vr), dt, _ptr(cu), len(cu) - 1, Hq,
                                      Hkv, d, block_size, topk,
                                      _routing(shared_routing, prefix_mean), _ptr(idx_in), _ptr(out), _ptr(lse), _ptr(idx), _ptr(nkeys))
    if rc:
        raise ValueError("oracle_forward: invalid arguments")
    return out, lse, idx, nkeys


def backward(q, k, v, dout, cu_seqlens, block_size, topk, indices=None, shared_routing=False,
             prefix_mean=False):
    """Gradients of sum(dout * out) by definition: (dq [T,Hq,d], dk [T,Hkv,d], dv [T,Hkv,d]),
    float64. The block choice (a hard top-k) passes no gradient."""
    qr, kr, vr, dt = _qkv(q, k, v)
    dr, dd = _raw(dout)
    if dd != dt or dr.shape != qr.shape:
        raise TypeError("dout must have q's shape and dtype")
    cu = _i32(cu_seqlens)
    T, Hq, d = qr.shape
    Hkv = kr.shape[1]
    idx_in = None if indices is None else _i32(indices)
    dq = np.zeros((T, Hq, d), dtype=np.float64)
    dk = np.zeros((T, Hkv, d), dtype=np.float64)
    dv = np.zeros((T, Hkv, d), dtype=np.float64)
    rc = _lib().oracle_backward_routed(_ptr(qr), _ptr(kr), _ptr(vr), _ptr(dr), dt, _ptr(cu),
                                       len(cu) - 1, Hq, Hkv, d, block_size, topk,
                                       _routing(shared_routing, prefix_mean), _ptr(idx_in), _ptr(dq),
                                       _ptr(dk),
                                       _ptr(dv))
    if rc:
        raise ValueError("oracle_backward: invalid arguments")
    return dq, dk, dv


def forward_rows(q, k, v, cu_seqlens, block_size, topk, rows, indices=None, q_rows=None,
                 num_q_heads=None, shared_routing=False, prefix_mean=False):
    """Sampled forward on rows (row = t*Hq + h): (out [n,d], lse [n], idx [n,topk], gap [n]).

    With q_rows ([n, d], the q vectors of the listed rows) q may be None and
    num_q_heads gives Hq; then the caller need not hold all of q."""
    if q_rows is not None:
        qr, dt = _raw(q_rows)
        kr, dk = _raw(k)
        vr, dv = _raw(v)
        if not (dt == dk == dv):
            raise TypeError("q_rows, k, v must share one dtype")
        Hq, d = int(num_q_heads), qr.shape[-1]
        T = kr.shape[0]
        qbase = None
    else:
        qr, kr, vr, dt = _qkv(q, k, v)
        T, Hq, d = qr.shape
        qbase = qr
    cu = _i32(cu_seqlens)
    Hkv = kr.shape[1]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n = len(rows)
    idx_in = None if indices is None else _i32(indices)
    out = np.zeros((n, d), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    idx = np.full((n, topk), -1, dtype=np.int32)
    gap = np.zeros(n, dtype=np.float64)
    rc = _lib().oracle_forward_rows_routed(_ptr(qbase), _ptr(kr), _ptr(vr), dt, _ptr(cu),
                                           len(cu) - 1, Hq, Hkv, d, block_size, topk,
                                           _routing(shared_routing, prefix_mean), _ptr(rows), n,
                                           _ptr(idx_in),
                                           _ptr(out), _ptr(lse), _ptr(idx), _ptr(gap),
                                           _ptr(qr) if q_rows is not None else None)
    if rc:
        raise ValueError("oracle_forward_rows: invalid arguments")
    return out, lse, idx, gap


def forward_mask(q, k, v, cu_seqlens, block_size, topk, indices=None, prefix_mean=False):
    """moba_naive view: dense boolean mask + masked dense softmax. out [T,Hq,d]."""
    qr, kr, vr, dt = _qkv(q, k, v)
    cu = _i32(cu_seqlens)
    T, Hq, d = qr.shape
    Hkv = kr.shape[1]
    idx_in = None if indices is None else _i32(indices)
    out = np.zeros((T, Hq, d), dtype=np.float64)
    rc = _lib().oracle_forward_mask_routed(_ptr(qr), _ptr(kr), _ptr(vr), dt, _ptr(cu), len(cu) - 1,
                                           Hq, Hkv, d, block_size, topk, _routing(False, prefix_mean),
                                           _ptr(idx_in), _ptr(out))
    if rc:
        raise ValueError("oracle_forward_mask: invalid arguments")
    return out


def forward_two_branch(q, k, v, cu_seqlens, block_size, topk, naive_sum=False):
    """Current + history branches merged by eq.(7)-(8) (or the wrong naive sum). out [T,Hq,d]."""
    qr, kr, vr, dt = _qkv(q, k, v)
    cu = _i32(cu_seqlens)
    T, Hq, d = qr.shape
    Hkv = kr.shape[1]
    out = np.zeros((T, Hq, d), dtype=np.float64)
    rc = _lib().oracle_forward_two_branch(_ptr(qr), _ptr(kr), _ptr(vr), dt, _ptr(cu), len(cu) - 1,
                                          Hq, Hkv, d, block_size, topk, int(naive_sum), _ptr(out))
    if rc:
        raise ValueError("oracle_forward_two_branch: invalid arguments")
    return out


def dense_causal(q, k, v, cu_seqlens):
    """Dense causal softmax attention: (out [T,Hq,d], lse [T,Hq])."""
    qr, kr, vr, dt = _qkv(q, k, v)
    cu = _i32(cu_seqlens)
    T, Hq, d = qr.shape
    Hkv = kr.shape[1]
    out = np.zeros((T, Hq, d), dtype=np.float64)
    lse = np.zeros((T, Hq), dtype=np.float64)
    rc = _lib().oracle_dense_causal(_ptr(qr), _ptr(kr), _ptr(vr), dt, _ptr(cu), len(cu) - 1, Hq,
                                    Hkv, d, _ptr(out), _ptr(lse))
    if rc:
        raise ValueError("oracle_dense_causal: invalid arguments")
    return out, lse
