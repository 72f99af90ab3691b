"""Python binding of libmoba.so, the B200 MoBA prefill forward pass.

Argument marshalling only: every step runs in the library's CUDA kernels.
torch provides device memory and the current stream. The binding refuses to
run if the compiled library is missing; there is no fallback of any kind.

Functions mirror the C ABI of include/moba.h:
    moba_meanpool, moba_meanpool_update, moba_gate_topk, moba_gate_topk_noalloc,
    moba_forward, moba_forward_with_indices, moba_backward, moba_decode,
    dense_causal_forward, moba_workspace_size, moba_num_blocks, moba_device_status,
    moba_selftest_bounded_wait.
Shapes, element types, devices and (when it is on the host) cu_seqlens are
checked here before the call: the C ABI takes them on trust, and a mismatch
would make a kernel read or write past a buffer.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoba.so")

MOBA_OK, MOBA_ERR_INVALID_ARG, MOBA_ERR_UNSUPPORTED, MOBA_ERR_CUDA = 0, -1, -2, -3
MOBA_ERR_TIMEOUT, MOBA_ERR_WORKSPACE, MOBA_ERR_BAD_INDICES, MOBA_ERR_CHECK = -4, -5, -6, -7
MOBA_BF16, MOBA_F32 = 0, 1

EXPORTS = ("moba_num_blocks", "moba_workspace_size", "moba_meanpool", "moba_gate_topk",
           "moba_forward", "moba_forward_with_indices", "dense_causal_forward",
           "moba_device_status", "moba_status_string")


class MobaParams(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("total_tokens", ctypes.c_int),
                ("max_seqlen", ctypes.c_int), ("num_q_heads", ctypes.c_int),
                ("num_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("block_size", ctypes.c_int), ("topk", ctypes.c_int), ("dtype", ctypes.c_int),
                ("routing", ctypes.c_int), ("own_block", ctypes.c_int),
                ("kv_layout", ctypes.c_int)]


class MobaError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn}: {msg} (status {code})")
        self.code = code


_lib = None


def _configure(L: ctypes.CDLL) -> ctypes.CDLL:
    P, V, Z = ctypes.POINTER(MobaParams), ctypes.c_void_p, ctypes.c_size_t
    L.moba_num_blocks.argtypes = [P]
    L.moba_num_blocks.restype = ctypes.c_int
    L.moba_workspace_size.argtypes = [P]
    L.moba_workspace_size.restype = Z
    L.moba_meanpool.argtypes = [P, V, V, V, V]
    L.moba_gate_topk.argtypes = [P, V, V, V, V, V, Z, V]
    L.moba_forward.argtypes = [P, V, V, V, V, V, V, V, Z, V]
    L.moba_forward_with_indices.argtypes = [P, V, V, V, V, V, V, V, V, Z, V]
    L.dense_causal_forward.argtypes = [P, V, V, V, V, V, V, V]
    L.moba_device_status.argtypes = [V, ctypes.c_int]
    L.moba_status_string.argtypes = [ctypes.c_int]
    L.moba_status_string.restype = ctypes.c_char_p
    for name in ("moba_meanpool", "moba_gate_topk", "moba_forward",
                 "moba_forward_with_indices", "dense_causal_forward", "moba_device_status"):
        getattr(L, name).restype = ctypes.c_int
    return L


def lib() -> ctypes.CDLL:
    """The loaded libmoba.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmoba.so not built at {LIB_PATH}; run "
                              "`python -m long_context_prefill_block_b200.build`")
        _lib = _configure(ctypes.CDLL(LIB_PATH))
    return _lib


def use_library(path: str) -> ctypes.CDLL:
    """Route every call of this module through another build of the library
    (the phase-trace build, libmoba_trace.so); must come before the first call."""
    global _lib
    if _lib is not None:
        raise RuntimeError("the library is already loaded")
    if not os.path.exists(path):
        raise ImportError(f"{path} not built")
    _lib = _configure(ctypes.CDLL(path))
    return _lib


def _check(fn: str, code: int) -> None:
    if code != MOBA_OK:
        raise MobaError(fn, code, lib().moba_status_string(code).decode())


def make_params(q: torch.Tensor, k: torch.Tensor, cu_seqlens: torch.Tensor, block_size: int,
                topk: int, max_seqlen: Optional[int] = None,
                shared_routing: bool = False, prefix_mean: bool = False) -> MobaParams:
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    batch = cu_seqlens.numel() - 1
    if max_seqlen is None:
        cu = cu_seqlens.detach().to("cpu", torch.int64)
        max_seqlen = int((cu[1:] - cu[:-1]).max()) if batch > 0 else 0
    if q.dtype == torch.bfloat16:
        dt = MOBA_BF16
    elif q.dtype == torch.float32:
        dt = MOBA_F32
    else:
        raise TypeError(f"unsupported dtype {q.dtype}")
    return MobaParams(batch, T, max_seqlen, Hq, Hkv, d, block_size, topk, dt,
                      1 if shared_routing else 0, 1 if prefix_mean else 0)


def _ptr(x: Optional[torch.Tensor]):
    return None if x is None else ctypes.c_void_p(x.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dev_i32(cu: torch.Tensor, device) -> torch.Tensor:
    return cu.to(device=device, dtype=torch.int32).contiguous()


def _check_inputs(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")
    devs = {t.device for t in ts if t is not None}
    if len(devs) > 1:
        raise ValueError(f"tensors on different devices: {sorted(map(str, devs))}")


def _check_qkv(q, k, v=None, out=None):
    """Shapes and element types the C ABI takes on trust: a mismatch would make the
    kernels read or write past the end of a buffer, so it is refused here."""
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("q and k must be [tokens, heads, head_dim]")
    if k.dtype != q.dtype or (v is not None and v.dtype != q.dtype):
        raise TypeError(f"q, k, v must share one dtype (got {q.dtype}, {k.dtype}"
                        f"{'' if v is None else ', ' + str(v.dtype)})")
    if k.shape[0] != q.shape[0] or k.shape[2] != q.shape[2]:
        raise ValueError(f"k {tuple(k.shape)} does not match q {tuple(q.shape)}")
    if q.shape[1] % k.shape[1] != 0:
        raise ValueError(f"{q.shape[1]} q heads are not a multiple of {k.shape[1]} kv heads")
    if v is not None and v.shape != k.shape:
        raise ValueError(f"v {tuple(v.shape)} does not match k {tuple(k.shape)}")
    if out is not None and (out.shape != q.shape or out.dtype != q.dtype):
        raise ValueError(f"out must be {tuple(q.shape)} {q.dtype}")


def _check_cu(cu_seqlens: torch.Tensor, total_tokens: int) -> None:
    """cu_seqlens already on the host: starts at 0, never decreases, ends at T."""
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be a 1-D tensor [batch + 1]")
    if cu_seqlens.is_cuda:
        return
    cu = cu_seqlens.to(torch.int64)
    if int(cu[0]) != 0 or int(cu[-1]) != total_tokens or bool((cu[1:] < cu[:-1]).any()):
        raise ValueError(f"cu_seqlens must start at 0, not decrease and end at {total_tokens}")


def moba_workspace_size(params: MobaParams) -> int:
    return int(lib().moba_workspace_size(ctypes.byref(params)))


def moba_num_blocks(params: MobaParams) -> int:
    return int(lib().moba_num_blocks(ctypes.byref(params)))


def workspace(params: MobaParams, device) -> torch.Tensor:
    return torch.empty(max(moba_workspace_size(params), 256), dtype=torch.uint8, device=device)


def _packed_view(k: torch.Tensor, head_major: bool) -> torch.Tensor:
    """The [T, Hkv, d] shape of a cache given [Hkv, T, d] when head_major (shape checks only)."""
    if not head_major:
        return k
    if k.dim() != 3:
        raise ValueError("a head-major cache must be [Hkv, T, d]")
    return k.transpose(0, 1)


def moba_meanpool(k: torch.Tensor, cu_seqlens: torch.Tensor, block_size: int,
                  max_seqlen: Optional[int] = None, kv_head_major: bool = False) -> torch.Tensor:
    """Block means fp32 [batch, num_blocks, Hkv, d]. k: [T, Hkv, d], or [Hkv, T, d] with
    kv_head_major (a decode cache laid out head by head)."""
    kp = _packed_view(k, kv_head_major)
    _check_qkv(kp, kp)
    _check_cu(cu_seqlens, kp.shape[0])
    _check_inputs(k)
    p = make_params(kp, kp, cu_seqlens, block_size, 1, max_seqlen)
    p.num_q_heads = p.num_kv_heads
    p.kv_layout = 1 if kv_head_major else 0
    cu = _dev_i32(cu_seqlens, k.device)
    kbar = torch.empty((p.batch, moba_num_blocks(p), p.num_kv_heads, p.head_dim),
                       dtype=torch.float32, device=k.device)
    _check("moba_meanpool", lib().moba_meanpool(ctypes.byref(p), _ptr(k), _ptr(cu), _ptr(kbar),
                                                _stream(k.device)))
    return kbar


def moba_meanpool_update(k_cache: torch.Tensor, cu_seqlens: torch.Tensor, cu_new: torch.Tensor,
                         kbar: torch.Tensor, block_size: int, max_new: int,
                         max_seqlen: Optional[int] = None,
                         kv_head_major: bool = False) -> torch.Tensor:
    """Recompute, in place, the block means kbar [batch, num_blocks, Hkv, d] of the blocks that
    hold each request's last cu_new[r+1] - cu_new[r] cache positions (just appended)."""
    kp = _packed_view(k_cache, kv_head_major)
    _check_qkv(kp, kp)
    _check_cu(cu_seqlens, kp.shape[0])
    _check_inputs(k_cache, kbar)
    p = make_params(kp, kp, cu_seqlens, block_size, 1, max_seqlen)
    p.num_q_heads = p.num_kv_heads
    p.kv_layout = 1 if kv_head_major else 0
    cu = _dev_i32(cu_seqlens, k_cache.device)
    cn = _dev_i32(cu_new, k_cache.device)
    fn = lib().moba_meanpool_update
    fn.argtypes = [ctypes.POINTER(MobaParams)] + [ctypes.c_void_p] * 3 + [ctypes.c_int,
                                                                        ctypes.c_void_p,
                                                                        ctypes.c_void_p]
    fn.restype = ctypes.c_int
    _check("moba_meanpool_update", fn(ctypes.byref(p), _ptr(k_cache), _ptr(cu), _ptr(cn),
                                      int(max_new), _ptr(kbar), _stream(k_cache.device)))
    return kbar


def decode_params(q, k_cache, cu_seqlens, block_size: int, topk: int, max_seqlen=None,
                  shared_routing: bool = False, kv_head_major: bool = False) -> MobaParams:
    """Parameters of a decode step: the cache's shape with q's heads."""
    kp = _packed_view(k_cache, kv_head_major)
    p = make_params(kp, kp, cu_seqlens, block_size, topk, max_seqlen, shared_routing)
    p.num_q_heads = q.shape[1]
    p.kv_layout = 1 if kv_head_major else 0
    return p


def moba_decode(q, k_cache, v_cache, cu_seqlens, cu_q, kbar, block_size: int, topk: int,
                max_seqlen=None, shared_routing: bool = False, return_lse: bool = False,
                return_idx: bool = False, ws: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, kv_head_major: bool = False):
    """Decode step: request r's queries (rows cu_q[r] .. cu_q[r+1]-1 of q [n, Hq, d]) sit at the
    last positions of its cache (tokens cu_seqlens[r] .. cu_seqlens[r+1]-1 of k_cache, v_cache:
    [T, Hkv, d], or [Hkv, T, d] with kv_head_major); kbar: the cache's block means. Returns
    out [n, Hq, d] (and lse [n, Hq], idx [n, Hq, topk])."""
    kp, vp = _packed_view(k_cache, kv_head_major), _packed_view(v_cache, kv_head_major)
    _check_qkv(kp, kp, vp)
    if q.dim() != 3 or q.dtype != k_cache.dtype or q.shape[2] != k_cache.shape[2]:
        raise ValueError("q must be [n, Hq, d] in the cache's dtype and head dim")
    _check_cu(cu_seqlens, kp.shape[0])
    _check_inputs(q, k_cache, v_cache, kbar, out)
    L = lib()
    p = decode_params(q, k_cache, cu_seqlens, block_size, topk, max_seqlen, shared_routing,
                      kv_head_major)
    n = q.shape[0]
    cu = _dev_i32(cu_seqlens, q.device)
    cq = _dev_i32(cu_q, q.device)
    L.moba_decode_workspace_size.argtypes = [ctypes.POINTER(MobaParams), ctypes.c_int]
    L.moba_decode_workspace_size.restype = ctypes.c_size_t
    if ws is None:
        ws = torch.empty(max(int(L.moba_decode_workspace_size(ctypes.byref(p), n)), 256),
                         dtype=torch.uint8, device=q.device)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device) if return_lse else None
    idx = (torch.empty((n, q.shape[1], topk), dtype=torch.int32, device=q.device)
           if return_idx else None)
    fn = L.moba_decode
    V = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(MobaParams), V, V, V, V, V, ctypes.c_int, V, V, V, V, V,
                   ctypes.c_size_t, V]
    fn.restype = ctypes.c_int
    _check("moba_decode", fn(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cu),
                             _ptr(cq), n, _ptr(kbar), _ptr(out), _ptr(lse), _ptr(idx), _ptr(ws),
                             ws.numel(), _stream(q.device)))
    res = (out,)
    if return_lse:
        res += (lse,)
    if return_idx:
        res += (idx,)
    return res[0] if len(res) == 1 else res


def moba_gate_topk(q, k, cu_seqlens, block_size: int, topk: int, max_seqlen=None,
                   ws: Optional[torch.Tensor] = None, shared_routing: bool = False,
                   prefix_mean: bool = False) -> torch.Tensor:
    """Chosen blocks per (token, q head): int32 [T, Hq, topk], ascending, -1 padded.
    shared_routing: the q heads of a kv head's group share the blocks of their mean score.
    prefix_mean: the own block is scored by the mean of its keys up to the query and competes
    for the k slots instead of being forced."""
    _check_qkv(q, k)
    _check_cu(cu_seqlens, q.shape[0])
    _check_inputs(q, k)
    p = make_params(q, k, cu_seqlens, block_size, topk, max_seqlen, shared_routing, prefix_mean)
    cu = _dev_i32(cu_seqlens, q.device)
    ws = workspace(p, q.device) if ws is None else ws
    idx = torch.empty((p.total_tokens, p.num_q_heads, topk), dtype=torch.int32, device=q.device)
    _check("moba_gate_topk", lib().moba_gate_topk(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(cu),
                                                  _ptr(idx), _ptr(ws), ws.numel(),
                                                  _stream(q.device)))
    return idx


def moba_gate_topk_noalloc(q, k, cu_seqlens, block_size: int, topk: int, max_seqlen=None,
                           idx: Optional[torch.Tensor] = None,
                           shared_routing: bool = False) -> torch.Tensor:
    """moba_gate_topk without a workspace, for callers that cannot allocate
    device memory: the block means use a fixed 4 MiB array inside the
    library (see include/moba.h for the limit and the sharing rules)."""
    _check_qkv(q, k)
    _check_cu(cu_seqlens, q.shape[0])
    if idx is not None and (idx.shape != (q.shape[0], q.shape[1], topk) or idx.dtype != torch.int32):
        raise ValueError(f"idx must be int32 {(q.shape[0], q.shape[1], topk)}")
    _check_inputs(q, k, idx)
    L = lib()
    fn = L.moba_gate_topk_noalloc
    fn.argtypes = [ctypes.POINTER(MobaParams)] + [ctypes.c_void_p] * 5
    fn.restype = ctypes.c_int
    p = make_params(q, k, cu_seqlens, block_size, topk, max_seqlen, shared_routing)
    cu = _dev_i32(cu_seqlens, q.device)
    if idx is None:
        idx = torch.empty((p.total_tokens, p.num_q_heads, topk), dtype=torch.int32,
                          device=q.device)
    _check("moba_gate_topk_noalloc", fn(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(cu), _ptr(idx),
                                        _stream(q.device)))
    return idx


def moba_forward(q, k, v, cu_seqlens, block_size: int, topk: int, max_seqlen=None,
                 return_lse: bool = False, ws: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None, shared_routing: bool = False,
                 prefix_mean: bool = False):
    """MoBA prefill forward: out [T, Hq, d] (input dtype) and optionally lse [T, Hq].
    shared_routing: the q heads of a kv head's group share the blocks of their mean score.
    prefix_mean: the own block is scored by the mean of its keys up to the query and competes
    for the k slots instead of being forced."""
    _check_qkv(q, k, v, out)
    _check_cu(cu_seqlens, q.shape[0])
    _check_inputs(q, k, v, out)
    p = make_params(q, k, cu_seqlens, block_size, topk, max_seqlen, shared_routing, prefix_mean)
    cu = _dev_i32(cu_seqlens, q.device)
    ws = workspace(p, q.device) if ws is None else ws
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device) if return_lse else None
    _check("moba_forward", lib().moba_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(cu),
                                              _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                              _stream(q.device)))
    return (out, lse) if return_lse else out


def moba_backward(q, k, v, cu_seqlens, out, lse, dout, block_size: int, topk: int,
                  idx: Optional[torch.Tensor] = None, max_seqlen=None,
                  shared_routing: bool = False, prefix_mean: bool = False):
    """Gradients of sum(dout * out) through the chosen blocks: (dq [T,Hq,d], dk, dv [T,Hkv,d])
    in fp32. out, lse: the forward's results; idx: its index rows, or None to run the gate
    again."""
    _check_qkv(q, k, v, out)
    _check_cu(cu_seqlens, q.shape[0])
    if dout.shape != q.shape or dout.dtype != q.dtype:
        raise ValueError(f"dout must be {tuple(q.shape)} {q.dtype}")
    if lse.shape != q.shape[:2] or lse.dtype != torch.float32:
        raise ValueError(f"lse must be float32 {tuple(q.shape[:2])}")
    if idx is not None and (idx.shape != (q.shape[0], q.shape[1], topk) or idx.dtype != torch.int32):
        raise ValueError(f"idx must be int32 {(q.shape[0], q.shape[1], topk)}")
    _check_inputs(q, k, v, out, dout, lse, idx)
    L = lib()
    p = make_params(q, k, cu_seqlens, block_size, topk, max_seqlen, shared_routing, prefix_mean)
    cu = _dev_i32(cu_seqlens, q.device)
    L.moba_backward_workspace_size.argtypes = [ctypes.POINTER(MobaParams), ctypes.c_int]
    L.moba_backward_workspace_size.restype = ctypes.c_size_t
    nbytes = int(L.moba_backward_workspace_size(ctypes.byref(p), 0 if idx is None else 1))
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    fn = L.moba_backward
    fn.argtypes = [ctypes.POINTER(MobaParams)] + [ctypes.c_void_p] * 12 + [ctypes.c_size_t,
                                                                         ctypes.c_void_p]
    fn.restype = ctypes.c_int
    _check("moba_backward", fn(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(cu), _ptr(out),
                               _ptr(lse), _ptr(dout), _ptr(idx), _ptr(dq), _ptr(dk), _ptr(dv),
                               _ptr(ws), ws.numel(), _stream(q.device)))
    return dq, dk, dv


def moba_forward_with_indices(q, k, v, cu_seqlens, idx, block_size: int, max_seqlen=None,
                              return_lse: bool = False, ws: Optional[torch.Tensor] = None,
                              prefix_mean: bool = False):
    """MoBA forward with caller-chosen blocks idx int32 [T, Hq, topk] (canonical form; with
    prefix_mean a row may leave out its own block and then reads none of it)."""
    _check_qkv(q, k, v)
    _check_cu(cu_seqlens, q.shape[0])
    if idx.dim() != 3 or idx.shape[:2] != q.shape[:2] or idx.dtype != torch.int32:
        raise ValueError(f"idx must be int32 [{q.shape[0]}, {q.shape[1]}, topk]")
    _check_inputs(q, k, v, idx)
    p = make_params(q, k, cu_seqlens, block_size, idx.shape[2], max_seqlen, prefix_mean=prefix_mean)
    cu = _dev_i32(cu_seqlens, q.device)
    ws = workspace(p, q.device) if ws is None else ws
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device) if return_lse else None
    _check("moba_forward_with_indices",
           lib().moba_forward_with_indices(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(cu),
                                           _ptr(idx), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                           _stream(q.device)))
    return (out, lse) if return_lse else out


def dense_causal_forward(q, k, v, cu_seqlens, max_seqlen=None, return_lse: bool = False,
                         out: Optional[torch.Tensor] = None):
    """Dense causal attention over each sequence (the comparison kernel)."""
    _check_qkv(q, k, v, out)
    _check_cu(cu_seqlens, q.shape[0])
    _check_inputs(q, k, v, out)
    p = make_params(q, k, cu_seqlens, 128, 1, max_seqlen)
    cu = _dev_i32(cu_seqlens, q.device)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device) if return_lse else None
    _check("dense_causal_forward",
           lib().dense_causal_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(cu),
                                      _ptr(out), _ptr(lse), _stream(q.device)))
    return (out, lse) if return_lse else out


def moba_selftest_bounded_wait(device=None) -> int:
    """Run the bounded-wait self-test kernel; returns the kernel's result code
    (2 = the wait gave up as it must). Read moba_device_status() afterwards."""
    fn = lib().moba_selftest_bounded_wait
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    done = torch.zeros(1, dtype=torch.int32, device=device or "cuda")
    _check("moba_selftest_bounded_wait", fn(_ptr(done), _stream(done.device)))
    torch.cuda.synchronize(done.device)
    return int(done.item())


def moba_device_status(device=None, clear: bool = True) -> int:
    """Synchronise the current stream and return (and clear) the device status word."""
    return int(lib().moba_device_status(_stream(device), int(clear)))
