"""ctypes binding of libmoba.so (the C ABI declared in include/moba.h).

Argument marshalling only: shapes are read off the tensors, pointers and the
current CUDA stream are passed through, and every step of the forward runs in
the library's kernels.  There is no CPU or PyTorch fallback: if libmoba.so is
missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOBA_DEBUG=1 selects the bounds-checked build (libmoba_debug.so: index
# checks, workspace guards); it must have been built with build --debug.
LIB_PATH = os.path.join(_PKG, "libmoba_debug.so" if os.environ.get("MOBA_DEBUG") == "1"
                        else "libmoba.so")

STATUS = {
    0: "MOBA_OK",
    1: "MOBA_ERR_INVALID_ARG",
    2: "MOBA_ERR_UNSUPPORTED",
    3: "MOBA_ERR_WORKSPACE",
    4: "MOBA_ERR_CUDA",
    5: "MOBA_ERR_TIMEOUT",
    6: "MOBA_ERR_BAD_SEQLENS",
    7: "MOBA_ERR_BAD_SELECTION",
    8: "MOBA_ERR_BOUNDS",
    9: "MOBA_ERR_CANARY",
}

EXPORTS = ("moba_status_string", "moba_workspace_size", "moba_gate", "moba_forward",
           "moba_forward_traced", "moba_full_workspace_size", "moba_forward_full",
           "moba_decode_workspace_size", "moba_decode_init", "moba_decode",
           "moba_backward_workspace_size", "moba_backward",
           "moba_gate_noalloc", "moba_gate_noalloc_check", "moba_check",
           "moba_debug_attention_wait_test", "moba_debug_build", "moba_debug_poison",
           "moba_debug_error_info")


class MobaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoba.so once.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m block_sparse_long_11_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    c_int, c_size, c_void, c_float = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float
    L.moba_status_string.argtypes = [c_int]
    L.moba_status_string.restype = ctypes.c_char_p
    L.moba_workspace_size.argtypes = [c_int] * 8
    L.moba_workspace_size.restype = c_size
    L.moba_gate.argtypes = [c_void, c_void, c_void, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                            c_void, c_void, c_size, c_void]
    L.moba_gate.restype = c_int
    L.moba_forward.argtypes = [c_void, c_void, c_void, c_void, c_int, c_int, c_int, c_int, c_int,
                               c_int, c_int, c_float, c_void, c_void, c_void, c_int, c_void, c_size,
                               c_void]
    L.moba_forward.restype = c_int
    L.moba_forward_traced.argtypes = L.moba_forward.argtypes + [c_void, c_int]
    L.moba_forward_traced.restype = c_int
    L.moba_full_workspace_size.argtypes = [c_int] * 5
    L.moba_full_workspace_size.restype = c_size
    L.moba_forward_full.argtypes = [c_void, c_void, c_void, c_void, c_int, c_int, c_int, c_int,
                                    c_int, c_float, c_void, c_void, c_void, c_size, c_void]
    L.moba_forward_full.restype = c_int
    L.moba_decode_workspace_size.argtypes = [c_int] * 7
    L.moba_decode_workspace_size.restype = c_size
    L.moba_decode_init.argtypes = [c_void, c_void, c_int, c_int, c_int, c_int, c_int, c_void,
                                   c_void, c_size, c_void]
    L.moba_decode_init.restype = c_int
    L.moba_decode.argtypes = [c_void, c_void, c_void, c_void, c_int, c_int, c_int, c_int, c_int,
                              c_int, c_int, c_float, c_void, c_void, c_void, c_void, c_void,
                              c_size, c_void]
    L.moba_decode.restype = c_int
    L.moba_backward_workspace_size.argtypes = [c_int] * 8
    L.moba_backward_workspace_size.restype = c_size
    L.moba_backward.argtypes = [c_void, c_void, c_void, c_void, c_void, c_void, c_void, c_void,
                                c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_float, c_void,
                                c_void, c_void, c_int, c_void, c_size, c_void]
    L.moba_backward.restype = c_int
    L.moba_check.argtypes = [c_void, c_void]
    L.moba_check.restype = c_int
    L.moba_gate_noalloc.argtypes = [c_void, c_void, c_void, c_int, c_int, c_int, c_int, c_int,
                                    c_int, c_int, c_void, c_void]
    L.moba_gate_noalloc.restype = c_int
    L.moba_gate_noalloc_check.argtypes = [c_void]
    L.moba_gate_noalloc_check.restype = c_int
    L.moba_debug_attention_wait_test.argtypes = [c_int]
    L.moba_debug_attention_wait_test.restype = c_int
    L.moba_debug_build.argtypes = []
    L.moba_debug_build.restype = c_int
    L.moba_debug_poison.argtypes = [c_int]
    L.moba_debug_poison.restype = c_int
    L.moba_debug_error_info.argtypes = [c_void, c_void, ctypes.POINTER(c_int)]
    L.moba_debug_error_info.restype = c_int
    _lib = L
    return L


def moba_status_string(code: int) -> str:
    return lib().moba_status_string(int(code)).decode()


def _stream_ptr(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check_qkv(q, k, v=None):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t is None:
            continue
        if t.dtype != torch.bfloat16 or t.dim() != 3 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor of rank 3 [T, H, d]")
    if k.shape[0] != q.shape[0] or k.shape[2] != q.shape[2]:
        raise ValueError("q and k disagree on T or head_dim")
    if v is not None and v.shape != k.shape:
        raise ValueError("v must have the shape of k")


def _check_cu(cu, device):
    if cu.dtype != torch.int32 or cu.dim() != 1 or not cu.is_contiguous() or cu.device != device:
        raise ValueError("cu_seqlens must be a contiguous int32 tensor on the device of q")


def moba_workspace_size(total_tokens: int, n_seqs: int, n_heads: int, n_kv_heads: int,
                        head_dim: int, block_size: int, topk: int, chunk_tokens: int = 0) -> int:
    n = lib().moba_workspace_size(total_tokens, n_seqs, n_heads, n_kv_heads, head_dim, block_size,
                                  topk, chunk_tokens)
    if n == 0:
        raise MobaError(2, "moba_workspace_size")
    return int(n)


class Workspace:
    """Device workspace (allocated by PyTorch) reused across calls of one shape."""

    def __init__(self):
        self.buf: Optional[torch.Tensor] = None

    def get(self, nbytes: int, device) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes or self.buf.device != device:
            self.buf = None
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        return self.buf


_default_ws = Workspace()


def moba_gate(q, k, cu_seqlens, block_size: int, topk: int, workspace: Optional[Workspace] = None,
              out: Optional[torch.Tensor] = None):
    """Gate alone: selected block indices idx [T, Hq, topk] (int32, ascending, -1 padded)."""
    _check_qkv(q, k)
    _check_cu(cu_seqlens, q.device)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    n_seqs = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((T, Hq, topk), dtype=torch.int32, device=q.device)
    nbytes = moba_workspace_size(T, n_seqs, Hq, Hkv, d, block_size, topk, 1)
    ws = (workspace or _default_ws).get(nbytes, q.device)
    rc = lib().moba_gate(q.data_ptr(), k.data_ptr(), cu_seqlens.data_ptr(), n_seqs, T, Hq, Hkv, d,
                         block_size, topk, out.data_ptr(), ws.data_ptr(), ws.numel(),
                         _stream_ptr(q.device))
    if rc != 0:
        raise MobaError(rc, "moba_gate")
    return out


def moba_gate_noalloc(q, k, cu_seqlens, block_size: int, topk: int,
                      out: Optional[torch.Tensor] = None):
    """moba_gate with the library's static device scratch instead of a workspace.

    For callers that must not allocate device memory while the gate runs; the
    index tensor (out) is still the caller's.  Calls on one device share the
    scratch, so calls that overlap on the GPU race.
    """
    _check_qkv(q, k)
    _check_cu(cu_seqlens, q.device)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    n_seqs = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((T, Hq, topk), dtype=torch.int32, device=q.device)
    rc = lib().moba_gate_noalloc(q.data_ptr(), k.data_ptr(), cu_seqlens.data_ptr(), n_seqs, T, Hq,
                                 Hkv, d, block_size, topk, out.data_ptr(), _stream_ptr(q.device))
    if rc != 0:
        raise MobaError(rc, "moba_gate_noalloc")
    return out


PARTIAL_BUDGET_BYTES = 48 << 30


def default_chunk_tokens(total_tokens: int, n_heads: int, head_dim: int, topk: int,
                         budget_bytes: int = PARTIAL_BUDGET_BYTES) -> int:
    """Query tokens per pass so the partial-output buffer stays within budget.

    Each query token needs n_heads * topk partial slots of (2 * head_dim + 4)
    bytes.  The tokens are split into equal passes (0 = a single pass).
    """
    per_token = n_heads * topk * (2 * head_dim + 4)
    if total_tokens * per_token <= budget_bytes:
        return 0
    n_pass = -(-total_tokens * per_token // budget_bytes)
    return -(-total_tokens // n_pass)


def moba_forward(q, k, v, cu_seqlens, block_size: int, topk: int, softmax_scale: float = 0.0,
                 chunk_tokens: Optional[int] = None, workspace: Optional[Workspace] = None,
                 return_idx: bool = False, out=None, lse=None, idx=None, stage_events=None):
    """MoBA causal prefill forward.  Returns (out [T, Hq, d] bf16, lse [T, Hq] fp32[, idx]).

    chunk_tokens: query tokens per pass of the partial buffer; None picks
    default_chunk_tokens(), 0 means one pass.
    stage_events: optional list of already-recorded torch.cuda.Event objects
    (enable_timing=True), re-recorded at the stage boundaries that
    moba_forward_traced documents.
    """
    _check_qkv(q, k, v)
    _check_cu(cu_seqlens, q.device)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    n_seqs = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    if return_idx and idx is None:
        idx = torch.empty((T, Hq, topk), dtype=torch.int32, device=q.device)
    if chunk_tokens is None:
        chunk_tokens = default_chunk_tokens(T, Hq, d, topk)
    nbytes = moba_workspace_size(T, n_seqs, Hq, Hkv, d, block_size, topk, chunk_tokens)
    ws = (workspace or _default_ws).get(nbytes, q.device)
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens.data_ptr(), n_seqs, T, Hq, Hkv, d,
            block_size, topk, float(softmax_scale), out.data_ptr(), lse.data_ptr(),
            idx.data_ptr() if idx is not None else None, chunk_tokens, ws.data_ptr(), ws.numel(),
            _stream_ptr(q.device))
    if stage_events is None:
        rc = lib().moba_forward(*args)
    else:
        handles = (ctypes.c_void_p * len(stage_events))(*[e.cuda_event for e in stage_events])
        rc = lib().moba_forward_traced(*args, handles, len(stage_events))
    if rc != 0:
        raise MobaError(rc, "moba_forward")
    return (out, lse, idx) if return_idx else (out, lse)


def moba_full_workspace_size(total_tokens: int, n_seqs: int, n_heads: int, n_kv_heads: int,
                             head_dim: int) -> int:
    n = lib().moba_full_workspace_size(total_tokens, n_seqs, n_heads, n_kv_heads, head_dim)
    if n == 0:
        raise MobaError(2, "moba_full_workspace_size")
    return int(n)


def moba_forward_full(q, k, v, cu_seqlens, softmax_scale: float = 0.0,
                      workspace: Optional[Workspace] = None, out=None, lse=None):
    """Dense causal attention (every key from the sequence start up to the
    query) through the library's attention kernel: what moba_forward gives
    when top-k covers every block.  Returns (out [T, Hq, d] bf16, lse [T, Hq])."""
    _check_qkv(q, k, v)
    _check_cu(cu_seqlens, q.device)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    n_seqs = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    nbytes = moba_full_workspace_size(T, n_seqs, Hq, Hkv, d)
    ws = (workspace or _default_ws).get(nbytes, q.device)
    rc = lib().moba_forward_full(q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens.data_ptr(),
                                 n_seqs, T, Hq, Hkv, d, float(softmax_scale), out.data_ptr(),
                                 lse.data_ptr(), ws.data_ptr(), ws.numel(), _stream_ptr(q.device))
    if rc != 0:
        raise MobaError(rc, "moba_forward_full")
    return out, lse


def _check_cache(kc, vc=None):
    for name, t in (("k_cache", kc), ("v_cache", vc)):
        if t is None:
            continue
        if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor [n_seqs, max_len, Hkv, d]")
    if vc is not None and vc.shape != kc.shape:
        raise ValueError("v_cache must have the shape of k_cache")


def decode_kbar_cache(k_cache, block_size: int) -> torch.Tensor:
    """An uninitialised block-mean cache [n_seqs, max_len // block_size, Hkv, d] fp32."""
    n, max_len, Hkv, d = k_cache.shape
    return torch.empty((n, max_len // block_size, Hkv, d), dtype=torch.float32,
                       device=k_cache.device)


def moba_decode_init(k_cache, seqlens, block_size: int, kbar=None,
                     workspace: Optional[Workspace] = None):
    """Means of every full block of every sequence of the cache (returns kbar)."""
    _check_cache(k_cache)
    _check_cu(seqlens, k_cache.device)
    n, max_len, Hkv, d = k_cache.shape
    if kbar is None:
        kbar = decode_kbar_cache(k_cache, block_size)
    ws = (workspace or _default_ws).get(256, k_cache.device)
    rc = lib().moba_decode_init(k_cache.data_ptr(), seqlens.data_ptr(), n, max_len, Hkv, d,
                                block_size, kbar.data_ptr() if kbar.numel() else None,
                                ws.data_ptr(), ws.numel(), _stream_ptr(k_cache.device))
    if rc != 0:
        raise MobaError(rc, "moba_decode_init")
    return kbar


def moba_decode(q, k_cache, v_cache, seqlens, kbar, block_size: int, topk: int,
                softmax_scale: float = 0.0, workspace: Optional[Workspace] = None,
                return_idx: bool = False, out=None, lse=None, idx=None):
    """One decode step: q [n_seqs, Hq, d] (the new tokens, whose k and v are
    already at position seqlens[s] - 1 of the caches).  Returns (out, lse[, idx])
    and extends kbar when a new token completes a block."""
    _check_cache(k_cache, v_cache)
    _check_cu(seqlens, q.device)
    n, max_len, Hkv, d = k_cache.shape
    if q.dtype != torch.bfloat16 or q.dim() != 3 or not q.is_contiguous() or q.shape[0] != n \
            or q.shape[2] != d:
        raise ValueError("q must be a contiguous bf16 tensor [n_seqs, Hq, d] matching the cache")
    Hq = q.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((n, Hq), dtype=torch.float32, device=q.device)
    if return_idx and idx is None:
        idx = torch.empty((n, Hq, topk), dtype=torch.int32, device=q.device)
    nbytes = lib().moba_decode_workspace_size(n, max_len, Hq, Hkv, d, block_size, topk)
    if nbytes == 0:
        raise MobaError(2, "moba_decode_workspace_size")
    ws = (workspace or _default_ws).get(int(nbytes), q.device)
    rc = lib().moba_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seqlens.data_ptr(),
                           n, max_len, Hq, Hkv, d, block_size, topk, float(softmax_scale),
                           kbar.data_ptr() if kbar is not None and kbar.numel() else None,
                           out.data_ptr(), lse.data_ptr(),
                           idx.data_ptr() if idx is not None else None, ws.data_ptr(), ws.numel(),
                           _stream_ptr(q.device))
    if rc != 0:
        raise MobaError(rc, "moba_decode")
    return (out, lse, idx) if return_idx else (out, lse)


BWD_PARTIAL_BUDGET_BYTES = 24 << 30


def moba_backward(q, k, v, out, lse, dout, cu_seqlens, idx, block_size: int, topk: int,
                  softmax_scale: float = 0.0, chunk_tokens: Optional[int] = None,
                  workspace: Optional[Workspace] = None):
    """Gradients (dq [T, Hq, d], dk, dv [T, Hkv, d], fp32) of sum(dout * out)
    for the forward's selection idx [T, Hq, topk] (moba_forward(...,
    return_idx=True)) and its out, lse.  chunk_tokens: query tokens per pass
    of the fp32 dQ partials (None keeps them within 24 GiB, 0 = one pass)."""
    _check_qkv(q, k, v)
    _check_cu(cu_seqlens, q.device)
    for name, t in (("out", out), ("dout", dout)):
        if t.dtype != torch.bfloat16 or t.shape != q.shape or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 tensor shaped like q")
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if lse.dtype != torch.float32 or tuple(lse.shape) != (T, Hq) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 tensor [T, Hq]")
    if idx.dtype != torch.int32 or tuple(idx.shape) != (T, Hq, topk) or not idx.is_contiguous():
        raise ValueError("idx must be the forward's contiguous int32 selection [T, Hq, topk]")
    dq = torch.empty((T, Hq, d), dtype=torch.float32, device=q.device)
    dk = torch.empty((T, Hkv, d), dtype=torch.float32, device=q.device)
    dv = torch.empty((T, Hkv, d), dtype=torch.float32, device=q.device)
    n_seqs = cu_seqlens.numel() - 1
    if chunk_tokens is None:
        per_token = Hq * topk * d * 4
        n_pass = max(1, -(-T * per_token // BWD_PARTIAL_BUDGET_BYTES))
        chunk_tokens = 0 if n_pass == 1 else -(-T // n_pass)
    nbytes = lib().moba_backward_workspace_size(T, n_seqs, Hq, Hkv, d, block_size, topk,
                                                chunk_tokens)
    if nbytes == 0:
        raise MobaError(2, "moba_backward_workspace_size")
    ws = (workspace or _default_ws).get(int(nbytes), q.device)
    rc = lib().moba_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             lse.data_ptr(), dout.data_ptr(), idx.data_ptr(),
                             cu_seqlens.data_ptr(), n_seqs, T, Hq, Hkv, d, block_size, topk,
                             float(softmax_scale), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                             chunk_tokens, ws.data_ptr(), ws.numel(), _stream_ptr(q.device))
    if rc != 0:
        raise MobaError(rc, "moba_backward")
    return dq, dk, dv


def moba_check(workspace: Optional[Workspace] = None, device=None):
    """Synchronise and raise if the last call on the workspace hit a device-side error."""
    ws = (workspace or _default_ws).buf
    if ws is None:
        return
    rc = lib().moba_check(ws.data_ptr(), _stream_ptr(ws.device))
    if rc != 0:
        raise MobaError(rc, "moba_check")
