"""Factorized sparse causal self-attention (Sparse Transformer strided / fixed patterns) for
NVIDIA B200 (sm_100a).

The compute lives in libst_attn.so (hand-written tcgen05/TMA kernels behind the C ABI of
include/st_attn.h).  This module is a thin binding with the same names: it marshals PyTorch
tensors (device memory and streams only) into the C calls.  There is no fallback path: a missing
library or a non-CUDA tensor is an error.

    lay = Layout(ST_FIXED, ST_PER_HEAD_ALTERNATING, num_heads=8, n=12288, l=128, c=32)
    lay.upload()
    o, lse = st_attn_fwd(q, k, v, lay)                  # q, k, v: [B, H, n, 64] bf16, CUDA
    dq, dk, dv = st_attn_bwd(q, k, v, o, lse, do, lay)
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _abi
from ._abi import (ST_BF16, ST_ERR_DEVICE_TIMEOUT, ST_FIXED, ST_FP32, ST_KIND_FA1, ST_KIND_FA2, ST_KIND_FU, ST_KIND_SA1,
                   ST_KIND_SA2, ST_KIND_SU, ST_MERGED, ST_PER_HEAD_ALTERNATING, ST_SINGLE_A1,
                   ST_SINGLE_A2, ST_STRIDED, StError)

__all__ = [
    "Layout", "st_attn_fwd", "st_attn_bwd", "st_attn_decode", "st_attn_fwd_workspace_bytes",
    "st_attn_bwd_workspace_bytes", "SparseAttention", "StError", "ST_ERR_DEVICE_TIMEOUT", "ST_STRIDED", "ST_FIXED",
    "ST_PER_HEAD_ALTERNATING", "ST_MERGED", "ST_SINGLE_A1", "ST_SINGLE_A2", "ST_BF16", "ST_FP32",
    "ST_KIND_SA1", "ST_KIND_SA2", "ST_KIND_SU", "ST_KIND_FA1", "ST_KIND_FA2", "ST_KIND_FU",
]

_c = ctypes


def _stream(stream):
    if stream is None:
        return _c.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return _c.c_void_p(stream.cuda_stream)
    return _c.c_void_p(int(stream))


class Layout:
    """Owner of an st_layout_t: the block layout of one pattern (st_layout_build)."""

    def __init__(self, family: int, head_mode: int, num_heads: int, n: int, l: int, c: int = 0,
                 block: int = 128, a2_offset_step: int = 0):
        self._lib = _abi.load()
        self._h = _c.c_void_p()
        pat = _abi.st_pattern_t(family, head_mode, num_heads, a2_offset_step)
        _abi.check(self._lib.st_layout_build(_c.byref(pat), n, l, c, block, _c.byref(self._h)),
                   "st_layout_build")
        self.family, self.head_mode, self.num_heads = family, head_mode, num_heads
        self.n, self.l, self.c, self.block = n, l, c, block

    @property
    def handle(self):
        return self._h

    def upload(self, stream=None) -> "Layout":
        _abi.check(self._lib.st_layout_upload(self._h, _stream(stream)), "st_layout_upload")
        return self

    def head_kind(self, head: int):
        kind, off = _c.c_int32(), _c.c_int32()
        _abi.check(self._lib.st_layout_head_kind(self._h, head, _c.byref(kind), _c.byref(off)),
                   "st_layout_head_kind")
        return kind.value, off.value

    def export(self, head: int):
        """Natural-frame CSR of a head: (row_ptr, col_idx, mask_id, masks[n_masks, words])."""
        rp, ci, mi, mk = (_c.c_void_p() for _ in range(4))
        nq, nnz, nm = _c.c_int32(), _c.c_int32(), _c.c_int32()
        _abi.check(self._lib.st_layout_export(self._h, head, _c.byref(rp), _c.byref(ci),
                                              _c.byref(mi), _c.byref(mk), _c.byref(nq),
                                              _c.byref(nnz), _c.byref(nm)), "st_layout_export")

        def arr(ptr, count, ctype, dtype):
            if count == 0:
                return np.zeros(0, dtype=dtype)
            return np.ctypeslib.as_array(_c.cast(ptr, _c.POINTER(ctype)), shape=(count,)).copy()

        words = self.block * self.block // 32
        row_ptr = arr(rp, nq.value + 1, _c.c_int32, np.int32)
        col_idx = arr(ci, nnz.value, _c.c_int32, np.int32)
        mask_id = arr(mi, nnz.value, _c.c_int32, np.int32)
        masks = arr(mk, nm.value * words, _c.c_uint32, np.uint32).reshape(nm.value, words)
        return row_ptr, col_idx, mask_id, masks

    def info(self) -> dict:
        inf = _abi.st_layout_info_t()
        _abi.check(self._lib.st_layout_info(self._h, _c.byref(inf)), "st_layout_info")
        return {f: getattr(inf, f) for f, _ in inf._fields_ if f != "reserved"}

    def exec_row(self, head: int, i: int) -> np.ndarray:
        keys = np.empty(self.n, dtype=np.int64)
        cnt = _c.c_int64()
        _abi.check(self._lib.st_layout_exec_row(self._h, head, i, keys.ctypes.data_as(_c.c_void_p),
                                                _c.byref(cnt)), "st_layout_exec_row")
        return keys[:cnt.value].copy()

    def decode_row_keys(self, head: int, pos: int) -> np.ndarray:
        """The cache rows the decode step reads for `head` at position `pos` (increasing)."""
        keys = np.empty(pos + 1, dtype=np.int64)
        cnt = _c.c_int64()
        _abi.check(self._lib.st_decode_row_keys(self._h, head, pos, keys.ctypes.data_as(_c.c_void_p),
                                                _c.byref(cnt)), "st_decode_row_keys")
        return keys[:cnt.value].copy()

    def check(self, stream=None) -> None:
        _abi.check(self._lib.st_layout_check(self._h, _stream(stream)), "st_layout_check")

    def selftest_wait_timeout(self, stream=None) -> None:
        """Launch one warp whose bounded wait runs out (after 1 s): the next check() raises
        StError with ST_ERR_DEVICE_TIMEOUT, and the context stays usable."""
        _abi.check(self._lib.st_selftest_wait_timeout(self._h, _stream(stream)), "st_selftest_wait_timeout")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._lib.st_layout_destroy(h)
            h.value = None  # (at interpreter exit the ctypes module may already be gone)


def _desc(q: torch.Tensor, v: torch.Tensor | None = None) -> _abi.st_desc_t:
    """Descriptor of a call: q is [batch, heads, n, d]; v (if given) [batch, heads, n, dv].  The
    value width is sent as 0 ("same as d") when the two widths agree."""
    if q.dim() != 4:
        raise ValueError("expected [batch, heads, n, d] tensors")
    B, H, n, d = q.shape
    if q.dtype == torch.bfloat16:
        dt = ST_BF16
    elif q.dtype == torch.float32:
        dt = ST_FP32
    else:
        raise TypeError(f"unsupported dtype {q.dtype}")
    dv = 0 if v is None or v.shape[-1] == d else int(v.shape[-1])
    return _abi.st_desc_t(B, H, n, d, dt, dv)


def _check_tensors(qk, vo=()):
    """qk: tensors of query-key width ([B, H, n, d]: q, k, dq, dk); vo: tensors of value width
    ([B, H, n, dv]: v, o, dO, dv).  All contiguous CUDA tensors of one dtype and device."""
    ref = qk[0]
    for t in (*qk, *vo):
        if not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors (no CPU path exists)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if t.dim() != 4 or t.dtype != ref.dtype or t.device != ref.device:
            raise ValueError("tensors must be [B, H, n, width] of one dtype and device")
    for t in qk:
        if t.shape != ref.shape:
            raise ValueError("q and k (and dq, dk) must share one shape [B, H, n, d]")
    for t in vo:
        if t.shape[:3] != ref.shape[:3] or t.shape[3] != vo[0].shape[3]:
            raise ValueError("v, o, dO (and dv) must share one shape [B, H, n, dv]")


def _ptr(t):
    return _c.c_void_p(t.data_ptr()) if t is not None else _c.c_void_p()


def st_attn_fwd_workspace_bytes(q: torch.Tensor, layout: Layout) -> int:
    d = _desc(q)
    return int(layout._lib.st_attn_fwd_workspace_bytes(_c.byref(d), layout.handle))


def st_attn_bwd_workspace_bytes(q: torch.Tensor, layout: Layout) -> int:
    d = _desc(q)
    return int(layout._lib.st_attn_bwd_workspace_bytes(_c.byref(d), layout.handle))


def st_attn_fwd(q, k, v, layout: Layout, o=None, lse=None, workspace=None, stream=None):
    """O and lse ([B, H, n] fp32, natural log) of factorized sparse attention."""
    _check_tensors((q, k), (v,) if o is None else (v, o))
    desc = _desc(q, v)
    B, H, n, _ = q.shape
    if o is None:
        o = torch.empty_like(v)
    if lse is None:
        lse = torch.empty((B, H, n), dtype=torch.float32, device=q.device)
    ws = int(layout._lib.st_attn_fwd_workspace_bytes(_c.byref(desc), layout.handle))
    if ws and workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=q.device)
    st = layout._lib.st_attn_fwd(_ptr(q), _ptr(k), _ptr(v), layout.handle, _ptr(o), _ptr(lse),
                                 _ptr(workspace), ws if workspace is not None else 0,
                                 _c.byref(desc), _stream(stream))
    _abi.check(st, "st_attn_fwd")
    return o, lse


def st_attn_bwd(q, k, v, o, lse, do, layout: Layout, dq=None, dk=None, dv=None, workspace=None,
                stream=None):
    """dQ, dK, dV of factorized sparse attention (recomputing P from the saved lse)."""
    _check_tensors((q, k), (v, o, do))
    desc = _desc(q, v)
    if dq is None:
        dq = torch.empty_like(q)
    if dk is None:
        dk = torch.empty_like(k)
    if dv is None:
        dv = torch.empty_like(v)
    ws = int(layout._lib.st_attn_bwd_workspace_bytes(_c.byref(desc), layout.handle))
    if workspace is None:
        workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=q.device)
    st = layout._lib.st_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do),
                                 layout.handle, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                 workspace.numel(), _c.byref(desc), _stream(stream))
    _abi.check(st, "st_attn_bwd")
    return dq, dk, dv


def st_attn_decode(q, k_cache, v_cache, layout: Layout, pos: int, o=None, lse=None, workspace=None,
                   stream=None):
    """Decode step: q [B, H, d] at position pos against k_cache [B, H, n, d] and v_cache
    [B, H, n, dv] (rows past pos unread; the kernels take d = dv = 64).  Returns o [B, H, dv] and
    lse [B, H] (fp32) -- row pos of the forward pass."""
    _check_tensors((k_cache,), (v_cache,))
    if not (q.is_cuda and q.is_contiguous() and q.dtype == k_cache.dtype and q.device == k_cache.device
            and q.dim() == 3 and tuple(q.shape) == (k_cache.shape[0], k_cache.shape[1], k_cache.shape[3])):
        raise ValueError("q must be a contiguous [B, H, d] CUDA tensor matching the key cache")
    desc = _desc(k_cache, v_cache)
    if o is None:
        o = q.new_empty((q.shape[0], q.shape[1], v_cache.shape[3]))
    if lse is None:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
    ws = int(layout._lib.st_attn_decode_workspace_bytes(_c.byref(desc), layout.handle))
    if workspace is None:
        workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=q.device)
    st = layout._lib.st_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), layout.handle, int(pos), _ptr(o),
                                    _ptr(lse), _ptr(workspace), workspace.numel(), _c.byref(desc),
                                    _stream(stream))
    _abi.check(st, "st_attn_decode")
    return o, lse


class SparseAttention(torch.autograd.Function):
    """Autograd wrapper: forward saves (q, k, v, o, lse); backward recomputes P."""

    @staticmethod
    def forward(ctx, q, k, v, layout):
        o, lse = st_attn_fwd(q, k, v, layout)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.layout = layout
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = st_attn_bwd(q, k, v, o, lse, do.contiguous(), ctx.layout)
        return dq, dk, dv, None
