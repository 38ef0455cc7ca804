"""Python binding of the C ABI (include/ea.h), one function per entry point.

Argument marshalling only: PyTorch provides device memory and the current
CUDA stream; every step of the computation runs in libea.so's kernels.
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional, Tuple

import numpy as np
import torch

from . import _lib
from ._lib import (EA_SELECT_ALL, EA_SELECT_FA, EA_SELECT_SA, EaAttnParams,  # noqa: F401
                   EaDecodeParams, EaVarlenParams, check)


def _stream_ptr(stream: Optional[torch.cuda.Stream], device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return int(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, ndim: Optional[int] = None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def make_params(B, Hq, Hkv, N, d, sink, window, softmax_scale=0.0,
                select=EA_SELECT_ALL) -> EaAttnParams:
    return EaAttnParams(int(B), int(Hq), int(Hkv), int(N), int(d), int(sink), int(window),
                        float(softmax_scale), int(select))


# ---------------------------------------------------------------- router
def ea_router_workspace_size(B: int, Hkv: int, N: int, d: int) -> int:
    return int(_lib.load().ea_router_workspace_size(B, Hkv, N, d))


def ea_router_decide(k: torch.Tensor, w1: torch.Tensor, b1: torch.Tensor, w2: torch.Tensor,
                     b2: torch.Tensor, threshold: float = 0.0, *,
                     workspace: Optional[torch.Tensor] = None,
                     route_mask: Optional[torch.Tensor] = None,
                     logits: Optional[torch.Tensor] = None, want_logits: bool = True,
                     stream: Optional[torch.cuda.Stream] = None
                     ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Route mask uint8 [B, Hq] (1 = sparse) and logits fp32 [B, Hq]."""
    lib = _lib.load()
    _need(k, "k", torch.bfloat16, 4)
    for name, t, nd in (("w1", w1, 2), ("b1", b1, 1), ("w2", w2, 2), ("b2", b2, 1)):
        _need(t, name, torch.float32, nd)
    B, Hkv, N, d = k.shape
    hidden = w1.shape[0]
    Hq = w2.shape[0]
    if w1.shape[1] != Hkv * d or b1.shape[0] != hidden or w2.shape[1] != hidden \
            or b2.shape[0] != Hq:
        raise ValueError("router weight shapes do not match the key states")
    dev = k.device
    need = lib.ea_router_workspace_size(B, Hkv, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    if route_mask is None:
        route_mask = torch.empty((B, Hq), dtype=torch.uint8, device=dev)
    if logits is None and want_logits:
        logits = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    rc = lib.ea_router_decide(k.data_ptr(), B, Hkv, N, d, w1.data_ptr(), b1.data_ptr(), hidden,
                              w2.data_ptr(), b2.data_ptr(), Hq, float(threshold),
                              route_mask.data_ptr(),
                              logits.data_ptr() if logits is not None else None,
                              workspace.data_ptr(), workspace.numel(), _stream_ptr(stream, dev))
    check(rc, "ea_router_decide")
    return route_mask, logits


def ea_router_decide_varlen(k: torch.Tensor, cu_seqlens: torch.Tensor, max_seqlen: int,
                            w1: torch.Tensor, b1: torch.Tensor, w2: torch.Tensor,
                            b2: torch.Tensor, threshold: float = 0.0, *,
                            workspace: Optional[torch.Tensor] = None,
                            route_mask: Optional[torch.Tensor] = None,
                            logits: Optional[torch.Tensor] = None, want_logits: bool = True,
                            stream: Optional[torch.cuda.Stream] = None
                            ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Router of a packed batch: k [T, Hkv, d], cu_seqlens int32 [B + 1] on the
    device; route mask uint8 [B, Hq] and logits fp32 [B, Hq]."""
    lib = _lib.load()
    _need(k, "k", torch.bfloat16, 3)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    for name, t, nd in (("w1", w1, 2), ("b1", b1, 1), ("w2", w2, 2), ("b2", b2, 1)):
        _need(t, name, torch.float32, nd)
    T, Hkv, d = k.shape
    B = cu_seqlens.numel() - 1
    hidden = w1.shape[0]
    Hq = w2.shape[0]
    if w1.shape[1] != Hkv * d or b1.shape[0] != hidden or w2.shape[1] != hidden \
            or b2.shape[0] != Hq:
        raise ValueError("router weight shapes do not match the key states")
    dev = k.device
    need = lib.ea_router_varlen_workspace_size(B, Hkv, int(max_seqlen), d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    if route_mask is None:
        route_mask = torch.empty((B, Hq), dtype=torch.uint8, device=dev)
    if logits is None and want_logits:
        logits = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    rc = lib.ea_router_decide_varlen(k.data_ptr(), cu_seqlens.data_ptr(), B, Hkv, T,
                                     int(max_seqlen), d, w1.data_ptr(), b1.data_ptr(), hidden,
                                     w2.data_ptr(), b2.data_ptr(), Hq, float(threshold),
                                     route_mask.data_ptr(),
                                     logits.data_ptr() if logits is not None else None,
                                     workspace.data_ptr(), workspace.numel(),
                                     _stream_ptr(stream, dev))
    check(rc, "ea_router_decide_varlen")
    return route_mask, logits


def ea_router_pool_rows(k: torch.Tensor, row0: int, nrows: int, *, x_out: torch.Tensor,
                        workspace: torch.Tensor,
                        stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Pooled key rows [row0, row0 + nrows) of the flattened (b, kv head)
    index of k [B, Hkv, N, d] into x_out (fp32, at least nrows * d values)."""
    lib = _lib.load()
    _need(k, "k", torch.bfloat16, 4)
    _need(x_out, "x_out", torch.float32)
    _need(workspace, "workspace", torch.uint8)
    B, Hkv, N, d = k.shape
    if x_out.numel() < nrows * d:
        raise ValueError("x_out must hold nrows * d values")
    rc = lib.ea_router_pool_rows(k.data_ptr(), B, Hkv, N, d, int(row0), int(nrows),
                                 x_out.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                 _stream_ptr(stream, k.device))
    check(rc, "ea_router_pool_rows")
    return x_out


def ea_router_mlp_workspace_size(B: int, hidden: int) -> int:
    return int(_lib.load().ea_router_mlp_workspace_size(B, hidden))


def ea_router_mlp(x: torch.Tensor, w1: torch.Tensor, b1: torch.Tensor, w2: torch.Tensor,
                  b2: torch.Tensor, threshold: float = 0.0, *, route_mask: torch.Tensor,
                  logits: Optional[torch.Tensor] = None, workspace: torch.Tensor,
                  stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """The router's MLP and threshold on pooled x [B, in_dim] (fp32)."""
    lib = _lib.load()
    _need(x, "x", torch.float32, 2)
    for name, t, nd in (("w1", w1, 2), ("b1", b1, 1), ("w2", w2, 2), ("b2", b2, 1)):
        _need(t, name, torch.float32, nd)
    _need(route_mask, "route_mask", torch.uint8)
    _need(workspace, "workspace", torch.uint8)
    B, in_dim = x.shape
    hidden, Hq = w1.shape[0], w2.shape[0]
    if w1.shape[1] != in_dim or b1.shape[0] != hidden or w2.shape[1] != hidden \
            or b2.shape[0] != Hq:
        raise ValueError("router weight shapes do not match x")
    if route_mask.numel() != B * Hq or (logits is not None and logits.numel() != B * Hq):
        raise ValueError("route_mask and logits must hold B * Hq entries")
    rc = lib.ea_router_mlp(x.data_ptr(), B, in_dim, w1.data_ptr(), b1.data_ptr(), hidden,
                           w2.data_ptr(), b2.data_ptr(), Hq, float(threshold),
                           route_mask.data_ptr(),
                           logits.data_ptr() if logits is not None else None,
                           workspace.data_ptr(), workspace.numel(), _stream_ptr(stream, x.device))
    check(rc, "ea_router_mlp")
    return route_mask


def _padded_router_shapes(k_shape, w1, b1, w2, b2):
    """(B, Hkv, N, d, hidden, Hq) of a padded router call; raises ValueError if
    the weights do not fit the key states."""
    if len(k_shape) != 4 or any(t.dim() != n for t, n in ((w1, 2), (b1, 1), (w2, 2), (b2, 1))):
        raise ValueError("k must be [B, Hkv, N, d]; w1, w2 2-D and b1, b2 1-D")
    B, Hkv, N, d = (int(x) for x in k_shape)
    hidden, Hq = int(w1.shape[0]), int(w2.shape[0])
    if w1.shape[1] != Hkv * d or b1.shape[0] != hidden or w2.shape[1] != hidden \
            or b2.shape[0] != Hq:
        raise ValueError("router weight shapes do not match the key states")
    return B, Hkv, N, d, hidden, Hq


def ea_router_decide_noalloc(k: torch.Tensor, w1: torch.Tensor, b1: torch.Tensor,
                             w2: torch.Tensor, b2: torch.Tensor, threshold: float = 0.0, *,
                             route_mask: torch.Tensor, logits: Optional[torch.Tensor] = None,
                             stream: Optional[torch.cuda.Stream] = None) -> None:
    """The router without a workspace argument, for callers that cannot
    allocate device memory when they route a layer (its scratch is a fixed
    array inside libea.so).  The caller passes the output buffers, route_mask
    uint8 [B, Hq] and optionally logits fp32 [B, Hq], on k's device; this
    wrapper allocates nothing either.  The call runs with k's device current,
    because the library uses the current device's copy of its scratch."""
    lib = _lib.load()
    B, Hkv, N, d, hidden, Hq = _padded_router_shapes(k.shape, w1, b1, w2, b2)
    if tuple(route_mask.shape) != (B, Hq):
        raise ValueError(f"route_mask must be [B, Hq] = [{B}, {Hq}]")
    if logits is not None and tuple(logits.shape) != (B, Hq):
        raise ValueError(f"logits must be [B, Hq] = [{B}, {Hq}]")
    _need(k, "k", torch.bfloat16, 4)
    for name, t, nd in (("w1", w1, 2), ("b1", b1, 1), ("w2", w2, 2), ("b2", b2, 1)):
        _need(t, name, torch.float32, nd)
    _need(route_mask, "route_mask", torch.uint8, 2)
    if logits is not None:
        _need(logits, "logits", torch.float32, 2)
    dev = k.device
    for name, t in (("w1", w1), ("b1", b1), ("w2", w2), ("b2", b2), ("route_mask", route_mask),
                    ("logits", logits)):
        if t is not None and t.device != dev:
            raise ValueError(f"{name} must be on {dev}, like k")
    with torch.cuda.device(dev):
        rc = lib.ea_router_decide_noalloc(k.data_ptr(), B, Hkv, N, d, w1.data_ptr(),
                                          b1.data_ptr(), hidden, w2.data_ptr(), b2.data_ptr(),
                                          Hq, float(threshold), route_mask.data_ptr(),
                                          logits.data_ptr() if logits is not None else None,
                                          _stream_ptr(stream, dev))
    check(rc, "ea_router_decide_noalloc")


# ---------------------------------------------------------------- attention
def ea_hybrid_attn_workspace_size(p: EaAttnParams) -> int:
    return int(_lib.load().ea_hybrid_attn_workspace_size(ctypes.byref(p)))


def attn_workspace(p: EaAttnParams, device) -> torch.Tensor:
    """A zeroed attention workspace (the status word starts at 0)."""
    n = ea_hybrid_attn_workspace_size(p)
    if n == 0:
        raise ValueError("invalid attention parameters")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def ea_hybrid_attn_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                           route_mask: torch.Tensor, sink: int, window: int, *,
                           softmax_scale: float = 0.0, select: int = EA_SELECT_ALL,
                           out: Optional[torch.Tensor] = None,
                           workspace: Optional[torch.Tensor] = None,
                           stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Fused hybrid prefill attention; returns out bf16 [B, Hq, N, d]."""
    lib = _lib.load()
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    _need(route_mask, "route_mask", torch.uint8)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, N, d] matching q")
    if route_mask.numel() != B * Hq:
        raise ValueError("route_mask must hold B * Hq entries")
    p = make_params(B, Hq, Hkv, N, d, sink, window, softmax_scale, select)
    if out is None:
        out = torch.empty_like(q)
    else:
        _need(out, "out", torch.bfloat16, 4)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    if workspace is None:
        workspace = attn_workspace(p, q.device)
    rc = lib.ea_hybrid_attn_prefill(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                    route_mask.data_ptr(), ctypes.byref(p), out.data_ptr(),
                                    workspace.data_ptr(), workspace.numel(),
                                    _stream_ptr(stream, q.device))
    check(rc, "ea_hybrid_attn_prefill")
    return out


def _prefill_selected(name: str, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                      route_mask: torch.Tensor, sel: torch.Tensor, sink: int, window: int, *,
                      softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None,
                      stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """The fused prefill on one shard, through the C entry point `name`:
    ea_hybrid_attn_prefill_groups (sel [B, Hkv] by kv group) or
    ea_hybrid_attn_prefill_heads (sel [B, Hq] by query head).  Only the
    selected heads run; other heads' rows of `out` are left as they were."""
    lib = _lib.load()
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    _need(route_mask, "route_mask", torch.uint8)
    _need(sel, "selection", torch.uint8)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, N, d] matching q")
    want = B * Hkv if name == "ea_hybrid_attn_prefill_groups" else B * Hq
    if route_mask.numel() != B * Hq or sel.numel() != want:
        raise ValueError("route_mask must hold B * Hq entries and the selection %d" % want)
    p = make_params(B, Hq, Hkv, N, d, sink, window, softmax_scale)
    if out is None:
        out = torch.empty_like(q)
    else:
        _need(out, "out", torch.bfloat16, 4)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    if workspace is None:
        workspace = attn_workspace(p, q.device)
    rc = getattr(lib, name)(q.data_ptr(), k.data_ptr(), v.data_ptr(), route_mask.data_ptr(),
                            sel.data_ptr(), ctypes.byref(p), out.data_ptr(),
                            workspace.data_ptr(), workspace.numel(),
                            _stream_ptr(stream, q.device))
    check(rc, name)
    return out


def ea_hybrid_attn_prefill_groups(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                  route_mask: torch.Tensor, group_sel: torch.Tensor,
                                  sink: int, window: int, **kw) -> torch.Tensor:
    """The fused prefill on one shard: only the query heads of the (b, kv
    head) groups with group_sel[b, hk] != 0 run; other heads' rows of `out`
    are left as they were."""
    return _prefill_selected("ea_hybrid_attn_prefill_groups", q, k, v, route_mask, group_sel,
                             sink, window, **kw)


def ea_hybrid_attn_prefill_heads(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                 route_mask: torch.Tensor, head_sel: torch.Tensor,
                                 sink: int, window: int, **kw) -> torch.Tensor:
    """The fused prefill on one shard: only the query heads with
    head_sel[b, h] != 0 run; other heads' rows of `out` are left as they
    were."""
    return _prefill_selected("ea_hybrid_attn_prefill_heads", q, k, v, route_mask, head_sel,
                             sink, window, **kw)


def ea_hybrid_attn_prefill_traced(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                  route_mask: torch.Tensor, sink: int, window: int, *,
                                  max_records: int = 65536, out: Optional[torch.Tensor] = None,
                                  workspace: Optional[torch.Tensor] = None,
                                  stream: Optional[torch.cuda.Stream] = None):
    """ea_hybrid_attn_prefill with a per-unit trace: (out, records int64
    [n, 11] = start_ns, first_s_ns, last_p_ns, end_ns, cta, rank, sparse,
    kv_tiles, level, head of slot 0, head of slot 1 (heads as b * Hq + h),
    total units).  Synchronises the device to read the trace back."""
    lib = _lib.load()
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    _need(route_mask, "route_mask", torch.uint8)
    B, Hq, N, d = q.shape
    p = make_params(B, Hq, k.shape[1], N, d, sink, window)
    out = torch.empty_like(q) if out is None else out
    workspace = attn_workspace(p, q.device) if workspace is None else workspace
    trace = torch.zeros(8 + 6 * int(max_records), dtype=torch.int64, device=q.device)
    rc = lib.ea_hybrid_attn_prefill_traced(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                           route_mask.data_ptr(), ctypes.byref(p),
                                           out.data_ptr(), workspace.data_ptr(),
                                           workspace.numel(), trace.data_ptr(),
                                           int(max_records), _stream_ptr(stream, q.device))
    check(rc, "ea_hybrid_attn_prefill_traced")
    t = trace.cpu().numpy()
    total = int(t[0])
    n = min(total, int(max_records))
    rec = t[8:8 + 6 * n].reshape(n, 6)
    cols = np.stack([rec[:, 0], rec[:, 1], rec[:, 2], rec[:, 3], rec[:, 4] >> 48,
                     rec[:, 4] & 0xffffffff, (rec[:, 5] >> 62) & 1, rec[:, 5] & 0xffffffff,
                     (rec[:, 4] >> 32) & 0xffff, (rec[:, 5] >> 44) & 0xfff,
                     (rec[:, 5] >> 32) & 0xfff], axis=1)
    return out, cols, total


# ---------------------------------------------------------------- packed batches
def make_varlen_params(B, Hq, Hkv, total, max_seqlen, d, sink, window, softmax_scale=0.0,
                       select=EA_SELECT_ALL) -> EaVarlenParams:
    return EaVarlenParams(int(B), int(Hq), int(Hkv), int(total), int(max_seqlen), int(d),
                          int(sink), int(window), float(softmax_scale), int(select))


def ea_hybrid_attn_prefill_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                  cu_seqlens: torch.Tensor, route_mask: torch.Tensor,
                                  max_seqlen: int, sink: int, window: int, *,
                                  softmax_scale: float = 0.0, select: int = EA_SELECT_ALL,
                                  out: Optional[torch.Tensor] = None,
                                  workspace: Optional[torch.Tensor] = None,
                                  stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Packed batch: q [T, Hq, d], k, v [T, Hkv, d], cu_seqlens int32 [B + 1]
    (device); returns out bf16 [T, Hq, d]."""
    lib = _lib.load()
    _need(q, "q", torch.bfloat16, 3)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    _need(route_mask, "route_mask", torch.uint8)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    if k.shape != (T, Hkv, d) or v.shape != k.shape:
        raise ValueError("k and v must be [T, Hkv, d] matching q")
    if route_mask.numel() != B * Hq:
        raise ValueError("route_mask must hold B * Hq entries")
    p = make_varlen_params(B, Hq, Hkv, T, max_seqlen, d, sink, window, softmax_scale, select)
    if out is None:
        out = torch.empty_like(q)
    else:
        _need(out, "out", torch.bfloat16, 3)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    if workspace is None:
        n = int(lib.ea_hybrid_attn_varlen_workspace_size(ctypes.byref(p)))
        if n == 0:
            raise ValueError("invalid packed-batch parameters")
        workspace = torch.zeros(n, dtype=torch.uint8, device=q.device)
    rc = lib.ea_hybrid_attn_prefill_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                           cu_seqlens.data_ptr(), route_mask.data_ptr(),
                                           ctypes.byref(p), out.data_ptr(), workspace.data_ptr(),
                                           workspace.numel(), _stream_ptr(stream, q.device))
    check(rc, "ea_hybrid_attn_prefill_varlen")
    return out


# ---------------------------------------------------------------- router + attention, one launch
def _router_shapes(w1, b1, w2, b2, in_dim):
    for name, t, nd in (("w1", w1, 2), ("b1", b1, 1), ("w2", w2, 2), ("b2", b2, 1)):
        _need(t, name, torch.float32, nd)
    hidden, Hq = w1.shape[0], w2.shape[0]
    if w1.shape[1] != in_dim or b1.shape[0] != hidden or w2.shape[1] != hidden \
            or b2.shape[0] != Hq:
        raise ValueError("router weight shapes do not match the key states")
    return hidden, Hq


def ea_hybrid_attn_prefill_routed(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                  w1: torch.Tensor, b1: torch.Tensor, w2: torch.Tensor,
                                  b2: torch.Tensor, sink: int, window: int,
                                  threshold: float = 0.0, *, softmax_scale: float = 0.0,
                                  select: int = EA_SELECT_ALL,
                                  route_mask: Optional[torch.Tensor] = None,
                                  logits: Optional[torch.Tensor] = None,
                                  out: Optional[torch.Tensor] = None,
                                  workspace: Optional[torch.Tensor] = None,
                                  stream: Optional[torch.cuda.Stream] = None):
    """Router and attention in one launch (padded q [B, Hq, N, d]); returns
    (out, route_mask, logits)."""
    lib = _lib.load()
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    hidden, Hq_r = _router_shapes(w1, b1, w2, b2, Hkv * d)
    if Hq_r != Hq or k.shape != (B, Hkv, N, d) or v.shape != k.shape:
        raise ValueError("shapes do not match")
    p = make_params(B, Hq, Hkv, N, d, sink, window, softmax_scale, select)
    dev = q.device
    if route_mask is None:
        route_mask = torch.empty((B, Hq), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        n = int(lib.ea_hybrid_attn_routed_workspace_size(ctypes.byref(p), hidden))
        if n == 0:
            raise ValueError("invalid parameters")
        workspace = torch.zeros(n, dtype=torch.uint8, device=dev)
    rc = lib.ea_hybrid_attn_prefill_routed(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                           w1.data_ptr(), b1.data_ptr(), hidden, w2.data_ptr(),
                                           b2.data_ptr(), float(threshold), route_mask.data_ptr(),
                                           logits.data_ptr() if logits is not None else None,
                                           ctypes.byref(p), out.data_ptr(), workspace.data_ptr(),
                                           workspace.numel(), _stream_ptr(stream, dev))
    check(rc, "ea_hybrid_attn_prefill_routed")
    return out, route_mask, logits


def ea_hybrid_attn_prefill_varlen_routed(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                         cu_seqlens: torch.Tensor, max_seqlen: int,
                                         w1: torch.Tensor, b1: torch.Tensor, w2: torch.Tensor,
                                         b2: torch.Tensor, sink: int, window: int,
                                         threshold: float = 0.0, *, softmax_scale: float = 0.0,
                                         select: int = EA_SELECT_ALL,
                                         route_mask: Optional[torch.Tensor] = None,
                                         logits: Optional[torch.Tensor] = None,
                                         out: Optional[torch.Tensor] = None,
                                         workspace: Optional[torch.Tensor] = None,
                                         stream: Optional[torch.cuda.Stream] = None):
    """Router and attention of a packed batch in one launch; returns
    (out [T, Hq, d], route_mask [B, Hq], logits)."""
    lib = _lib.load()
    _need(q, "q", torch.bfloat16, 3)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    hidden, Hq_r = _router_shapes(w1, b1, w2, b2, Hkv * d)
    if Hq_r != Hq or k.shape != (T, Hkv, d) or v.shape != k.shape:
        raise ValueError("shapes do not match")
    p = make_varlen_params(B, Hq, Hkv, T, max_seqlen, d, sink, window, softmax_scale, select)
    dev = q.device
    if route_mask is None:
        route_mask = torch.empty((B, Hq), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        n = int(lib.ea_hybrid_attn_varlen_routed_workspace_size(ctypes.byref(p), hidden))
        if n == 0:
            raise ValueError("invalid parameters")
        workspace = torch.zeros(n, dtype=torch.uint8, device=dev)
    rc = lib.ea_hybrid_attn_prefill_varlen_routed(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens.data_ptr(), w1.data_ptr(),
        b1.data_ptr(), hidden, w2.data_ptr(), b2.data_ptr(), float(threshold),
        route_mask.data_ptr(), logits.data_ptr() if logits is not None else None,
        ctypes.byref(p), out.data_ptr(), workspace.data_ptr(), workspace.numel(),
        _stream_ptr(stream, dev))
    check(rc, "ea_hybrid_attn_prefill_varlen_routed")
    return out, route_mask, logits


# ---------------------------------------------------------------- training
def ea_hybrid_attn_prefill_lse(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                               route_mask: torch.Tensor, sink: int, window: int, *,
                               softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                               lse: Optional[torch.Tensor] = None,
                               workspace: Optional[torch.Tensor] = None,
                               stream: Optional[torch.cuda.Stream] = None):
    """Forward for training: (out bf16 [B, Hq, N, d], lse fp32 [B, Hq, N])."""
    lib = _lib.load()
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    _need(route_mask, "route_mask", torch.uint8)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    p = make_params(B, Hq, Hkv, N, d, sink, window, softmax_scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _need(lse, "lse", torch.float32, 3)
    if workspace is None:
        workspace = attn_workspace(p, q.device)
    rc = lib.ea_hybrid_attn_prefill_lse(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                        route_mask.data_ptr(), ctypes.byref(p), out.data_ptr(),
                                        lse.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                        _stream_ptr(stream, q.device))
    check(rc, "ea_hybrid_attn_prefill_lse")
    return out, lse


def ea_hybrid_attn_prefill_train(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                 route_mask: torch.Tensor, sink: int, window: int, *,
                                 softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                                 lse: Optional[torch.Tensor] = None,
                                 out_other: Optional[torch.Tensor] = None,
                                 workspace: Optional[torch.Tensor] = None,
                                 stream: Optional[torch.cuda.Stream] = None):
    """Training forward, both modes in one launch: (out [chosen mode], lse
    fp32 [B, Hq, N], out_other [the other mode])."""
    lib = _lib.load()
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, 4)
    _need(route_mask, "route_mask", torch.uint8)
    B, Hq, N, d = q.shape
    p = make_params(B, Hq, k.shape[1], N, d, sink, window, softmax_scale)
    out = torch.empty_like(q) if out is None else out
    out_other = torch.empty_like(q) if out_other is None else out_other
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = attn_workspace(p, q.device)
    rc = lib.ea_hybrid_attn_prefill_train(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                          route_mask.data_ptr(), ctypes.byref(p), out.data_ptr(),
                                          lse.data_ptr(), out_other.data_ptr(),
                                          workspace.data_ptr(), workspace.numel(),
                                          _stream_ptr(stream, q.device))
    check(rc, "ea_hybrid_attn_prefill_train")
    return out, lse, out_other


# ---------------------------------------------------------------- FP8
def ea_fp8_vt_stride(N: int) -> int:
    """Row stride (bytes) of the transposed e4m3 V layout: N rounded up to 16."""
    return int(_lib.load().ea_fp8_vt_stride(int(N)))


def ea_quantize_fp8(x: torch.Tensor, transpose: bool = False, *,
                    codes: Optional[torch.Tensor] = None, scale: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None):
    """Per-head e4m3 quantization of bf16 x [B, H, N, d]: (codes uint8
    [B, H, N, d], or [B, H, d, ea_fp8_vt_stride(N)] when transposed; scale
    fp32 [B, H])."""
    lib = _lib.load()
    _need(x, "x", torch.bfloat16, 4)
    B, H, N, d = x.shape
    dev = x.device
    shape = (B, H, d, ea_fp8_vt_stride(N)) if transpose else (B, H, N, d)
    if codes is None:
        codes = torch.empty(shape, dtype=torch.uint8, device=dev)
    if scale is None:
        scale = torch.empty((B, H), dtype=torch.float32, device=dev)
    _need(codes, "codes", torch.uint8, 4)
    _need(scale, "scale", torch.float32)
    if tuple(codes.shape) != shape or scale.numel() != B * H:
        raise ValueError("codes / scale buffers do not match x")
    if workspace is None:
        workspace = torch.empty(int(lib.ea_quantize_fp8_workspace_size(B * H)), dtype=torch.uint8,
                                device=dev)
    rc = lib.ea_quantize_fp8(x.data_ptr(), B * H, N, d, 1 if transpose else 0, codes.data_ptr(),
                             scale.data_ptr(), workspace.data_ptr(), workspace.numel(),
                             _stream_ptr(stream, dev))
    check(rc, "ea_quantize_fp8")
    return codes, scale


def ea_hybrid_attn_prefill_fp8(q8: torch.Tensor, k8: torch.Tensor, vt8: torch.Tensor,
                               q_scale: torch.Tensor, k_scale: torch.Tensor,
                               v_scale: torch.Tensor, route_mask: torch.Tensor, sink: int,
                               window: int, *, softmax_scale: float = 0.0,
                               select: int = EA_SELECT_ALL, out: Optional[torch.Tensor] = None,
                               workspace: Optional[torch.Tensor] = None,
                               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """The fused attention over e4m3 inputs (as ea_quantize_fp8 writes them):
    out bf16 [B, Hq, N, d]."""
    lib = _lib.load()
    for name, t in (("q8", q8), ("k8", k8), ("vt8", vt8)):
        _need(t, name, torch.uint8, 4)
    for name, t in (("q_scale", q_scale), ("k_scale", k_scale), ("v_scale", v_scale)):
        _need(t, name, torch.float32)
    _need(route_mask, "route_mask", torch.uint8)
    B, Hq, N, d = q8.shape
    Hkv = k8.shape[1]
    if tuple(k8.shape) != (B, Hkv, N, d) or tuple(vt8.shape) != (B, Hkv, d, ea_fp8_vt_stride(N)):
        raise ValueError("k8 / vt8 shapes do not match q8")
    if q_scale.numel() != B * Hq or k_scale.numel() != B * Hkv or v_scale.numel() != B * Hkv:
        raise ValueError("one scale per (batch, head) is required")
    p = make_params(B, Hq, Hkv, N, d, sink, window, softmax_scale, select)
    if out is None:
        out = torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=q8.device)
    if workspace is None:
        workspace = attn_workspace(p, q8.device)
    rc = lib.ea_hybrid_attn_prefill_fp8(q8.data_ptr(), k8.data_ptr(), vt8.data_ptr(),
                                        q_scale.data_ptr(), k_scale.data_ptr(),
                                        v_scale.data_ptr(), route_mask.data_ptr(),
                                        ctypes.byref(p), out.data_ptr(), workspace.data_ptr(),
                                        workspace.numel(), _stream_ptr(stream, q8.device))
    check(rc, "ea_hybrid_attn_prefill_fp8")
    return out


def ea_hybrid_attn_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                            out: torch.Tensor, dout: torch.Tensor, lse: torch.Tensor,
                            route_mask: torch.Tensor, sink: int, window: int, *,
                            softmax_scale: float = 0.0, dq: Optional[torch.Tensor] = None,
                            dk: Optional[torch.Tensor] = None, dv: Optional[torch.Tensor] = None,
                            workspace: Optional[torch.Tensor] = None,
                            stream: Optional[torch.cuda.Stream] = None):
    """(dq, dk, dv) bf16 of L = sum(dout * out) for the hybrid attention."""
    lib = _lib.load()
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        _need(t, name, torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    _need(route_mask, "route_mask", torch.uint8)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    p = make_params(B, Hq, Hkv, N, d, sink, window, softmax_scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        n = int(lib.ea_hybrid_attn_backward_workspace_size(ctypes.byref(p)))
        if n == 0:
            raise ValueError("unsupported backward parameters (d must be 128)")
        workspace = torch.zeros(n, dtype=torch.uint8, device=q.device)
    rc = lib.ea_hybrid_attn_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                     dout.data_ptr(), lse.data_ptr(), route_mask.data_ptr(),
                                     ctypes.byref(p), dq.data_ptr(), dk.data_ptr(),
                                     dv.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                     _stream_ptr(stream, q.device))
    check(rc, "ea_hybrid_attn_backward")
    return dq, dk, dv


def _router_train_dims(k, w1, b1, w2, b2, g0, g1, tau):
    _need(k, "k", torch.bfloat16, 4)
    for name, t, nd in (("w1", w1, 2), ("b1", b1, 1), ("w2", w2, 2), ("b2", b2, 1),
                        ("g0", g0, 2), ("g1", g1, 2)):
        _need(t, name, torch.float32, nd)
    B, Hkv, N, d = k.shape
    hidden, Hq = _router_shapes(w1, b1, w2, b2, Hkv * d)
    if tuple(g0.shape) != (B, Hq) or tuple(g1.shape) != (B, Hq):
        raise ValueError("Gumbel noise must be [B, Hq]")
    if not tau > 0.0:
        raise ValueError("tau must be positive")
    return B, Hkv, N, d, hidden, Hq


def ea_router_decide_gumbel(k: torch.Tensor, w1: torch.Tensor, b1: torch.Tensor,
                            w2: torch.Tensor, b2: torch.Tensor, g0: torch.Tensor,
                            g1: torch.Tensor, tau: float, *,
                            route_mask: Optional[torch.Tensor] = None,
                            r_soft: Optional[torch.Tensor] = None,
                            logits: Optional[torch.Tensor] = None,
                            workspace: Optional[torch.Tensor] = None,
                            stream: Optional[torch.cuda.Stream] = None):
    """Training-time routing: (r_hard uint8 [B, Hq], r_soft fp32, logits fp32),
    into the given buffers when passed."""
    lib = _lib.load()
    B, Hkv, N, d, hidden, Hq = _router_train_dims(k, w1, b1, w2, b2, g0, g1, tau)
    dev = k.device
    if workspace is None:
        workspace = torch.empty(max(int(lib.ea_router_gumbel_workspace_size(
            B, Hkv, N, d, hidden, Hq)), 16), dtype=torch.uint8, device=dev)
    r_hard = torch.empty((B, Hq), dtype=torch.uint8, device=dev) if route_mask is None \
        else route_mask
    if r_soft is None:
        r_soft = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    if logits is None:
        logits = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    for name, t, dt in (("route_mask", r_hard, torch.uint8), ("r_soft", r_soft, torch.float32),
                        ("logits", logits, torch.float32)):
        _need(t, name, dt)
        if t.numel() != B * Hq:
            raise ValueError(f"{name} must hold B * Hq values")
    rc = lib.ea_router_decide_gumbel(k.data_ptr(), B, Hkv, N, d, w1.data_ptr(), b1.data_ptr(),
                                     hidden, w2.data_ptr(), b2.data_ptr(), Hq, g0.data_ptr(),
                                     g1.data_ptr(), float(tau), r_hard.data_ptr(),
                                     r_soft.data_ptr(), logits.data_ptr(), workspace.data_ptr(),
                                     workspace.numel(), _stream_ptr(stream, dev))
    check(rc, "ea_router_decide_gumbel")
    return r_hard, r_soft, logits


def ea_router_ste_backward(k: torch.Tensor, w1: torch.Tensor, b1: torch.Tensor,
                           w2: torch.Tensor, b2: torch.Tensor, g0: torch.Tensor,
                           g1: torch.Tensor, tau: float, dout: torch.Tensor,
                           out: torch.Tensor, out_other: torch.Tensor,
                           route_mask: Optional[torch.Tensor] = None, *,
                           dk_accum: Optional[torch.Tensor] = None,
                           workspace: Optional[torch.Tensor] = None,
                           stream: Optional[torch.cuda.Stream] = None):
    """Router gradients through the straight-through estimator:
    (dr [B, Hq], dw1, db1, dw2, db2, dk_pool [B, Hkv*d]) fp32; when dk_accum
    (bf16 [B, Hkv, N, d]) is given, dk_pool is added to it in place.  out /
    out_other: each head's chosen / other mode (route_mask None: O_FA / O_SA)."""
    lib = _lib.load()
    B, Hkv, N, d, hidden, Hq = _router_train_dims(k, w1, b1, w2, b2, g0, g1, tau)
    for name, t in (("dout", dout), ("out", out), ("out_other", out_other)):
        _need(t, name, torch.bfloat16, 4)
        if tuple(t.shape) != (B, Hq, N, d):
            raise ValueError(f"{name} must be [B, Hq, N, d]")
    if route_mask is not None:
        _need(route_mask, "route_mask", torch.uint8, 2)
    if dk_accum is not None:
        _need(dk_accum, "dk_accum", torch.bfloat16, 4)
        if dk_accum.shape != k.shape:
            raise ValueError("dk_accum must have the shape of k")
    dev = k.device
    if workspace is None:
        workspace = torch.empty(max(int(lib.ea_router_ste_backward_workspace_size(
            B, Hkv, N, d, hidden, Hq)), 16), dtype=torch.uint8, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    dr = torch.empty((B, Hq), **f32)
    dw1, db1 = torch.empty_like(w1), torch.empty_like(b1)
    dw2, db2 = torch.empty_like(w2), torch.empty_like(b2)
    dk_pool = torch.empty((B, Hkv * d), **f32)
    rc = lib.ea_router_ste_backward(
        k.data_ptr(), B, Hkv, N, d, w1.data_ptr(), b1.data_ptr(), hidden, w2.data_ptr(),
        b2.data_ptr(), Hq, g0.data_ptr(), g1.data_ptr(), float(tau), dout.data_ptr(),
        out.data_ptr(), out_other.data_ptr(),
        route_mask.data_ptr() if route_mask is not None else None, dr.data_ptr(), dw1.data_ptr(),
        db1.data_ptr(),
        dw2.data_ptr(), db2.data_ptr(), dk_pool.data_ptr(),
        dk_accum.data_ptr() if dk_accum is not None else None, workspace.data_ptr(),
        workspace.numel(), _stream_ptr(stream, dev))
    check(rc, "ea_router_ste_backward")
    return dr, dw1, db1, dw2, db2, dk_pool


def ea_get_device_status(workspace: torch.Tensor,
                         stream: Optional[torch.cuda.Stream] = None) -> int:
    lib = _lib.load()
    st = ctypes.c_int(0)
    rc = lib.ea_get_device_status(workspace.data_ptr(), _stream_ptr(stream, workspace.device),
                                  ctypes.byref(st))
    check(rc, "ea_get_device_status")
    return int(st.value)


# ---------------------------------------------------------------- schedule view
def _host_mask(mask) -> np.ndarray:
    m = mask.detach().cpu().numpy() if isinstance(mask, torch.Tensor) else np.asarray(mask)
    return np.ascontiguousarray(m.astype(np.uint8).reshape(-1))


def ea_schedule_units(mask, p: EaAttnParams) -> np.ndarray:
    """[U, 6] int32 rows (sparse, b, h0, h1, row0, n_kv_tiles) in schedule order.
    A paired unit (h1 != h0) holds rows [row0, row0 + 128) of heads h0 and h1;
    a single unit (h1 == h0) rows [row0, row0 + 256) of head h0."""
    lib = _lib.load()
    m = _host_mask(mask)
    n = lib.ea_schedule_units(m.ctypes.data, ctypes.byref(p), None, 0)
    if n < 0:
        raise ValueError("invalid schedule arguments")
    out = np.zeros((max(n, 1), 6), dtype=np.int32)
    lib.ea_schedule_units(m.ctypes.data, ctypes.byref(p), out.ctypes.data, n)
    return out[:n]


def ea_schedule_units_varlen(mask, p: EaVarlenParams, cu_seqlens) -> np.ndarray:
    """Schedule of a packed batch (cu_seqlens on the host): [U, 6] int32 rows."""
    lib = _lib.load()
    m = _host_mask(mask)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    n = lib.ea_schedule_units_varlen(m.ctypes.data, ctypes.byref(p), cu.ctypes.data, None, 0)
    if n < 0:
        raise ValueError("invalid schedule arguments")
    out = np.zeros((max(n, 1), 6), dtype=np.int32)
    lib.ea_schedule_units_varlen(m.ctypes.data, ctypes.byref(p), cu.ctypes.data,
                                 out.ctypes.data, n)
    return out[:n]


def ea_schedule_unit_tiles(mask, p: EaAttnParams, rank: int):
    """(tiles int32 [T], codes int32 [T, 2]) of one unit."""
    lib = _lib.load()
    m = _host_mask(mask)
    cap = (p.N + 127) // 128 + 1
    tiles = np.zeros(cap, dtype=np.int32)
    codes = np.zeros((cap, 2), dtype=np.int32)
    n = lib.ea_schedule_unit_tiles(m.ctypes.data, ctypes.byref(p), int(rank), tiles.ctypes.data,
                                   codes.ctypes.data, cap)
    if n < 0:
        raise ValueError("invalid schedule arguments")
    return tiles[:n], codes[:n]


def ea_attn_grid_size(p: EaAttnParams, num_sms: int) -> int:
    return int(_lib.load().ea_attn_grid_size(ctypes.byref(p), int(num_sms)))


# ---------------------------------------------------------------- host-buffer path
def ea_hybrid_attn_host_workspace_size(p: EaAttnParams, hidden: int = 0) -> int:
    return int(_lib.load().ea_hybrid_attn_host_workspace_size(ctypes.byref(p), int(hidden)))


def ea_shutdown() -> None:
    """Release the library's copy streams (see include/ea.h)."""
    check(_lib.load().ea_shutdown(), "ea_shutdown")


def ea_hybrid_attn_host_chunks(p: EaAttnParams, kv_heads_per_chunk: int = 0) -> int:
    return int(_lib.load().ea_hybrid_attn_host_chunks(ctypes.byref(p), int(kv_heads_per_chunk)))


def _host_ptr(t: torch.Tensor, name: str, dtype, numel: int) -> int:
    if t.device.type != "cpu" or t.dtype != dtype or not t.is_contiguous() or t.numel() != numel:
        raise ValueError(f"{name} must be a contiguous host {dtype} tensor of {numel} elements")
    return t.data_ptr()


def ea_hybrid_attn_prefill_host(q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor,
                                sink: int, window: int, *, out_host: torch.Tensor,
                                workspace: torch.Tensor, router=None, threshold: float = 0.0,
                                route_mask_host: Optional[torch.Tensor] = None,
                                route_mask_out_host: Optional[torch.Tensor] = None,
                                kv_heads_per_chunk: int = 0, softmax_scale: float = 0.0,
                                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Prefill from host buffers (q, k, v, out on the host; pinned for the
    copies to overlap the compute).  router = (w1, b1, w2, b2) device tensors,
    or None with route_mask_host given.  The work is enqueued on `stream`;
    synchronise it before reading out_host."""
    lib = _lib.load()
    B, Hq, N, d = q_host.shape
    Hkv = k_host.shape[1]
    if tuple(k_host.shape) != (B, Hkv, N, d) or v_host.shape != k_host.shape:
        raise ValueError("k_host and v_host must be [B, Hkv, N, d] matching q_host")
    p = make_params(B, Hq, Hkv, N, d, sink, window, softmax_scale)
    nq, nkv = B * Hq * N * d, B * Hkv * N * d
    args = [_host_ptr(q_host, "q_host", torch.bfloat16, nq),
            _host_ptr(k_host, "k_host", torch.bfloat16, nkv),
            _host_ptr(v_host, "v_host", torch.bfloat16, nkv)]
    if router is not None:
        w1, b1, w2, b2 = router
        for name, t, nd in (("w1", w1, 2), ("b1", b1, 1), ("w2", w2, 2), ("b2", b2, 1)):
            _need(t, name, torch.float32, nd)
        args += [None, w1.data_ptr(), b1.data_ptr(), int(w1.shape[0]), w2.data_ptr(),
                 b2.data_ptr(), float(threshold)]
        device = w1.device
    else:
        if route_mask_host is None:
            raise ValueError("route_mask_host is required without a router")
        args += [_host_ptr(route_mask_host, "route_mask_host", torch.uint8, B * Hq), None, None,
                 0, None, None, 0.0]
        device = workspace.device
    _host_ptr(out_host, "out_host", torch.bfloat16, nq)
    mask_out = None
    if route_mask_out_host is not None:
        mask_out = _host_ptr(route_mask_out_host, "route_mask_out_host", torch.uint8, B * Hq)
    if workspace.device.type != "cuda" or workspace.dtype != torch.uint8:
        raise ValueError("workspace must be a device uint8 tensor")
    rc = lib.ea_hybrid_attn_prefill_host(*args, ctypes.byref(p), out_host.data_ptr(), mask_out,
                                         int(kv_heads_per_chunk), workspace.data_ptr(),
                                         workspace.numel(), _stream_ptr(stream, device))
    check(rc, "ea_hybrid_attn_prefill_host")
    return out_host


class HostPrefill:
    """One layer's prefill from HOST buffers through ea_hybrid_attn_prefill_host:
    the router (resident device weights) or the caller's mask, then the fused
    attention, with the q/k/v uploads and the out download split by kv-head
    chunks so they overlap the compute.  The device workspace (device copies
    of the inputs and output) and the pinned host output are allocated once
    and reused across calls."""

    def __init__(self, B, Hq, Hkv, N, d, w1, b1, w2, b2, sink, window, device="cuda",
                 threshold=0.0, kv_heads_per_chunk=0):
        self.has_router = w1 is not None
        self.shape_q = (B, Hq, N, d)
        self.shape_kv = (B, Hkv, N, d)
        self.sink, self.window, self.threshold = int(sink), int(window), float(threshold)
        self.kv_heads_per_chunk = int(kv_heads_per_chunk)
        dev = torch.device(device)
        self.router = None
        hidden = 0
        if self.has_router:
            self.router = tuple(t.to(dev).contiguous() for t in (w1, b1, w2, b2))
            hidden = int(w1.shape[0])
        p = make_params(B, Hq, Hkv, N, d, sink, window)
        n = ea_hybrid_attn_host_workspace_size(p, hidden)
        if n == 0:
            raise ValueError("invalid prefill parameters")
        self.workspace = torch.zeros(n, dtype=torch.uint8, device=dev)
        self.chunks = ea_hybrid_attn_host_chunks(p, self.kv_heads_per_chunk)
        self.out_host = torch.empty(self.shape_q, dtype=torch.bfloat16, pin_memory=True)

    def h2d_bytes(self) -> int:
        n = (math.prod(self.shape_q) + 2 * math.prod(self.shape_kv)) * 2
        return n if self.has_router else n + self.shape_q[0] * self.shape_q[1]

    def d2h_bytes(self) -> int:
        return math.prod(self.shape_q) * 2

    def __call__(self, q_host, k_host, v_host, mask_host=None, stream=None):
        if not self.has_router and mask_host is None:
            raise ValueError("HostPrefill without router weights needs mask_host [B, Hq]")
        return ea_hybrid_attn_prefill_host(
            q_host, k_host, v_host, self.sink, self.window, out_host=self.out_host,
            workspace=self.workspace, router=self.router, threshold=self.threshold,
            route_mask_host=None if self.has_router else mask_host.reshape(-1),
            kv_heads_per_chunk=self.kv_heads_per_chunk, stream=stream)


# ---------------------------------------------------------------- decode
def ea_decode_kv_policy(mask, Hkv: int):
    """(cache_slot int32 [B, Hkv], n_full, n_sa): a compact cache for every kv
    head whose query heads are all SA, a full cache for the others."""
    lib = _lib.load()
    m = np.ascontiguousarray(
        (mask.detach().cpu().numpy() if isinstance(mask, torch.Tensor) else np.asarray(mask))
        .astype(np.uint8))
    B, Hq = m.shape
    slots = np.zeros((B, Hkv), dtype=np.int32)
    nf, ns = ctypes.c_int(0), ctypes.c_int(0)
    rc = lib.ea_decode_kv_policy(m.ctypes.data, B, Hq, Hkv, slots.ctypes.data, ctypes.byref(nf),
                                 ctypes.byref(ns))
    if rc != 0:
        raise ValueError("invalid kv policy arguments")
    return slots, int(nf.value), int(ns.value)


def make_decode_params(B, Hq, Hkv, d, sink, window, max_len, n_full, n_sa,
                       softmax_scale=0.0) -> EaDecodeParams:
    return EaDecodeParams(int(B), int(Hq), int(Hkv), int(d), int(sink), int(window),
                          int(max_len), float(softmax_scale), int(n_full), int(n_sa))


def decode_workspace(p: EaDecodeParams, device) -> torch.Tensor:
    n = int(_lib.load().ea_decode_workspace_size(ctypes.byref(p)))
    if n == 0:
        raise ValueError("invalid decode parameters")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def ea_hybrid_attn_decode(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                          pos: torch.Tensor, route_mask: torch.Tensor, cache_slot: torch.Tensor,
                          k_full, v_full, k_sa, v_sa, sink: int, window: int, max_len: int, *,
                          softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None,
                          stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """One decode step: append k_new/v_new at pos, attend, return out [B, Hq, d]."""
    lib = _lib.load()
    _need(q, "q", torch.bfloat16, 3)
    _need(k_new, "k_new", torch.bfloat16, 3)
    _need(v_new, "v_new", torch.bfloat16, 3)
    _need(pos, "pos", torch.int32, 1)
    _need(route_mask, "route_mask", torch.uint8)
    _need(cache_slot, "cache_slot", torch.int32)
    B, Hq, d = q.shape
    Hkv = k_new.shape[1]
    for name, t in (("k_full", k_full), ("v_full", v_full), ("k_sa", k_sa), ("v_sa", v_sa)):
        if t is not None:
            _need(t, name, torch.bfloat16, 3)
    n_full = k_full.shape[0] if k_full is not None else 0
    n_sa = k_sa.shape[0] if k_sa is not None else 0
    if k_full is not None and tuple(k_full.shape[1:]) != (max_len, d):
        raise ValueError("k_full must be [n_full, max_len, d]")
    if k_sa is not None and tuple(k_sa.shape[1:]) != (sink + window, d):
        raise ValueError("k_sa must be [n_sa, sink + window, d]")
    for a, b_, name in ((k_full, v_full, "v_full"), (k_sa, v_sa, "v_sa")):
        if (a is None) != (b_ is None) or (a is not None and a.shape != b_.shape):
            raise ValueError(f"{name} must match its k cache")
    p = make_decode_params(B, Hq, Hkv, d, sink, window, max_len, n_full, n_sa, softmax_scale)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = decode_workspace(p, q.device)
    ptr = (lambda t: t.data_ptr() if t is not None else None)
    rc = lib.ea_hybrid_attn_decode(q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(),
                                   pos.data_ptr(), route_mask.data_ptr(), cache_slot.data_ptr(),
                                   ptr(k_full), ptr(v_full), ptr(k_sa), ptr(v_sa),
                                   ctypes.byref(p), out.data_ptr(), workspace.data_ptr(),
                                   workspace.numel(), _stream_ptr(stream, q.device))
    check(rc, "ea_hybrid_attn_decode")
    return out
