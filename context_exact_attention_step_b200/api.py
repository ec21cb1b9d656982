"""PyTorch-facing binding of the C ABI (argument marshalling only).

Each function checks shapes/dtypes/devices, allocates outputs and workspaces
with PyTorch when the caller does not pass them, and calls the function of the
same name in ``libcp_attn.so`` on the current CUDA stream.  Every step of the
computation runs in the library's CUDA kernels; nothing here computes.
"""
from __future__ import annotations

import ctypes
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np
import torch

from . import _lib
from ._lib import check, cp_chunk, lib

_LAYOUTS = {"contiguous": _lib.CP_LAYOUT_CONTIGUOUS, "zigzag": _lib.CP_LAYOUT_ZIGZAG,
            "striped": _lib.CP_LAYOUT_STRIPED}


def _vp(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream: Optional[torch.cuda.Stream] = None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(name: str, t: torch.Tensor, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _chunks(chunks: Optional[Sequence[Tuple[int, int]]], rows: int):
    if chunks is None:
        chunks = [(0, rows)]
    arr = (cp_chunk * len(chunks))()
    for i, (s, n) in enumerate(chunks):
        arr[i].start, arr[i].len = int(s), int(n)
    return arr, len(chunks)


def _cu_host(cu) -> Tuple[Optional[ctypes.Array], int, Optional[np.ndarray]]:
    if cu is None:
        return None, 0, None
    a = np.ascontiguousarray(np.asarray(cu.cpu() if isinstance(cu, torch.Tensor) else cu, dtype=np.int32))
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), int(a.size - 1), a


def block_attn_fwd(q, k, v, q_chunks=None, k_chunks=None, causal=True, cu_seqlens=None, softmax_scale=0.0,
                   o=None, lse=None, stream=None):
    """One block pair: q [n_q, hq, dh] vs k, v [n_k, hkv, dh] (bf16, CUDA).
    q_chunks / k_chunks: [(global_start, len), ...] covering the rows in order
    (default: positions 0..n-1).  cu_seqlens: CUDA int32 [n_docs + 1] or None.
    Returns (O [n_q, hq, dh] fp32, LSE [hq, n_q] fp32)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda(n, t, torch.bfloat16)
    n_q, hq, dh = q.shape
    n_k, hkv, _ = k.shape
    if o is None:
        o = torch.empty((n_q, hq, dh), device=q.device, dtype=torch.float32)
    if lse is None:
        lse = torch.empty((hq, n_q), device=q.device, dtype=torch.float32)
    qc, nqc = _chunks(q_chunks, n_q)
    kc, nkc = _chunks(k_chunks, n_k)
    n_docs = 0
    if cu_seqlens is not None:
        _need_cuda("cu_seqlens", cu_seqlens, torch.int32)
        n_docs = cu_seqlens.numel() - 1
    check(lib().cp_block_attn_fwd(_vp(q), _vp(k), _vp(v), _lib.CP_BF16, n_q, n_k, hq, hkv, dh, qc, nqc, kc, nkc,
                                  _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE, _vp(cu_seqlens), n_docs,
                                  float(softmax_scale), _vp(o), _vp(lse), _stream(stream)))
    return o, lse


def lse_merge(o_parts: Sequence[torch.Tensor], lse_parts: Sequence[torch.Tensor], o_out=None, lse_out=None,
              bf16_out=False, stream=None):
    """Fold partials O_i [rows, h, dh] fp32 with LSE_i [h, rows] fp32."""
    n = len(o_parts)
    rows, h, dh = o_parts[0].shape
    for i in range(n):
        _need_cuda(f"o_parts[{i}]", o_parts[i], torch.float32)
        _need_cuda(f"lse_parts[{i}]", lse_parts[i], torch.float32)
    if o_out is None:
        o_out = torch.empty((rows, h, dh), device=o_parts[0].device, dtype=torch.float32)
    if lse_out is None:
        lse_out = torch.empty((h, rows), device=o_parts[0].device, dtype=torch.float32)
    o16 = torch.empty((rows, h, dh), device=o_out.device, dtype=torch.bfloat16) if bf16_out else None
    op = (ctypes.c_void_p * n)(*[t.data_ptr() for t in o_parts])
    lp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in lse_parts])
    check(lib().cp_lse_merge(n, op, lp, rows, h, dh, _vp(o_out), _vp(lse_out), _vp(o16), _stream(stream)))
    return (o_out, lse_out, o16) if bf16_out else (o_out, lse_out)


def ring_attn_workspace_size(S, hq, hkv, dh, P, layout="contiguous", causal=True, dtype=torch.bfloat16,
                             cu_seqlens=None) -> int:
    cu_p, n_docs, _keep = _cu_host(cu_seqlens)
    out = ctypes.c_size_t(0)
    check(lib().cp_ring_attn_workspace_size(S, hq, hkv, dh, P, _LAYOUTS[layout],
                                            _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE,
                                            _lib.CP_FP32 if dtype == torch.float32 else _lib.CP_BF16, cu_p, n_docs,
                                            ctypes.byref(out)))
    return int(out.value)


def ring_attn_fwd(q, k, v, P, layout="contiguous", causal=True, cu_seqlens=None, cu_seqlens_dev=None,
                  softmax_scale=0.0, o=None, lse=None, workspace=None, stream=None):
    """Ring attention over P virtual ranks.  q [S, hq, dh], k, v [S, hkv, dh]
    (bf16 or fp32, CUDA) in the rank-major order of ``layout``.  cu_seqlens:
    host int32 document table (list / CPU tensor) or None; its device copy is
    made here unless ``cu_seqlens_dev`` is given.  Returns (O [S, hq, dh] fp32,
    LSE [hq, S] fp32) in the same order."""
    dtype = q.dtype
    if dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q must be bf16 or fp32")
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda(n, t, dtype)
    S, hq, dh = q.shape
    hkv = k.shape[1]
    cu_p, n_docs, cu_np = _cu_host(cu_seqlens)
    if n_docs > 0 and cu_seqlens_dev is None:
        cu_seqlens_dev = torch.from_numpy(cu_np).to(q.device)
    if o is None:
        o = torch.empty((S, hq, dh), device=q.device, dtype=torch.float32)
    if lse is None:
        lse = torch.empty((hq, S), device=q.device, dtype=torch.float32)
    if workspace is None:
        need = ring_attn_workspace_size(S, hq, hkv, dh, P, layout, causal, dtype, cu_seqlens)
        workspace = torch.empty(max(need, 256), device=q.device, dtype=torch.uint8)
    check(lib().cp_ring_attn_fwd(_vp(q), _vp(k), _vp(v), _lib.CP_FP32 if dtype == torch.float32 else _lib.CP_BF16,
                                 S, hq, hkv, dh, P, _LAYOUTS[layout],
                                 _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE, cu_p, _vp(cu_seqlens_dev),
                                 n_docs, float(softmax_scale), _vp(o), _vp(lse), _vp(workspace),
                                 workspace.numel(), _stream(stream)))
    return o, lse


def ring_attn_fwd_noalloc(q, k, v, P, layout="contiguous", causal=True, cu_seqlens=None, cu_seqlens_dev=None,
                          softmax_scale=0.0, o=None, lse=None, stream=None):
    """ring_attn_fwd without a workspace, for callers that may not allocate
    device memory while they run: the library keeps the partial results in
    its own fixed scratch array (CP_NOALLOC_SCRATCH_BYTES per device).  Pass
    preallocated ``o``, ``lse`` and ``cu_seqlens_dev`` to allocate nothing on
    this path either.  Calls overlapping on the GPU share that scratch and
    race; the first call on a device must come before any stream capture."""
    dtype = q.dtype
    if dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q must be bf16 or fp32")
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda(n, t, dtype)
    S, hq, dh = q.shape
    hkv = k.shape[1]
    cu_p, n_docs, cu_np = _cu_host(cu_seqlens)
    if n_docs > 0 and cu_seqlens_dev is None:
        cu_seqlens_dev = torch.from_numpy(cu_np).to(q.device)
    if o is None:
        o = torch.empty((S, hq, dh), device=q.device, dtype=torch.float32)
    if lse is None:
        lse = torch.empty((hq, S), device=q.device, dtype=torch.float32)
    check(lib().cp_ring_attn_fwd_noalloc(_vp(q), _vp(k), _vp(v),
                                         _lib.CP_FP32 if dtype == torch.float32 else _lib.CP_BF16, S, hq, hkv, dh, P,
                                         _LAYOUTS[layout], _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE,
                                         cu_p, _vp(cu_seqlens_dev), n_docs, float(softmax_scale), _vp(o), _vp(lse),
                                         _stream(stream)))
    return o, lse


def ulysses_permute(x, P, direction="seq_to_head", out=None, stream=None):
    """seq_to_head: x [S, h, dh] (= [P][S/P][h][dh]) -> [P, S, h/P, dh].
    head_to_seq: x [P, S, h/P, dh] -> [S, h, dh].  Bit-exact copy."""
    _need_cuda("x", x)
    eb = x.element_size()
    if direction == "seq_to_head":
        S, h, dh = x.shape
        shape = (P, S, h // P, dh)
        d = _lib.CP_SEQ_TO_HEAD
    else:
        p_, S, hg, dh = x.shape
        h = hg * P
        shape = (S, h, dh)
        d = _lib.CP_HEAD_TO_SEQ
    if out is None:
        out = torch.empty(shape, device=x.device, dtype=x.dtype)
    check(lib().cp_ulysses_permute(_vp(x), _vp(out), P, S, h, dh, eb, d, _stream(stream)))
    return out


def head_block_split(x, P, inverse=False, out=None, stream=None):
    """inverse=False: x [n, h, dh] -> [P, n, h/P, dh] (block r for rank r);
    inverse=True: x [P, n, h/P, dh] -> [n, h, dh].  Bit-exact copy."""
    _need_cuda("x", x)
    if not inverse:
        n, h, dh = x.shape
        shape = (P, n, h // P, dh)
    else:
        p_, n, hg, dh = x.shape
        h = hg * P
        shape = (n, h, dh)
    if out is None:
        out = torch.empty(shape, device=x.device, dtype=x.dtype)
    check(lib().cp_head_block_split(_vp(x), _vp(out), n, h, dh, P, x.element_size(), 1 if inverse else 0,
                                    _stream(stream)))
    return out


def zigzag_reorder(x, P, inverse=False, seq_dim=0, out=None, stream=None):
    """Natural <-> rank-major zigzag order along ``seq_dim`` (0 for [S, ...]
    tensors, 1 for [h, S] LSE tensors)."""
    _need_cuda("x", x)
    if seq_dim == 0:
        batch, S = 1, x.shape[0]
        row_bytes = x[0].numel() * x.element_size() if x.dim() > 1 else x.element_size()
    elif seq_dim == 1 and x.dim() == 2:
        batch, S = x.shape
        row_bytes = x.element_size()
    else:
        raise ValueError("seq_dim must be 0, or 1 for a 2-D tensor")
    if out is None:
        out = torch.empty_like(x)
    check(lib().cp_zigzag_reorder(_vp(x), _vp(out), P, S, batch, row_bytes, 1 if inverse else 0, _stream(stream)))
    return out


def striped_reorder(x, P, inverse=False, seq_dim=0, out=None, stream=None):
    """Natural <-> rank-major striped order (token t on rank t mod P) along
    ``seq_dim`` (0 for [S, ...] tensors, 1 for [h, S] LSE tensors)."""
    _need_cuda("x", x)
    if seq_dim == 0:
        batch, S = 1, x.shape[0]
        row_bytes = x[0].numel() * x.element_size() if x.dim() > 1 else x.element_size()
    elif seq_dim == 1 and x.dim() == 2:
        batch, S = x.shape
        row_bytes = x.element_size()
    else:
        raise ValueError("seq_dim must be 0, or 1 for a 2-D tensor")
    if out is None:
        out = torch.empty_like(x)
    check(lib().cp_striped_reorder(_vp(x), _vp(out), P, S, batch, row_bytes, 1 if inverse else 0, _stream(stream)))
    return out


def ulysses_attn_workspace_size(S, hq, hkv, dh, P) -> int:
    out = ctypes.c_size_t(0)
    check(lib().cp_ulysses_attn_workspace_size(S, hq, hkv, dh, P, ctypes.byref(out)))
    return int(out.value)


def ulysses_attn_fwd(q, k, v, P, causal=True, softmax_scale=0.0, o=None, lse=None, workspace=None, stream=None):
    """Ulysses path: q [S, hq, dh], k, v [S, hkv, dh] bf16 in natural order
    (rank p holds rows p*S/P..).  Returns (O [S, hq, dh] fp32, LSE [hq, S])."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda(n, t, torch.bfloat16)
    S, hq, dh = q.shape
    hkv = k.shape[1]
    if o is None:
        o = torch.empty((S, hq, dh), device=q.device, dtype=torch.float32)
    if lse is None:
        lse = torch.empty((hq, S), device=q.device, dtype=torch.float32)
    if workspace is None:
        workspace = torch.empty(ulysses_attn_workspace_size(S, hq, hkv, dh, P), device=q.device, dtype=torch.uint8)
    check(lib().cp_ulysses_attn_fwd(_vp(q), _vp(k), _vp(v), S, hq, hkv, dh, P,
                                    _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE, float(softmax_scale),
                                    _vp(o), _vp(lse), _vp(workspace), workspace.numel(), _stream(stream)))
    return o, lse


def usp_attn_workspace_size(S, hq, hkv, dh, Pr, Pu, layout="contiguous", causal=True, cu_seqlens=None) -> int:
    cu_p, n_docs, _keep = _cu_host(cu_seqlens)
    out = ctypes.c_size_t(0)
    check(lib().cp_usp_attn_workspace_size(S, hq, hkv, dh, Pr, Pu, _LAYOUTS[layout],
                                           _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE, cu_p, n_docs,
                                           ctypes.byref(out)))
    return int(out.value)


def usp_attn_fwd(q, k, v, Pr, Pu, layout="contiguous", causal=True, cu_seqlens=None, cu_seqlens_dev=None,
                 softmax_scale=0.0, o=None, lse=None, workspace=None, stream=None):
    """Ulysses inside groups of Pu virtual ranks, Ring across Pr groups.
    q [S, hq, dh], k, v [S, hkv, dh] bf16 (CUDA) in the rank-major order of
    ``layout`` over Pr ring shards (the buffer ring_attn_fwd takes with
    P = Pr).  Returns (O [S, hq, dh] fp32, LSE [hq, S] fp32) in that order."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda(n, t, torch.bfloat16)
    S, hq, dh = q.shape
    hkv = k.shape[1]
    cu_p, n_docs, cu_np = _cu_host(cu_seqlens)
    if n_docs > 0 and cu_seqlens_dev is None:
        cu_seqlens_dev = torch.from_numpy(cu_np).to(q.device)
    if o is None:
        o = torch.empty((S, hq, dh), device=q.device, dtype=torch.float32)
    if lse is None:
        lse = torch.empty((hq, S), device=q.device, dtype=torch.float32)
    if workspace is None:
        need = usp_attn_workspace_size(S, hq, hkv, dh, Pr, Pu, layout, causal, cu_seqlens)
        workspace = torch.empty(max(need, 256), device=q.device, dtype=torch.uint8)
    check(lib().cp_usp_attn_fwd(_vp(q), _vp(k), _vp(v), S, hq, hkv, dh, Pr, Pu, _LAYOUTS[layout],
                                _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE, cu_p, _vp(cu_seqlens_dev),
                                n_docs, float(softmax_scale), _vp(o), _vp(lse), _vp(workspace), workspace.numel(),
                                _stream(stream)))
    return o, lse


def ring_attn_bwd_workspace_size(S, hq, hkv, dh, P, layout="contiguous", causal=True, cu_seqlens=None) -> int:
    cu_p, n_docs, _keep = _cu_host(cu_seqlens)
    out = ctypes.c_size_t(0)
    check(lib().cp_ring_attn_bwd_workspace_size(S, hq, hkv, dh, P, _LAYOUTS[layout],
                                                _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE, cu_p, n_docs,
                                                ctypes.byref(out)))
    return int(out.value)


def ring_attn_bwd(q, k, v, o, lse, do, P, layout="contiguous", causal=True, cu_seqlens=None, cu_seqlens_dev=None,
                  softmax_scale=0.0, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients of ring_attn_fwd.  q [S, hq, dh], k, v [S, hkv, dh], do
    [S, hq, dh] bf16 and the forward's o [S, hq, dh], lse [hq, S] fp32, all
    CUDA and in the rank-major order of ``layout``.  Returns (dQ [S, hq, dh],
    dK [S, hkv, dh], dV [S, hkv, dh]) fp32 in the same order."""
    for n, t in (("q", q), ("k", k), ("v", v), ("do", do)):
        _need_cuda(n, t, torch.bfloat16)
    _need_cuda("o", o, torch.float32)
    _need_cuda("lse", lse, torch.float32)
    S, hq, dh = q.shape
    hkv = k.shape[1]
    cu_p, n_docs, cu_np = _cu_host(cu_seqlens)
    if n_docs > 0 and cu_seqlens_dev is None:
        cu_seqlens_dev = torch.from_numpy(cu_np).to(q.device)
    if dq is None:
        dq = torch.empty((S, hq, dh), device=q.device, dtype=torch.float32)
    if dk is None:
        dk = torch.empty((S, hkv, dh), device=q.device, dtype=torch.float32)
    if dv is None:
        dv = torch.empty((S, hkv, dh), device=q.device, dtype=torch.float32)
    if workspace is None:
        need = ring_attn_bwd_workspace_size(S, hq, hkv, dh, P, layout, causal, cu_seqlens)
        workspace = torch.empty(max(need, 256), device=q.device, dtype=torch.uint8)
    check(lib().cp_ring_attn_bwd(_vp(q), _vp(k), _vp(v), _vp(o), _vp(lse), _vp(do), S, hq, hkv, dh, P,
                                 _LAYOUTS[layout], _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE, cu_p,
                                 _vp(cu_seqlens_dev), n_docs, float(softmax_scale), _vp(dq), _vp(dk), _vp(dv),
                                 _vp(workspace), workspace.numel(), _stream(stream)))
    return dq, dk, dv


BWD_DQ = _lib.CP_BWD_DQ      # block_attn_bwd parts: the dQ kernel
BWD_DKDV = _lib.CP_BWD_DKDV  # the dK/dV kernel


def attn_bwd_prep(o, lse, do, lg=None, dd=None, stream=None):
    """Per-row vectors of the backward: lg = LSE * log2(e) (0 where LSE is
    -inf) and dd = rowsum(dO * O), both [hq, n] fp32, from the forward's o
    [n, hq, dh], lse [hq, n] fp32 and do [n, hq, dh] bf16 (CUDA)."""
    _need_cuda("o", o, torch.float32)
    _need_cuda("lse", lse, torch.float32)
    _need_cuda("do", do, torch.bfloat16)
    n, hq, dh = o.shape
    if lg is None:
        lg = torch.empty((hq, n), device=o.device, dtype=torch.float32)
    if dd is None:
        dd = torch.empty((hq, n), device=o.device, dtype=torch.float32)
    check(lib().cp_attn_bwd_prep(_vp(o), _vp(do), _vp(lse), n, hq, dh, _vp(lg), _vp(dd), _stream(stream)))
    return lg, dd


def block_attn_bwd(q, k, v, do, lg, dd, q_chunks=None, k_chunks=None, causal=True, cu_seqlens=None,
                   softmax_scale=0.0, dq=None, dk=None, dv=None, parts=BWD_DQ | BWD_DKDV, accumulate=False,
                   stream=None):
    """Gradient contribution of one block pair: q, do [n_q, hq, dh] vs k, v
    [n_k, hkv, dh] (bf16, CUDA), lg, dd from ``attn_bwd_prep`` of the query
    rows; chunks and mask as ``block_attn_fwd``.  parts: BWD_DQ, BWD_DKDV or
    both.  accumulate: add to dq / dk / dv instead of overwriting them.
    Returns (dq [n_q, hq, dh], dk, dv [n_k, hkv, dh]) fp32 (None for a part
    not computed and not given)."""
    for n, t in (("q", q), ("k", k), ("v", v), ("do", do)):
        _need_cuda(n, t, torch.bfloat16)
    _need_cuda("lg", lg, torch.float32)
    _need_cuda("dd", dd, torch.float32)
    n_q, hq, dh = q.shape
    n_k, hkv, _ = k.shape
    if parts & _lib.CP_BWD_DQ and dq is None:
        dq = torch.empty((n_q, hq, dh), device=q.device, dtype=torch.float32)
    if parts & _lib.CP_BWD_DKDV:
        if dk is None:
            dk = torch.empty((n_k, hkv, dh), device=q.device, dtype=torch.float32)
        if dv is None:
            dv = torch.empty((n_k, hkv, dh), device=q.device, dtype=torch.float32)
    qc, nqc = _chunks(q_chunks, n_q)
    kc, nkc = _chunks(k_chunks, n_k)
    n_docs = 0
    if cu_seqlens is not None:
        _need_cuda("cu_seqlens", cu_seqlens, torch.int32)
        n_docs = cu_seqlens.numel() - 1
    check(lib().cp_block_attn_bwd(_vp(q), _vp(k), _vp(v), _vp(do), _vp(lg), _vp(dd), n_q, n_k, hq, hkv, dh, qc, nqc,
                                  kc, nkc, _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE, _vp(cu_seqlens),
                                  n_docs, float(softmax_scale), _vp(dq), _vp(dk), _vp(dv), int(parts),
                                  1 if accumulate else 0, _stream(stream)))
    return dq, dk, dv


def _bwd_outputs(q, k, dq, dk, dv):
    S, hq, dh = q.shape
    hkv = k.shape[1]
    if dq is None:
        dq = torch.empty((S, hq, dh), device=q.device, dtype=torch.float32)
    if dk is None:
        dk = torch.empty((S, hkv, dh), device=q.device, dtype=torch.float32)
    if dv is None:
        dv = torch.empty((S, hkv, dh), device=q.device, dtype=torch.float32)
    return dq, dk, dv


def _bwd_check(q, k, v, o, lse, do):
    for n, t in (("q", q), ("k", k), ("v", v), ("do", do)):
        _need_cuda(n, t, torch.bfloat16)
    _need_cuda("o", o, torch.float32)
    _need_cuda("lse", lse, torch.float32)


def usp_attn_bwd(q, k, v, o, lse, do, Pr, Pu, layout="contiguous", causal=True, cu_seqlens=None,
                 cu_seqlens_dev=None, softmax_scale=0.0, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients of usp_attn_fwd: tensors as for ring_attn_bwd, in the
    forward's storage order (``layout`` over Pr ring groups)."""
    _bwd_check(q, k, v, o, lse, do)
    S, hq, dh = q.shape
    hkv = k.shape[1]
    cu_p, n_docs, cu_np = _cu_host(cu_seqlens)
    if n_docs > 0 and cu_seqlens_dev is None:
        cu_seqlens_dev = torch.from_numpy(cu_np).to(q.device)
    dq, dk, dv = _bwd_outputs(q, k, dq, dk, dv)
    if workspace is None:
        out = ctypes.c_size_t(0)
        check(lib().cp_usp_attn_bwd_workspace_size(S, hq, hkv, dh, Pr, Pu, _LAYOUTS[layout],
                                                   _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE, cu_p,
                                                   n_docs, ctypes.byref(out)))
        workspace = torch.empty(max(int(out.value), 256), device=q.device, dtype=torch.uint8)
    check(lib().cp_usp_attn_bwd(_vp(q), _vp(k), _vp(v), _vp(o), _vp(lse), _vp(do), S, hq, hkv, dh, Pr, Pu,
                                _LAYOUTS[layout], _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE, cu_p,
                                _vp(cu_seqlens_dev), n_docs, float(softmax_scale), _vp(dq), _vp(dk), _vp(dv),
                                _vp(workspace), workspace.numel(), _stream(stream)))
    return dq, dk, dv


def ulysses_attn_bwd(q, k, v, o, lse, do, P, causal=True, softmax_scale=0.0, dq=None, dk=None, dv=None,
                     workspace=None, stream=None):
    """Gradients of ulysses_attn_fwd, tensors in natural sequence order."""
    _bwd_check(q, k, v, o, lse, do)
    S, hq, dh = q.shape
    hkv = k.shape[1]
    dq, dk, dv = _bwd_outputs(q, k, dq, dk, dv)
    if workspace is None:
        out = ctypes.c_size_t(0)
        check(lib().cp_ulysses_attn_bwd_workspace_size(S, hq, hkv, dh, P, ctypes.byref(out)))
        workspace = torch.empty(max(int(out.value), 256), device=q.device, dtype=torch.uint8)
    check(lib().cp_ulysses_attn_bwd(_vp(q), _vp(k), _vp(v), _vp(o), _vp(lse), _vp(do), S, hq, hkv, dh, P,
                                    _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE, float(softmax_scale),
                                    _vp(dq), _vp(dk), _vp(dv), _vp(workspace), workspace.numel(), _stream(stream)))
    return dq, dk, dv


def ring_schedule(S, P, layout="contiguous", causal=True, cu_seqlens=None):
    """Host-only view of the ring-step schedule: arrays of P*P entries indexed
    r*P + t (see cp_ring_schedule)."""
    cu_p, n_docs, _keep = _cu_host(cu_seqlens)
    src = np.zeros(P * P, np.int32)
    launched = np.zeros(P * P, np.int32)
    q_rows = np.zeros(P * P, np.int32)
    live = np.zeros(P * P, np.int64)
    p32 = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    check(lib().cp_ring_schedule(S, P, _LAYOUTS[layout], _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE, cu_p,
                                 n_docs, p32(src), p32(launched), p32(q_rows),
                                 live.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))))
    return dict(src=src, launched=launched, q_rows=q_rows, live_pairs=live)


def count_live_pairs(S, causal=True, cu_seqlens=None) -> int:
    cu_p, n_docs, _keep = _cu_host(cu_seqlens)
    out = ctypes.c_int64(0)
    check(lib().cp_count_live_pairs(S, _lib.CP_MASK_CAUSAL if causal else _lib.CP_MASK_NONE, cu_p, n_docs,
                                    ctypes.byref(out)))
    return int(out.value)


def kernel_launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    n = ctypes.c_uint64(0)
    check(lib().cp_kernel_launch_count(ctypes.byref(n)))
    return int(n.value)


def set_profile_events(attn_begin=None, attn_end=None, merge_end=None):
    """Record torch.cuda.Event objects around the attention / merge phases of
    the next composite calls on this thread (None turns it off).  Each event
    must have been recorded once so that its CUDA handle exists."""
    h = lambda e: ctypes.c_void_p(e.cuda_event) if e is not None else ctypes.c_void_p(0)
    check(lib().cp_set_profile_events(h(attn_begin), h(attn_end), h(merge_end)))


def selftest_wait_timeout(timeout_ns=1_000_000, stream=None):
    """Launch the bounded-wait self-test (see cp_selftest_wait_timeout)."""
    check(lib().cp_selftest_wait_timeout(int(timeout_ns), _stream(stream)))


def device_error(clear=True) -> int:
    bits = ctypes.c_uint32(0)
    check(lib().cp_device_error(ctypes.byref(bits), 1 if clear else 0))
    return int(bits.value)
