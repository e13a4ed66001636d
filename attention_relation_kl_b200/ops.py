"""PyTorch-facing binding of librelkl.so, with the C ABI's names.

Argument marshalling only: every computation runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current CUDA stream.  There is
no CPU fallback; calls raise if the library is missing or a tensor is not on a
CUDA device.

Layout contract (include/relkl.h): teacher and student are [B, H, N, d]
tensors with a contiguous last dimension; kl is [B, H, N] float32, stats is
[B, H, N, 4] float32 (m, lse_t, lse_s, w) and dX_s is [B, H, N, d] float32.
"""
from __future__ import annotations

import ctypes
from typing import Dict, List, Optional, Sequence, Tuple

import torch

from . import _abi
from ._abi import check, relkl_desc

__all__ = ["relkl_fwd", "relkl_bwd", "relkl_fwd_qkv", "relkl_bwd_qkv", "relkl_workspace_bytes",
           "relkl_workspace_init", "relkl_get_device_error", "relkl_set_wait_timeout_ns",
           "relkl_path_for", "workspace", "make_desc", "relation_kl", "RelationKL",
           "relkl_fwd_noalloc", "relkl_rope_bwd", "relkl_weight_grad", "student_weight_grads",
           "relkl_cast_bf16"]

_DTYPES = {torch.bfloat16: _abi.RELKL_BF16, torch.float32: _abi.RELKL_FP32}


def _lengths_ptr(lengths: Optional[torch.Tensor], x: torch.Tensor) -> Optional[int]:
    """Device pointer of per-batch valid lengths (int32 [B] on x's device), or None."""
    if lengths is None:
        return None
    if (lengths.dtype != torch.int32 or lengths.dim() != 1 or lengths.shape[0] != x.shape[0]
            or not lengths.is_contiguous() or lengths.device != x.device):
        raise ValueError("lengths must be a contiguous int32 [B] tensor on the inputs' device")
    return int(lengths.data_ptr())


def _cu_ptr(cu_seqlens: Optional[torch.Tensor], x: torch.Tensor) -> Optional[int]:
    """Device pointer of packed-sequence offsets (int32 [n_seq + 1] on x's device), or None."""
    if cu_seqlens is None:
        return None
    if (cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1
            or not cu_seqlens.is_contiguous() or cu_seqlens.device != x.device):
        raise ValueError("cu_seqlens must be a contiguous int32 [n_seq + 1] tensor on the "
                         "inputs' device")
    if x.shape[0] != 1:
        raise ValueError("packed sequences use [1, H, N, d] tensors")
    return int(cu_seqlens.data_ptr())


def make_desc(x: torch.Tensor, causal: bool = True, scale: float = 0.0,
              lengths: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None,
              max_seqlen: int = 0) -> relkl_desc:
    """C descriptor of a [B, H, N, d] tensor.  ``cu_seqlens`` (int32 [n_seq + 1],
    device) makes it packed sequences on one token axis, B = 1; ``max_seqlen``
    must then bound every sequence's length."""
    if x.dim() != 4:
        raise ValueError("expected a [B, H, N, d] tensor")
    if x.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {x.dtype}")
    d = relkl_desc()
    d.B, d.H, d.N, d.d = (int(v) for v in x.shape)
    for i in range(3):          # a dimension of extent 1 has no meaningful stride
        d.stride[i] = int(x.stride(i)) if x.shape[i] != 1 else 0
    d.stride[3] = 1 if (x.shape[3] == 1 or x.stride(3) == 1) else int(x.stride(3))
    d.dtype = _DTYPES[x.dtype]
    d.causal = 1 if causal else 0
    d.scale = float(scale)
    d.reserved = 0
    d.lengths = _lengths_ptr(lengths, x)
    d.cu_seqlens = _cu_ptr(cu_seqlens, x)
    d.n_seq = 0 if cu_seqlens is None else int(cu_seqlens.numel()) - 1
    d.max_seqlen = 0 if cu_seqlens is None else int(max_seqlen)
    if cu_seqlens is not None and not 0 <= d.max_seqlen <= d.N:
        raise ValueError("max_seqlen must lie in [0, N]")
    return d


def _stream(device: torch.device, stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _cuda(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")


def _check_out(t: torch.Tensor, shape, name: str, device: torch.device) -> None:
    """A caller-provided output must be exactly what the kernels write through
    the raw pointer: contiguous float32 of the given shape on the inputs' device."""
    if t is None:
        raise ValueError(f"{name} must be given")
    if (t.dtype != torch.float32 or tuple(t.shape) != tuple(shape) or not t.is_contiguous()
            or t.device != device):
        raise ValueError(f"{name} must be a contiguous float32 tensor of shape {tuple(shape)} "
                         f"on {device} (got {t.dtype} {tuple(t.shape)} on {t.device}, "
                         f"contiguous={t.is_contiguous()})")


_WS: Dict[int, torch.Tensor] = {}


def relkl_workspace_bytes() -> int:
    return int(_abi.lib().relkl_workspace_bytes())


def relkl_workspace_init(ws: torch.Tensor, stream=None) -> None:
    with torch.cuda.device(ws.device):
        code = _abi.lib().relkl_workspace_init(_ptr(ws), ws.numel() * ws.element_size(),
                                               _stream(ws.device, stream))
    check(code, "relkl_workspace_init")


def workspace(device=None) -> torch.Tensor:
    """A zeroed per-device workspace (the device error record), cached."""
    device = torch.device(device or "cuda")
    idx = device.index if device.index is not None else torch.cuda.current_device()
    ws = _WS.get(idx)
    if ws is None:
        ws = torch.empty(relkl_workspace_bytes(), dtype=torch.uint8, device=f"cuda:{idx}")
        relkl_workspace_init(ws)
        _WS[idx] = ws
    return ws


def relkl_path_for(x: torch.Tensor, causal: bool = True, scale: float = 0.0) -> int:
    d = make_desc(x, causal, scale)
    return int(_abi.lib().relkl_path_for(ctypes.byref(d)))


def _arr(vals, ctype=ctypes.c_void_p):
    return (ctype * len(vals))(*[v if v is not None else None for v in vals])


def _part(part) -> Tuple[int, int]:
    p, n = (0, 1) if part is None else (int(part[0]), int(part[1]))
    if n < 1 or not 0 <= p < n:
        raise ValueError("part must be (index, count) with 0 <= index < count")
    return p, n


def relkl_fwd_qkv(pairs: Sequence[Tuple[torch.Tensor, torch.Tensor]], causal: bool = True,
                  scale: float = 0.0, *, out: Optional[Sequence[Tuple[torch.Tensor, torch.Tensor]]] = None,
                  ws: Optional[torch.Tensor] = None, stream=None,
                  lengths: Optional[torch.Tensor] = None, part=None,
                  cu_seqlens: Optional[torch.Tensor] = None, max_seqlen: int = 0):
    """Forward over 1..3 relations in one launch.  Returns [(kl, stats)] per relation.
    ``cu_seqlens``/``max_seqlen``: packed sequences on one token axis ([1, H, N, d]
    tensors; see relkl_desc), shared by the relations.
    ``lengths``: optional int32 [B] valid lengths (right padding), shared by the relations.
    ``part``: (index, count) to compute only that part of every unit's rows
    (relkl_fwd_qkv_part); outputs allocated here are then zero elsewhere."""
    p_idx, n_parts = _part(part)
    n = len(pairs)
    if not 1 <= n <= 3:
        raise ValueError("1 to 3 relations per call")
    dev = pairs[0][0].device
    descs = (relkl_desc * n)()
    outs = []
    for r, (xt, xs) in enumerate(pairs):
        _cuda(xt, "x_t")
        _cuda(xs, "x_s")
        if xt.shape != xs.shape or xt.stride() != xs.stride() or xt.dtype != xs.dtype:
            raise ValueError("teacher and student must share shape, strides and dtype")
        descs[r] = make_desc(xt, causal, scale, lengths, cu_seqlens, max_seqlen)
        B, H, N, _ = xt.shape
        if xt.device != dev or xs.device != dev:
            raise ValueError("every relation must live on the same device")
        if out is not None:
            kl, st = out[r]
            _check_out(kl, (B, H, N), "kl", dev)
            _check_out(st, (B, H, N, 4), "stats", dev)
        else:
            # rows a call may leave untouched (other parts, tokens past the
            # last packed sequence) come back as zeros
            alloc = torch.empty if (n_parts == 1 and cu_seqlens is None) else torch.zeros
            kl = alloc((B, H, N), dtype=torch.float32, device=dev)
            st = alloc((B, H, N, 4), dtype=torch.float32, device=dev)
        outs.append((kl, st))
    ws = workspace(dev) if ws is None else ws
    args = (n, descs, _arr([_ptr(p[0]) for p in pairs]), _arr([_ptr(p[1]) for p in pairs]),
            _arr([_ptr(o[0]) for o in outs]), _arr([_ptr(o[1]) for o in outs]))
    tail = (_ptr(ws), ws.numel(), _stream(dev, stream))
    with torch.cuda.device(dev):
        if n_parts == 1:
            code = _abi.lib().relkl_fwd_qkv(*args, *tail)
        else:
            code = _abi.lib().relkl_fwd_qkv_part(*args, p_idx, n_parts, *tail)
    check(code, "relkl_fwd_qkv")
    return outs


def relkl_bwd_qkv(pairs: Sequence[Tuple[torch.Tensor, torch.Tensor]], stats: Sequence[torch.Tensor],
                  dkl: Optional[Sequence[Optional[torch.Tensor]]] = None, causal: bool = True,
                  scale: float = 0.0, *, out: Optional[Sequence[torch.Tensor]] = None,
                  ws: Optional[torch.Tensor] = None, stream=None,
                  lengths: Optional[torch.Tensor] = None, part=None,
                  cu_seqlens: Optional[torch.Tensor] = None,
                  max_seqlen: int = 0, dx_dtype: torch.dtype = torch.float32) -> List[torch.Tensor]:
    """Backward over 1..3 relations in one launch.  Returns dX_s per relation (float32).
    ``part``: (index, count) to return only that part's rows' contribution to
    dX_s (relkl_bwd_qkv_part); ``stats`` must then hold every row.
    ``dx_dtype=torch.bfloat16`` returns bf16 copies instead (relkl_cast_bf16 of
    the float32 result, which is then ``out`` or a temporary)."""
    if dx_dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("dx_dtype must be torch.float32 or torch.bfloat16")
    p_idx, n_parts = _part(part)
    n = len(pairs)
    if not 1 <= n <= 3 or len(stats) != n:
        raise ValueError("1 to 3 relations per call, with one stats tensor each")
    dev = pairs[0][0].device
    descs = (relkl_desc * n)()
    dxs = []
    for r, (xt, xs) in enumerate(pairs):
        _cuda(xt, "x_t")
        _cuda(xs, "x_s")
        if xt.shape != xs.shape or xt.stride() != xs.stride() or xt.dtype != xs.dtype:
            raise ValueError("teacher and student must share shape, strides and dtype")
        if xt.device != dev or xs.device != dev:
            raise ValueError("every relation must live on the same device")
        descs[r] = make_desc(xt, causal, scale, lengths, cu_seqlens, max_seqlen)
        B, H, N, _ = xt.shape
        _check_out(stats[r], (B, H, N, 4), "stats", dev)
        if dkl is not None and dkl[r] is not None:
            _check_out(dkl[r], (B, H, N), "dkl", dev)
        dx = out[r] if out is not None else torch.empty(xs.shape, dtype=torch.float32, device=dev)
        _check_out(dx, tuple(xs.shape), "dx_s", dev)
        dxs.append(dx)
    ws = workspace(dev) if ws is None else ws
    dkl_arr = None if dkl is None else _arr([_ptr(g) for g in dkl])
    args = (n, descs, _arr([_ptr(p[0]) for p in pairs]), _arr([_ptr(p[1]) for p in pairs]),
            _arr([_ptr(s) for s in stats]), dkl_arr, _arr([_ptr(d) for d in dxs]))
    tail = (_ptr(ws), ws.numel(), _stream(dev, stream))
    with torch.cuda.device(dev):
        if n_parts == 1:
            code = _abi.lib().relkl_bwd_qkv(*args, *tail)
        else:
            code = _abi.lib().relkl_bwd_qkv_part(*args, p_idx, n_parts, *tail)
    check(code, "relkl_bwd_qkv")
    if dx_dtype == torch.bfloat16:
        return [relkl_cast_bf16(dx, stream=stream) for dx in dxs]
    return dxs


def relkl_cast_bf16(src: torch.Tensor, *, out: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """bf16 copy of a float32 tensor (round to nearest, ties to even)."""
    _cuda(src, "src")
    if src.dtype != torch.float32 or not src.is_contiguous():
        raise ValueError("src must be a contiguous float32 tensor")
    if out is None:
        out = torch.empty(src.shape, dtype=torch.bfloat16, device=src.device)
    if (out.dtype != torch.bfloat16 or not out.is_contiguous() or out.device != src.device
            or out.numel() != src.numel()):
        raise ValueError("out must be a contiguous bfloat16 tensor of src's size on its device")
    with torch.cuda.device(src.device):
        code = _abi.lib().relkl_cast_bf16(_ptr(src), _ptr(out), src.numel(),
                                          _stream(src.device, stream))
    check(code, "relkl_cast_bf16")
    return out


def relkl_fwd(x_t: torch.Tensor, x_s: torch.Tensor, causal: bool = True, scale: float = 0.0, *,
              kl: Optional[torch.Tensor] = None, stats: Optional[torch.Tensor] = None,
              ws: Optional[torch.Tensor] = None, stream=None,
              lengths: Optional[torch.Tensor] = None,
              cu_seqlens: Optional[torch.Tensor] = None, max_seqlen: int = 0):
    """Per-row KL [B,H,N] and statistics [B,H,N,4] of one relation.  Pass both
    ``kl`` and ``stats`` to write into existing tensors, or neither."""
    if (kl is None) != (stats is None):
        raise ValueError("pass both kl and stats, or neither")
    out = None if kl is None else [(kl, stats)]
    return relkl_fwd_qkv([(x_t, x_s)], causal, scale, out=out, ws=ws, stream=stream,
                         lengths=lengths, cu_seqlens=cu_seqlens, max_seqlen=max_seqlen)[0]


def relkl_bwd(x_t: torch.Tensor, x_s: torch.Tensor, stats: torch.Tensor,
              dkl: Optional[torch.Tensor] = None, causal: bool = True, scale: float = 0.0, *,
              dx_s: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
              stream=None, lengths: Optional[torch.Tensor] = None,
              cu_seqlens: Optional[torch.Tensor] = None, max_seqlen: int = 0,
              dx_dtype: torch.dtype = torch.float32) -> torch.Tensor:
    """dL/dX_s (float32, or a bf16 copy with dx_dtype=torch.bfloat16) with
    L = sum_i dkl_i kl_i (dkl=None: 1/N per row, 1/L_b with lengths)."""
    return relkl_bwd_qkv([(x_t, x_s)], [stats], None if dkl is None else [dkl], causal, scale,
                         out=None if dx_s is None else [dx_s], ws=ws, stream=stream,
                         lengths=lengths, cu_seqlens=cu_seqlens, max_seqlen=max_seqlen,
                         dx_dtype=dx_dtype)[0]


def relkl_fwd_noalloc(x_t: torch.Tensor, x_s: torch.Tensor, causal: bool = True,
                      scale: float = 0.0, *, kl: Optional[torch.Tensor] = None,
                      stats: Optional[torch.Tensor] = None, stream=None,
                      lengths: Optional[torch.Tensor] = None):
    """relkl_fwd for callers that cannot provide a device workspace.

    The library call itself allocates nothing: its scratch lives in a static
    device array inside librelkl.so.  This wrapper only allocates the outputs
    when they are not passed in.  Tensor-core path only (bf16, d in {64, 128}).
    Calls that overlap on the GPU share that array and race on it.
    """
    _cuda(x_t, "x_t")
    _cuda(x_s, "x_s")
    if x_t.shape != x_s.shape or x_t.stride() != x_s.stride() or x_t.dtype != x_s.dtype:
        raise ValueError("teacher and student must share shape, strides and dtype")
    if x_s.device != x_t.device:
        raise ValueError("teacher and student must live on the same device")
    desc = make_desc(x_t, causal, scale, lengths)
    B, H, N, _ = x_t.shape
    if kl is None:
        kl = torch.empty((B, H, N), dtype=torch.float32, device=x_t.device)
    if stats is None:
        stats = torch.empty((B, H, N, 4), dtype=torch.float32, device=x_t.device)
    _check_out(kl, (B, H, N), "kl", x_t.device)
    _check_out(stats, (B, H, N, 4), "stats", x_t.device)
    with torch.cuda.device(x_t.device):
        code = _abi.lib().relkl_fwd_noalloc(ctypes.byref(desc), _ptr(x_t), _ptr(x_s), _ptr(kl),
                                            _ptr(stats), _stream(x_t.device, stream))
    check(code, "relkl_fwd_noalloc")
    return kl, stats


def relkl_get_device_error(ws: Optional[torch.Tensor] = None, stream=None) -> Tuple[int, int]:
    """Synchronise the stream and read the workspace record: (status, wait site)."""
    ws = workspace() if ws is None else ws
    where = ctypes.c_uint32(0)
    with torch.cuda.device(ws.device):
        code = _abi.lib().relkl_get_device_error(_ptr(ws), _stream(ws.device, stream),
                                                 ctypes.byref(where))
    return int(code), int(where.value)


def relkl_set_wait_timeout_ns(ns: int) -> int:
    return int(_abi.lib().relkl_set_wait_timeout_ns(int(ns)))


class RelationKL(torch.autograd.Function):
    """kl rows of one relation; backward runs relkl_bwd (teacher is frozen)."""

    @staticmethod
    def forward(ctx, x_t, x_s, causal=True, scale=0.0, lengths=None):
        kl, stats = relkl_fwd(x_t.detach(), x_s.detach(), causal, scale, lengths=lengths)
        ctx.save_for_backward(x_t, x_s, stats)
        ctx.causal, ctx.scale, ctx.lengths = causal, scale, lengths
        return kl

    @staticmethod
    def backward(ctx, dkl):
        x_t, x_s, stats = ctx.saved_tensors
        dx = relkl_bwd(x_t.detach(), x_s.detach(), stats, dkl.contiguous().float(), ctx.causal,
                       ctx.scale, lengths=ctx.lengths)
        return None, dx, None, None, None


def relation_kl(x_t: torch.Tensor, x_s: torch.Tensor, causal: bool = True,
                scale: float = 0.0, lengths: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Differentiable per-row KL(R_t || R_s) of one relation, shape [B, H, N]
    (rows past ``lengths[b]`` are padding: kl 0, no gradient)."""
    return RelationKL.apply(x_t, x_s, causal, scale, lengths)


# ------------------------------------------------ chain rule to the weights

def relkl_rope_bwd(dx_post: torch.Tensor, base: float, pos_scale: float = 1.0,
                   pos_offset: float = 0.0, apply: bool = True,
                   out_dtype: torch.dtype = torch.bfloat16, *,
                   out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """RoPE backward plus head/token transpose: [B, H, N, d] fp32 -> [B, N, H, d]."""
    _cuda(dx_post, "dx_post")
    if dx_post.dtype != torch.float32 or dx_post.dim() != 4 or not dx_post.is_contiguous():
        raise ValueError("dx_post must be a contiguous float32 [B, H, N, d] tensor")
    if out_dtype not in _DTYPES:
        raise TypeError(f"unsupported output dtype {out_dtype}")
    B, H, N, d = (int(v) for v in dx_post.shape)
    if out is None:
        out = torch.empty(B, N, H, d, dtype=out_dtype, device=dx_post.device)
    if (out.dtype != out_dtype or tuple(out.shape) != (B, N, H, d) or not out.is_contiguous()
            or out.device != dx_post.device):
        raise ValueError(f"out must be a contiguous {out_dtype} [B, N, H, d] tensor on "
                         f"{dx_post.device}")
    rope = _abi.relkl_rope(float(base), float(pos_scale), float(pos_offset), 1 if apply else 0, 0)
    with torch.cuda.device(dx_post.device):
        code = _abi.lib().relkl_rope_bwd(B, H, N, d, _ptr(dx_post), ctypes.byref(rope),
                                         _DTYPES[out_dtype], _ptr(out),
                                         _stream(dx_post.device, stream))
    check(code, "relkl_rope_bwd")
    return out


def relkl_weight_grad(h: torch.Tensor, dx_pre: torch.Tensor, *, out: Optional[torch.Tensor] = None,
                      ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """dW [D, cols] fp32 = h^T dx_pre over token rows (h [..., D], dx_pre [..., cols], bf16)."""
    _cuda(h, "h")
    _cuda(dx_pre, "dx_pre")
    if h.dtype != torch.bfloat16 or dx_pre.dtype != torch.bfloat16:
        raise TypeError("h and dx_pre must be bfloat16")
    if not h.is_contiguous() or not dx_pre.is_contiguous():
        raise ValueError("h and dx_pre must be contiguous")
    D = int(h.shape[-1])
    rows = h.numel() // D
    cols = dx_pre.numel() // rows if rows else 0
    if rows * cols != dx_pre.numel():
        raise ValueError("h and dx_pre disagree on the number of token rows")
    if dx_pre.device != h.device:
        raise ValueError("h and dx_pre must live on the same device")
    if out is None:
        out = torch.empty(D, cols, dtype=torch.float32, device=h.device)
    _check_out(out, (D, cols), "dw", h.device)
    ws = workspace(h.device) if ws is None else ws
    with torch.cuda.device(h.device):
        code = _abi.lib().relkl_weight_grad(rows, D, cols, _ptr(h), _ptr(dx_pre), _ptr(out),
                                            _ptr(ws), ws.numel(), _stream(h.device, stream))
    check(code, "relkl_weight_grad")
    return out


def student_weight_grads(pairs: Dict[str, Tuple[torch.Tensor, torch.Tensor]], h_s: torch.Tensor,
                         rope_base: float, pos_scale: float, causal: bool = True,
                         dkl: Optional[Dict[str, torch.Tensor]] = None) -> Dict[str, torch.Tensor]:
    """dW_q, dW_k, dW_v of the student: relation-KL forward and backward over the
    relations given ({rel: (x_t, x_s)}, one fused launch each), RoPE backward for q
    and k at the student's positions, and the weight gradient against h_s [B, N, D]."""
    rels = list(pairs)
    outs = relkl_fwd_qkv([pairs[r] for r in rels], causal)
    dxs = relkl_bwd_qkv([pairs[r] for r in rels], [o[1] for o in outs],
                        None if dkl is None else [dkl.get(r) for r in rels], causal)
    grads = {}
    for r, dx in zip(rels, dxs):
        pre = relkl_rope_bwd(dx, rope_base, pos_scale, 0.0, apply=(r != "v"))
        grads[r] = relkl_weight_grad(h_s, pre)
    return grads

