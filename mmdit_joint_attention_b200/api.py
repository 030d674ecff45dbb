"""Python entry points over the C ABI, taking torch CUDA tensors.

Each function only checks dtypes / shapes / contiguity, then passes raw device
pointers and the current CUDA stream to the matching libmmdit.so call (same
name without the ``mmdit_`` prefix).  PyTorch provides device memory and
streams; the arithmetic runs in the library's sm_100a kernels.

Layouts: q/k/v/o [B, N, H, 128]; x/branch/y [B, N, C]; shift/scale/gate
[B, C] fp32; RMSNorm scales [128] fp32; ctx_len int32 [B] on the device.
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional, Sequence, Tuple

import torch

from . import _lib
from ._lib import Grid, check

_DT = {torch.float32: _lib.MMDIT_F32, torch.bfloat16: _lib.MMDIT_BF16}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype(*ts: torch.Tensor) -> int:
    dt = ts[0].dtype
    for t in ts:
        if t.dtype != dt:
            raise TypeError(f"mixed dtypes {dt} / {t.dtype}")
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
    if dt not in _DT:
        raise TypeError(f"unsupported dtype {dt}")
    return _DT[dt]


def _f32(*ts: torch.Tensor) -> None:
    for t in ts:
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise TypeError("scales / shifts / gates must be contiguous fp32 CUDA tensors")


def make_grid(grid: Sequence[int], pos_scale=(1.0, 1.0, 1.0), rope_base: float = 10000.0,
              split=(16, 56, 56)) -> Grid:
    g = Grid()
    g.T, g.H, g.W = (int(v) for v in grid)
    for a in range(3):
        g.pos_scale[a] = float(pos_scale[a])
        g.split[a] = int(split[a])
    g.rope_base = float(rope_base)
    return g


def qk_norm_rope(q: torch.Tensor, k: torch.Tensor, q_scale: torch.Tensor, k_scale: torch.Tensor,
                 grid: Optional[Sequence[int]] = None, pos_scale=(1.0, 1.0, 1.0),
                 eps: float = 1e-6, rope_base: float = 10000.0, split=(16, 56, 56),
                 q_out: Optional[torch.Tensor] = None, k_out: Optional[torch.Tensor] = None,
                 stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-head RMSNorm of q and k, then 3D RoPE when ``grid`` = (T, H, W) is
    given (visual stream).  In place unless q_out / k_out are given."""
    dt = _dtype(q, k)
    _f32(q_scale, k_scale)
    B, N, H, D = q.shape
    if k.shape != q.shape:
        raise ValueError("q and k shapes differ")
    q_out = q if q_out is None else q_out
    k_out = k if k_out is None else k_out
    g = make_grid(grid, pos_scale, rope_base, split) if grid is not None else None
    st = _lib.lib().mmdit_qk_norm_rope(
        _ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), _ptr(q_scale), _ptr(k_scale), B, N, H, D,
        ctypes.byref(g) if g is not None else None, eps, dt, _stream(stream))
    check("mmdit_qk_norm_rope", st)
    return q_out, k_out


def qk_norm_rope_bwd(q: torch.Tensor, k: torch.Tensor, q_scale: torch.Tensor,
                     k_scale: torch.Tensor, dq_out: torch.Tensor, dk_out: torch.Tensor,
                     grid: Optional[Sequence[int]] = None, pos_scale=(1.0, 1.0, 1.0),
                     eps: float = 1e-6, rope_base: float = 10000.0, split=(16, 56, 56),
                     dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
                     stream=None):
    """Backward of qk_norm_rope: (dq, dk, dq_scale, dk_scale) for the forward
    inputs q, k and the gradients dq_out, dk_out of its outputs."""
    dt = _dtype(q, k, dq_out, dk_out)
    _f32(q_scale, k_scale)
    B, N, H, D = q.shape
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dgq = torch.empty(D, dtype=torch.float32, device=q.device)
    dgk = torch.empty(D, dtype=torch.float32, device=q.device)
    g = make_grid(grid, pos_scale, rope_base, split) if grid is not None else None
    st = _lib.lib().mmdit_qk_norm_rope_bwd(
        _ptr(q), _ptr(k), _ptr(dq_out), _ptr(dk_out), _ptr(q_scale), _ptr(k_scale), _ptr(dq),
        _ptr(dk), _ptr(dgq), _ptr(dgk), B, N, H, D, ctypes.byref(g) if g is not None else None,
        eps, dt, _stream(stream))
    check("mmdit_qk_norm_rope_bwd", st)
    return dq, dk, dgq, dgk


def qk_norm_rope_text(q: torch.Tensor, k: torch.Tensor, q_scale: torch.Tensor,
                      k_scale: torch.Tensor, pos_offset: float = 0.0, eps: float = 1e-6,
                      rope_base: float = 10000.0, split=(16, 56, 56),
                      q_out: Optional[torch.Tensor] = None, k_out: Optional[torch.Tensor] = None,
                      stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-head RMSNorm of q and k, then MM-RoPE text positions: token n at
    pos_offset + n on all three axis chunks.  In place unless outputs are given."""
    dt = _dtype(q, k)
    _f32(q_scale, k_scale)
    B, N, H, D = q.shape
    if k.shape != q.shape:
        raise ValueError("q and k shapes differ")
    q_out = q if q_out is None else q_out
    k_out = k if k_out is None else k_out
    r = _lib.TextRope()
    r.pos_offset = float(pos_offset)
    r.rope_base = float(rope_base)
    for a in range(3):
        r.split[a] = int(split[a])
    st = _lib.lib().mmdit_qk_norm_rope_text(
        _ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), _ptr(q_scale), _ptr(k_scale), B, N, H, D,
        ctypes.byref(r), eps, dt, _stream(stream))
    check("mmdit_qk_norm_rope_text", st)
    return q_out, k_out


def qk_norm_rope_text_bwd(q: torch.Tensor, k: torch.Tensor, q_scale: torch.Tensor,
                          k_scale: torch.Tensor, dq_out: torch.Tensor, dk_out: torch.Tensor,
                          pos_offset: float = 0.0, eps: float = 1e-6, rope_base: float = 10000.0,
                          split=(16, 56, 56), dq: Optional[torch.Tensor] = None,
                          dk: Optional[torch.Tensor] = None, stream=None):
    """Backward of qk_norm_rope_text: (dq, dk, dq_scale, dk_scale)."""
    dt = _dtype(q, k, dq_out, dk_out)
    _f32(q_scale, k_scale)
    B, N, H, D = q.shape
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dgq = torch.empty(D, dtype=torch.float32, device=q.device)
    dgk = torch.empty(D, dtype=torch.float32, device=q.device)
    r = _lib.TextRope()
    r.pos_offset = float(pos_offset)
    r.rope_base = float(rope_base)
    for a in range(3):
        r.split[a] = int(split[a])
    st = _lib.lib().mmdit_qk_norm_rope_text_bwd(
        _ptr(q), _ptr(k), _ptr(dq_out), _ptr(dk_out), _ptr(q_scale), _ptr(k_scale), _ptr(dq),
        _ptr(dk), _ptr(dgq), _ptr(dgk), B, N, H, D, ctypes.byref(r), eps, dt, _stream(stream))
    check("mmdit_qk_norm_rope_text_bwd", st)
    return dq, dk, dgq, dgk


def attention_workspace(device=None) -> torch.Tensor:
    """A device workspace for the split tail of joint_attention(_fwd):
    MMDIT_ATTENTION_WORKSPACE_BYTES bytes, enough for every problem."""
    return torch.empty(_lib.ATTENTION_WORKSPACE_BYTES, dtype=torch.uint8,
                       device=device if device is not None else torch.cuda.current_device())


def _attention_call(name, q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis, o_ctx, lse,
                    workspace, softmax_scale, stream):
    dt = _dtype(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx)
    B, Nv, H, D = q_vis.shape
    Nc = q_ctx.shape[1]
    if ctx_len is not None and (ctx_len.dtype != torch.int32 or not ctx_len.is_cuda):
        raise TypeError("ctx_len must be an int32 CUDA tensor")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    ptrs = [_ptr(t) for t in (q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis, o_ctx)]
    if workspace is None:
        if lse is None:
            st = _lib.lib().mmdit_joint_attention(*ptrs, B, Nv, Nc, H, D, softmax_scale, dt,
                                                  _stream(stream))
        else:
            name = "mmdit_joint_attention_fwd"
            st = _lib.lib().mmdit_joint_attention_fwd(*ptrs, _ptr(lse), B, Nv, Nc, H, D,
                                                      softmax_scale, dt, _stream(stream))
    else:
        if workspace.dtype != torch.uint8 or not workspace.is_cuda or not workspace.is_contiguous():
            raise TypeError("workspace must be a contiguous uint8 CUDA tensor")
        name = "mmdit_joint_attention_ws"
        st = _lib.lib().mmdit_joint_attention_ws(*ptrs, _ptr(lse), _ptr(workspace),
                                                 workspace.numel(), B, Nv, Nc, H, D,
                                                 softmax_scale, dt, _stream(stream))
    check(name, st)


def joint_attention(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len=None,
                    softmax_scale: Optional[float] = None, o_vis=None, o_ctx=None,
                    stream=None, workspace: Optional[torch.Tensor] = None
                    ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Non-causal attention over the concatenation [visual; cond] of both
    streams, output split back into (o_vis, o_ctx).  With a ``workspace``
    (``attention_workspace()``) the items past the last whole wave of CTAs are
    split over their keys (mmdit_joint_attention_ws)."""
    if o_vis is None:
        o_vis = torch.empty_like(q_vis)
    if o_ctx is None:
        o_ctx = torch.empty_like(q_ctx)
    _attention_call("mmdit_joint_attention", q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len,
                    o_vis, o_ctx, None, workspace, softmax_scale, stream)
    return o_vis, o_ctx


def k_norm_rope(k: torch.Tensor, k_scale: torch.Tensor, grid: Optional[Sequence[int]] = None,
                pos_scale=(1.0, 1.0, 1.0), eps: float = 1e-6, rope_base: float = 10000.0,
                split=(16, 56, 56), k_out: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """RMSNorm (+ 3D RoPE with a grid) of k alone, in place unless k_out is given;
    for joint_attention_qnorm, which normalises q itself."""
    dt = _dtype(k)
    _f32(k_scale)
    B, N, H, D = k.shape
    k_out = k if k_out is None else k_out
    g = make_grid(grid, pos_scale, rope_base, split) if grid is not None else None
    st = _lib.lib().mmdit_k_norm_rope(_ptr(k), _ptr(k_out), _ptr(k_scale), B, N, H, D,
                                      ctypes.byref(g) if g is not None else None, eps, dt,
                                      _stream(stream))
    check("mmdit_k_norm_rope", st)
    return k_out


def joint_attention_qnorm(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, q_scale_vis, q_scale_ctx,
                          grid: Optional[Sequence[int]] = None, pos_scale=(1.0, 1.0, 1.0),
                          ctx_len=None, eps: float = 1e-6, rope_base: float = 10000.0,
                          split=(16, 56, 56), softmax_scale: Optional[float] = None, o_vis=None,
                          o_ctx=None, stream=None, workspace: Optional[torch.Tensor] = None
                          ) -> Tuple[torch.Tensor, torch.Tensor]:
    """joint_attention on raw q: the kernel RMS-normalises q (and rotates the
    visual rows when ``grid`` is given) after loading it.  k must already be
    normalised (k_norm_rope).  With ``workspace`` (attention_workspace()), the
    launch's tail is split over its keys as in joint_attention."""
    dt = _dtype(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx)
    _f32(q_scale_vis, q_scale_ctx)
    B, Nv, H, D = q_vis.shape
    Nc = q_ctx.shape[1]
    o_vis = torch.empty_like(q_vis) if o_vis is None else o_vis
    o_ctx = torch.empty_like(q_ctx) if o_ctx is None else o_ctx
    if ctx_len is not None and (ctx_len.dtype != torch.int32 or not ctx_len.is_cuda):
        raise TypeError("ctx_len must be an int32 CUDA tensor")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    g = make_grid(grid, pos_scale, rope_base, split) if grid is not None else None
    args = (_ptr(q_vis), _ptr(k_vis), _ptr(v_vis), _ptr(q_ctx), _ptr(k_ctx), _ptr(v_ctx),
            _ptr(ctx_len), _ptr(o_vis), _ptr(o_ctx), _ptr(q_scale_vis), _ptr(q_scale_ctx),
            ctypes.byref(g) if g is not None else None, eps)
    tail = (B, Nv, Nc, H, D, softmax_scale, dt, _stream(stream))
    if workspace is None:
        name = "mmdit_joint_attention_qnorm"
        st = _lib.lib().mmdit_joint_attention_qnorm(*args, *tail)
    else:
        if workspace.dtype != torch.uint8 or not workspace.is_cuda or not workspace.is_contiguous():
            raise TypeError("workspace must be a contiguous uint8 CUDA tensor")
        name = "mmdit_joint_attention_qnorm_ws"
        st = _lib.lib().mmdit_joint_attention_qnorm_ws(*args, _ptr(workspace), workspace.numel(),
                                                       *tail)
    check(name, st)
    return o_vis, o_ctx


def joint_attention_fwd(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len=None,
                        softmax_scale: Optional[float] = None, o_vis=None, o_ctx=None, lse=None,
                        stream=None, workspace: Optional[torch.Tensor] = None
                        ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """joint_attention that also returns the row log-sum-exp lse [B, H, Nv + Nc]
    (fp32, natural log, +inf for rows without an output) for the backward."""
    B, Nv, H, D = q_vis.shape
    Nc = q_ctx.shape[1]
    o_vis = torch.empty_like(q_vis) if o_vis is None else o_vis
    o_ctx = torch.empty_like(q_ctx) if o_ctx is None else o_ctx
    if lse is None:
        lse = torch.empty((B, H, Nv + Nc), dtype=torch.float32, device=q_vis.device)
    _f32(lse)
    _attention_call("mmdit_joint_attention_fwd", q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx,
                    ctx_len, o_vis, o_ctx, lse, workspace, softmax_scale, stream)
    return o_vis, o_ctx, lse


def bwd_workspace_bytes(B: int, Nv: int, Nc: int, H: int) -> int:
    """Bytes of the one-pass backward's fp32 dQ accumulator [B, Nv + Nc, H, 128]."""
    return B * (Nv + Nc) * H * 128 * 4


def bwd_workspace(B: int, Nv: int, Nc: int, H: int, device=None) -> torch.Tensor:
    """A workspace with which joint_attention_bwd runs the one-pass backward."""
    return torch.empty(bwd_workspace_bytes(B, Nv, Nc, H), dtype=torch.uint8,
                       device=device if device is not None else torch.device("cuda"))


def _workspace_arg(workspace):
    if workspace is None:
        return None, 0
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise TypeError("workspace must be a contiguous CUDA tensor")
    return workspace, workspace.numel() * workspace.element_size()


def joint_attention_bwd(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, o_vis, o_ctx, do_vis, do_ctx,
                        lse, ctx_len=None, softmax_scale: Optional[float] = None, delta=None,
                        grads: Optional[dict] = None, workspace=None, stream=None) -> dict:
    """Gradients dq/dk/dv of both streams for upstream gradients do_vis, do_ctx
    of the joint attention, given its outputs and lse (joint_attention_fwd).
    ``delta`` is the fp32 [B, H, Nv + Nc] workspace (allocated here if None);
    ``grads`` may hold preallocated outputs under the returned keys.  With a
    ``workspace`` of bwd_workspace_bytes (bwd_workspace) a bf16 backward runs
    in one pass (dQ reduced in fp32, not bit-reproducible)."""
    dt = _dtype(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, o_vis, o_ctx, do_vis, do_ctx)
    B, Nv, H, D = q_vis.shape
    Nc = q_ctx.shape[1]
    if delta is None:
        delta = torch.empty((B, H, Nv + Nc), dtype=torch.float32, device=q_vis.device)
    _f32(lse, delta)
    g = dict(grads or {})
    for k, ref in (("dq_vis", q_vis), ("dk_vis", k_vis), ("dv_vis", v_vis), ("dq_ctx", q_ctx),
                   ("dk_ctx", k_ctx), ("dv_ctx", v_ctx)):
        if k not in g:
            g[k] = torch.empty_like(ref)
    if ctx_len is not None and (ctx_len.dtype != torch.int32 or not ctx_len.is_cuda):
        raise TypeError("ctx_len must be an int32 CUDA tensor")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if workspace is None:
        st = _lib.lib().mmdit_joint_attention_bwd(
            _ptr(q_vis), _ptr(k_vis), _ptr(v_vis), _ptr(q_ctx), _ptr(k_ctx), _ptr(v_ctx),
            _ptr(ctx_len), _ptr(o_vis), _ptr(o_ctx), _ptr(do_vis), _ptr(do_ctx), _ptr(lse),
            _ptr(delta), _ptr(g["dq_vis"]), _ptr(g["dk_vis"]), _ptr(g["dv_vis"]),
            _ptr(g["dq_ctx"]), _ptr(g["dk_ctx"]), _ptr(g["dv_ctx"]), B, Nv, Nc, H, D,
            softmax_scale, dt, _stream(stream))
        check("mmdit_joint_attention_bwd", st)
        return g
    ws, nbytes = _workspace_arg(workspace)
    st = _lib.lib().mmdit_joint_attention_bwd_ws(
        _ptr(q_vis), _ptr(k_vis), _ptr(v_vis), _ptr(q_ctx), _ptr(k_ctx), _ptr(v_ctx),
        _ptr(ctx_len), _ptr(o_vis), _ptr(o_ctx), _ptr(do_vis), _ptr(do_ctx), _ptr(lse),
        _ptr(delta), _ptr(ws), nbytes, _ptr(g["dq_vis"]), _ptr(g["dk_vis"]), _ptr(g["dv_vis"]),
        _ptr(g["dq_ctx"]), _ptr(g["dk_ctx"]), _ptr(g["dv_ctx"]), B, Nv, Nc, H, D, softmax_scale,
        dt, _stream(stream))
    check("mmdit_joint_attention_bwd_ws", st)
    return g


def quantize_int8(x: torch.Tensor, block: int, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Symmetric int8 codes of bf16 x [B, N, H, 128] with one scale per ``block``
    (1 or 128) tokens of a (sample, head): (codes int8, scales [B, H, blocks])."""
    if x.dtype != torch.bfloat16:
        raise TypeError("quantize_int8 takes bf16")
    _dtype(x)
    B, N, H, D = x.shape
    codes = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    scales = torch.empty((B, H, (N + block - 1) // block), dtype=torch.float32, device=x.device)
    st = _lib.lib().mmdit_quantize_int8(_ptr(x), _ptr(codes), _ptr(scales), B, N, H, D, block,
                                        _stream(stream))
    check("mmdit_quantize_int8", st)
    return codes, scales


def quantize_v_e4m3(v_vis: torch.Tensor, v_ctx: torch.Tensor, ctx_len=None, stream=None):
    """E4M3 codes (uint8) of v for both streams and the per-(sample, head,
    channel) scales [B, H, 128]."""
    _dtype(v_vis, v_ctx)
    B, Nv, H, D = v_vis.shape
    Nc = v_ctx.shape[1]
    cv = torch.empty(v_vis.shape, dtype=torch.uint8, device=v_vis.device)
    cc = torch.empty(v_ctx.shape, dtype=torch.uint8, device=v_vis.device)
    sv = torch.empty((B, H, D), dtype=torch.float32, device=v_vis.device)
    st = _lib.lib().mmdit_quantize_v_e4m3(_ptr(v_vis), _ptr(v_ctx), _ptr(ctx_len), _ptr(cv),
                                          _ptr(cc), _ptr(sv), B, Nv, Nc, H, D, _stream(stream))
    check("mmdit_quantize_v_e4m3", st)
    return cv, cc, sv


def joint_attention_q8(q8, k8, v8, scales: dict, ctx_len=None,
                       softmax_scale: Optional[float] = None, o_vis=None, o_ctx=None,
                       stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """8-bit joint attention.  q8, k8, v8: (vis, ctx) pairs of code tensors;
    scales: dict with sq_vis, sq_ctx, sk_vis, sk_ctx, sv."""
    qv, qc = q8
    kv, kc = k8
    vv, vc = v8
    B, Nv, H, D = qv.shape
    Nc = qc.shape[1]
    if o_vis is None:
        o_vis = torch.empty(qv.shape, dtype=torch.bfloat16, device=qv.device)
    if o_ctx is None:
        o_ctx = torch.empty(qc.shape, dtype=torch.bfloat16, device=qv.device)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    st = _lib.lib().mmdit_joint_attention_q8(
        _ptr(qv), _ptr(kv), _ptr(vv), _ptr(qc), _ptr(kc), _ptr(vc), _ptr(scales["sq_vis"]),
        _ptr(scales["sq_ctx"]), _ptr(scales["sk_vis"]), _ptr(scales["sk_ctx"]),
        _ptr(scales["sv"]), _ptr(ctx_len), _ptr(o_vis), _ptr(o_ctx), B, Nv, Nc, H, D,
        softmax_scale, _stream(stream))
    check("mmdit_joint_attention_q8", st)
    return o_vis, o_ctx


def joint_attention_8bit(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len=None,
                         softmax_scale: Optional[float] = None, stream=None):
    """Quantise bf16 q, k, v (q per token, k per 128-token block, v per
    channel) and run the 8-bit joint attention.  Returns (o_vis, o_ctx, parts)
    with the codes and scales in ``parts``."""
    qv8, sqv = quantize_int8(q_vis, 1, stream)
    qc8, sqc = quantize_int8(q_ctx, 1, stream)
    kv8, skv = quantize_int8(k_vis, 128, stream)
    kc8, skc = quantize_int8(k_ctx, 128, stream)
    vv8, vc8, sv = quantize_v_e4m3(v_vis, v_ctx, ctx_len, stream)
    sc = {"sq_vis": sqv, "sq_ctx": sqc, "sk_vis": skv, "sk_ctx": skc, "sv": sv}
    ov, oc = joint_attention_q8((qv8, qc8), (kv8, kc8), (vv8, vc8), sc, ctx_len, softmax_scale,
                                stream=stream)
    parts = {"q_vis": qv8, "q_ctx": qc8, "k_vis": kv8, "k_ctx": kc8, "v_vis": vv8, "v_ctx": vc8,
             **sc}
    return ov, oc, parts


def make_window(parts: Sequence[int]) -> _lib.Window:
    w = _lib.Window()
    for a in range(3):
        w.parts[a] = int(parts[a])
    return w


def qk_norm_rope_window(q: torch.Tensor, k: torch.Tensor, q_scale: torch.Tensor,
                        k_scale: torch.Tensor, grid: Sequence[int], parts: Sequence[int],
                        pos_scale=(1.0, 1.0, 1.0), eps: float = 1e-6, rope_base: float = 10000.0,
                        split=(16, 56, 56), q_out: Optional[torch.Tensor] = None,
                        k_out: Optional[torch.Tensor] = None,
                        stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """qk_norm_rope of the visual stream (raster order in) with the rows stored
    in the window-major order of the 3D window partition ``parts`` = (windows
    along T, H, W).  Outputs are new tensors unless q_out / k_out are given
    (never the inputs)."""
    dt = _dtype(q, k)
    _f32(q_scale, k_scale)
    B, N, H, D = q.shape
    if k.shape != q.shape:
        raise ValueError("q and k shapes differ")
    q_out = torch.empty_like(q) if q_out is None else q_out
    k_out = torch.empty_like(k) if k_out is None else k_out
    g = make_grid(grid, pos_scale, rope_base, split)
    w = make_window(parts)
    st = _lib.lib().mmdit_qk_norm_rope_window(
        _ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), _ptr(q_scale), _ptr(k_scale), B, N, H, D,
        ctypes.byref(g), ctypes.byref(w), eps, dt, _stream(stream))
    check("mmdit_qk_norm_rope_window", st)
    return q_out, k_out


def window_permute(x: torch.Tensor, grid: Sequence[int], parts: Sequence[int],
                   inverse: bool = False, out: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """Reorder the token rows of x [B, N, ...] (N = T*H*W) from raster to
    window-major order (inverse: back to raster)."""
    dt = _dtype(x)
    B, N = x.shape[0], x.shape[1]
    C = x.numel() // max(B * N, 1)
    y = torch.empty_like(x) if out is None else out
    g = make_grid(grid)
    w = make_window(parts)
    st = _lib.lib().mmdit_window_permute(_ptr(x), _ptr(y), B, N, C, ctypes.byref(g),
                                         ctypes.byref(w), 1 if inverse else 0, dt,
                                         _stream(stream))
    check("mmdit_window_permute", st)
    return y


def joint_window_attention(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, grid: Sequence[int],
                           parts: Sequence[int], ctx_len=None,
                           softmax_scale: Optional[float] = None, o_vis=None, o_ctx=None,
                           stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """3D window joint attention.  The visual q/k/v are in window-major order
    (as qk_norm_rope_window / window_permute write them); o_vis comes back in
    raster order.  A visual row sees its own window plus the valid
    conditioning keys; a conditioning row sees every valid key."""
    dt = _dtype(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx)
    B, Nv, H, D = q_vis.shape
    Nc = q_ctx.shape[1]
    if o_vis is None:
        o_vis = torch.empty_like(q_vis)
    if o_ctx is None:
        o_ctx = torch.empty_like(q_ctx)
    if ctx_len is not None and (ctx_len.dtype != torch.int32 or not ctx_len.is_cuda):
        raise TypeError("ctx_len must be an int32 CUDA tensor")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    g = make_grid(grid)
    w = make_window(parts)
    st = _lib.lib().mmdit_joint_window_attention(
        _ptr(q_vis), _ptr(k_vis), _ptr(v_vis), _ptr(q_ctx), _ptr(k_ctx), _ptr(v_ctx),
        _ptr(ctx_len), _ptr(o_vis), _ptr(o_ctx), B, Nv, Nc, H, D, ctypes.byref(g),
        ctypes.byref(w), softmax_scale, dt, _stream(stream))
    check("mmdit_joint_window_attention", st)
    return o_vis, o_ctx


def joint_window_attention_fwd(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, grid: Sequence[int],
                               parts: Sequence[int], ctx_len=None,
                               softmax_scale: Optional[float] = None, o_vis=None, o_ctx=None,
                               lse=None, stream=None):
    """joint_window_attention that also returns the row log-sum-exp for the
    window backward: (o_vis [raster order], o_ctx, lse [B, H, Nv + Nc] with the
    visual rows in window-major order)."""
    dt = _dtype(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx)
    B, Nv, H, D = q_vis.shape
    Nc = q_ctx.shape[1]
    o_vis = torch.empty_like(q_vis) if o_vis is None else o_vis
    o_ctx = torch.empty_like(q_ctx) if o_ctx is None else o_ctx
    if lse is None:
        lse = torch.empty((B, H, Nv + Nc), dtype=torch.float32, device=q_vis.device)
    _f32(lse)
    if ctx_len is not None and (ctx_len.dtype != torch.int32 or not ctx_len.is_cuda):
        raise TypeError("ctx_len must be an int32 CUDA tensor")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    g = make_grid(grid)
    w = make_window(parts)
    st = _lib.lib().mmdit_joint_window_attention_fwd(
        _ptr(q_vis), _ptr(k_vis), _ptr(v_vis), _ptr(q_ctx), _ptr(k_ctx), _ptr(v_ctx),
        _ptr(ctx_len), _ptr(o_vis), _ptr(o_ctx), _ptr(lse), B, Nv, Nc, H, D, ctypes.byref(g),
        ctypes.byref(w), softmax_scale, dt, _stream(stream))
    check("mmdit_joint_window_attention_fwd", st)
    return o_vis, o_ctx, lse


def joint_window_attention_bwd(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, o_vis, o_ctx, do_vis,
                               do_ctx, lse, grid: Sequence[int], parts: Sequence[int],
                               ctx_len=None, softmax_scale: Optional[float] = None, delta=None,
                               grads: Optional[dict] = None, raster_in: bool = True,
                               workspace=None, stream=None) -> dict:
    """Gradients of the 3D window joint attention.  q/k/v_vis are window-major
    (as for joint_window_attention) and lse comes from
    joint_window_attention_fwd.  With ``raster_in`` (the default) o_vis and
    do_vis are in raster order, as the forward writes o_vis, and are permuted
    to window-major here; the returned dq/dk/dv_vis are window-major, like
    q/k/v_vis.  ``workspace``: as for joint_attention_bwd."""
    dt = _dtype(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, o_vis, o_ctx, do_vis, do_ctx)
    B, Nv, H, D = q_vis.shape
    Nc = q_ctx.shape[1]
    if raster_in:
        o_vis = window_permute(o_vis, grid, parts, stream=stream)
        do_vis = window_permute(do_vis, grid, parts, stream=stream)
    if delta is None:
        delta = torch.empty((B, H, Nv + Nc), dtype=torch.float32, device=q_vis.device)
    _f32(lse, delta)
    g = dict(grads or {})
    for k, ref in (("dq_vis", q_vis), ("dk_vis", k_vis), ("dv_vis", v_vis), ("dq_ctx", q_ctx),
                   ("dk_ctx", k_ctx), ("dv_ctx", v_ctx)):
        if k not in g:
            g[k] = torch.empty_like(ref)
    if ctx_len is not None and (ctx_len.dtype != torch.int32 or not ctx_len.is_cuda):
        raise TypeError("ctx_len must be an int32 CUDA tensor")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    gr = make_grid(grid)
    w = make_window(parts)
    if workspace is None:
        st = _lib.lib().mmdit_joint_window_attention_bwd(
            _ptr(q_vis), _ptr(k_vis), _ptr(v_vis), _ptr(q_ctx), _ptr(k_ctx), _ptr(v_ctx),
            _ptr(ctx_len), _ptr(o_vis), _ptr(o_ctx), _ptr(do_vis), _ptr(do_ctx), _ptr(lse),
            _ptr(delta), _ptr(g["dq_vis"]), _ptr(g["dk_vis"]), _ptr(g["dv_vis"]),
            _ptr(g["dq_ctx"]), _ptr(g["dk_ctx"]), _ptr(g["dv_ctx"]), B, Nv, Nc, H, D,
            ctypes.byref(gr), ctypes.byref(w), softmax_scale, dt, _stream(stream))
        check("mmdit_joint_window_attention_bwd", st)
        return g
    ws, nbytes = _workspace_arg(workspace)
    st = _lib.lib().mmdit_joint_window_attention_bwd_ws(
        _ptr(q_vis), _ptr(k_vis), _ptr(v_vis), _ptr(q_ctx), _ptr(k_ctx), _ptr(v_ctx),
        _ptr(ctx_len), _ptr(o_vis), _ptr(o_ctx), _ptr(do_vis), _ptr(do_ctx), _ptr(lse),
        _ptr(delta), _ptr(ws), nbytes, _ptr(g["dq_vis"]), _ptr(g["dk_vis"]), _ptr(g["dv_vis"]),
        _ptr(g["dq_ctx"]), _ptr(g["dk_ctx"]), _ptr(g["dv_ctx"]), B, Nv, Nc, H, D,
        ctypes.byref(gr), ctypes.byref(w), softmax_scale, dt, _stream(stream))
    check("mmdit_joint_window_attention_bwd_ws", st)
    return g


def adaln_modulate(x: torch.Tensor, shift: torch.Tensor, scale: torch.Tensor,
                   eps: float = 1e-6, out: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """LN(x) * (1 + scale) + shift per sample."""
    dt = _dtype(x)
    _f32(shift, scale)
    B, N, C = x.shape
    y = torch.empty_like(x) if out is None else out
    st = _lib.lib().mmdit_adaln_modulate(_ptr(x), _ptr(shift), _ptr(scale), _ptr(y), B, N, C,
                                         eps, dt, _stream(stream))
    check("mmdit_adaln_modulate", st)
    return y


def adaln_modulate_pair(x_vis: torch.Tensor, shift_vis: torch.Tensor, scale_vis: torch.Tensor,
                        x_ctx: torch.Tensor, shift_ctx: torch.Tensor, scale_ctx: torch.Tensor,
                        eps: float = 1e-6, out_vis: Optional[torch.Tensor] = None,
                        out_ctx: Optional[torch.Tensor] = None,
                        stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """adaln_modulate of the visual and the conditioning stream in one launch,
    each with its own (shift, scale); same results as two calls."""
    dt = _dtype(x_vis, x_ctx)
    _f32(shift_vis, scale_vis, shift_ctx, scale_ctx)
    B, Nv, C = x_vis.shape
    Bc, Nc, Cc = x_ctx.shape
    if (Bc, Cc) != (B, C):
        raise ValueError("the two streams differ in batch or width")
    y_vis = torch.empty_like(x_vis) if out_vis is None else out_vis
    y_ctx = torch.empty_like(x_ctx) if out_ctx is None else out_ctx
    st = _lib.lib().mmdit_adaln_modulate_pair(
        _ptr(x_vis), _ptr(shift_vis), _ptr(scale_vis), _ptr(y_vis), Nv, _ptr(x_ctx),
        _ptr(shift_ctx), _ptr(scale_ctx), _ptr(y_ctx), Nc, B, C, eps, dt, _stream(stream))
    check("mmdit_adaln_modulate_pair", st)
    return y_vis, y_ctx


def gated_residual(x: torch.Tensor, branch: torch.Tensor, gate: torch.Tensor,
                   out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """x + gate * branch (in place into x unless ``out`` is given)."""
    dt = _dtype(x, branch)
    _f32(gate)
    B, N, C = x.shape
    out = x if out is None else out
    st = _lib.lib().mmdit_gated_residual(_ptr(x), _ptr(branch), _ptr(gate), _ptr(out), B, N, C,
                                         dt, _stream(stream))
    check("mmdit_gated_residual", st)
    return out


def adaln_modulate_bwd(x: torch.Tensor, scale: torch.Tensor, dy: torch.Tensor,
                       eps: float = 1e-6, dx: Optional[torch.Tensor] = None,
                       dshift: Optional[torch.Tensor] = None,
                       dscale: Optional[torch.Tensor] = None, stream=None
                       ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Backward of adaln_modulate: (dx, dshift, dscale) for the gradient dy of y
    (each allocated here unless given; dshift and dscale are overwritten)."""
    dt = _dtype(x, dy)
    _f32(scale)
    B, N, C = x.shape
    if dx is None:
        dx = torch.empty_like(x)
    if dshift is None:
        dshift = torch.empty((B, C), dtype=torch.float32, device=x.device)
    if dscale is None:
        dscale = torch.empty((B, C), dtype=torch.float32, device=x.device)
    _f32(dshift, dscale)
    st = _lib.lib().mmdit_adaln_modulate_bwd(_ptr(x), _ptr(scale), _ptr(dy), _ptr(dx),
                                             _ptr(dshift), _ptr(dscale), B, N, C, eps, dt,
                                             _stream(stream))
    check("mmdit_adaln_modulate_bwd", st)
    return dx, dshift, dscale


def gated_residual_bwd(branch: torch.Tensor, gate: torch.Tensor, dout: torch.Tensor,
                       dbranch: Optional[torch.Tensor] = None,
                       dgate: Optional[torch.Tensor] = None,
                       stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Backward of gated_residual: (dbranch, dgate) for the gradient dout of
    the output (each allocated here unless given; dgate is overwritten); the
    gradient of x is dout itself."""
    dt = _dtype(branch, dout)
    _f32(gate)
    B, N, C = branch.shape
    if dbranch is None:
        dbranch = torch.empty_like(branch)
    if dgate is None:
        dgate = torch.empty((B, C), dtype=torch.float32, device=branch.device)
    _f32(dgate)
    st = _lib.lib().mmdit_gated_residual_bwd(_ptr(branch), _ptr(gate), _ptr(dout), None,
                                             _ptr(dbranch), _ptr(dgate), B, N, C, dt,
                                             _stream(stream))
    check("mmdit_gated_residual_bwd", st)
    return dbranch, dgate


def residual_modulate(x: torch.Tensor, branch: torch.Tensor, gate: torch.Tensor,
                      shift: torch.Tensor, scale: torch.Tensor, eps: float = 1e-6,
                      x_out: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                      stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """x_out = x + gate * branch (in place into x unless ``x_out`` is given), then
    y = LN(x_out) * (1 + scale) + shift, in one pass over memory."""
    dt = _dtype(x, branch)
    _f32(gate, shift, scale)
    B, N, C = x.shape
    x_out = x if x_out is None else x_out
    y = torch.empty_like(x) if y is None else y
    st = _lib.lib().mmdit_residual_modulate(_ptr(x), _ptr(branch), _ptr(gate), _ptr(shift),
                                            _ptr(scale), _ptr(x_out), _ptr(y), B, N, C, eps, dt,
                                            _stream(stream))
    check("mmdit_residual_modulate", st)
    return x_out, y


def device_status(stream=None) -> int:
    """Synchronise and read-and-clear the library's device status word."""
    return _lib.lib().mmdit_device_status(_stream(stream))


def block_forward(t: dict, grid: Sequence[int], pos_scale=(1.0, 1.0, 1.0), eps: float = 1e-6,
                  stream=None, workspace: Optional[torch.Tensor] = None) -> dict:
    """One pass of the whole path on device tensors ``t`` (keys as produced by
    ``inputs.make_inputs``): adaLN modulate of both streams in one launch (y_vis, y_ctx),
    QK-RMSNorm (+ RoPE on the visual stream) in place on q/k, joint attention
    (o_vis, o_ctx), and the gated residual x += gate * o in place, with the
    attention output standing in for the branch (the projections around
    attention are not part of this path).  The attention splits its tail
    (``joint_attention``'s ``workspace``; one is allocated when none is given),
    as the host-buffer executor does.  Returns the output tensors."""
    B, Nv, H, D = t["q_vis"].shape
    if workspace is None:
        workspace = attention_workspace(t["q_vis"].device)
    Nc = t["q_ctx"].shape[1]
    out = {}
    out["y_vis"], out["y_ctx"] = adaln_modulate_pair(
        t["x_vis"], t["shift_vis"], t["scale_vis"], t["x_ctx"], t["shift_ctx"], t["scale_ctx"],
        eps, out_vis=t.get("y_vis"), out_ctx=t.get("y_ctx"), stream=stream)
    qk_norm_rope(t["q_vis"], t["k_vis"], t["gq_vis"], t["gk_vis"], grid=grid,
                 pos_scale=pos_scale, eps=eps, stream=stream)
    qk_norm_rope(t["q_ctx"], t["k_ctx"], t["gq_ctx"], t["gk_ctx"], grid=None, eps=eps,
                 stream=stream)
    out["o_vis"], out["o_ctx"] = joint_attention(
        t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"], t["v_ctx"],
        t.get("ctx_len"), o_vis=t.get("o_vis"), o_ctx=t.get("o_ctx"), stream=stream,
        workspace=workspace)
    for s, n in (("vis", Nv), ("ctx", Nc)):
        out["x_" + s] = gated_residual(t["x_" + s], out["o_" + s].view(B, n, H * D),
                                       t["gate_" + s], stream=stream)
    return out


class BlockHostExecutor:
    """``block_forward``'s path run step after step from HOST tensors, through
    mmdit_block_forward_host: the library copies each step's inputs in, runs the
    six calls and copies the outputs back, overlapping the copies of some
    steps with the kernels of others on streams of its own.

    The device workspace (``slots`` slots, one step each) is allocated here
    with torch; the RMSNorm scales are device tensors kept for the executor's
    lifetime.  A step is a dict of CPU tensors keyed like ``mmdit_block_step``
    (``_lib.BLOCK_STEP_FIELDS``); ``y_*`` and ``o_*`` may be left out (not
    copied back), ``ctx_len`` too (every cond token valid).  Pinned host memory
    lets the copies overlap the kernels."""

    def __init__(self, B: int, Nv: int, Nc: int, H: int, grid: Sequence[int],
                 gq_vis: torch.Tensor, gk_vis: torch.Tensor, gq_ctx: torch.Tensor,
                 gk_ctx: torch.Tensor, pos_scale=(1.0, 1.0, 1.0), rope_base: float = 10000.0,
                 split=(16, 56, 56), eps: float = 1e-6, softmax_scale: Optional[float] = None,
                 dtype: torch.dtype = torch.bfloat16, slots: int = 3):
        _f32(gq_vis, gk_vis, gq_ctx, gk_ctx)
        if dtype not in _DT:
            raise TypeError(f"unsupported dtype {dtype}")
        D = gq_vis.shape[0]
        self.dtype, self.B, self.N, self.C = dtype, B, {"vis": Nv, "ctx": Nc}, H * D
        c = _lib.BlockConfig()
        c.B, c.Nv, c.Nc, c.H, c.D = B, Nv, Nc, H, D
        c.grid = make_grid(grid, pos_scale, rope_base, split)
        c.gq_vis, c.gk_vis = gq_vis.data_ptr(), gk_vis.data_ptr()
        c.gq_ctx, c.gk_ctx = gq_ctx.data_ptr(), gk_ctx.data_ptr()
        c.norm_eps = c.ln_eps = eps
        c.softmax_scale = 1.0 / math.sqrt(D) if softmax_scale is None else softmax_scale
        c.dt = _DT[dtype]
        self.cfg = c
        self._scales = (gq_vis, gk_vis, gq_ctx, gk_ctx)
        nbytes = _lib.lib().mmdit_block_slot_bytes(ctypes.byref(c))
        if nbytes < 0:
            raise _lib.MmditError("mmdit_block_slot_bytes", int(nbytes))
        self.slot_bytes = int(nbytes)
        self.workspace = torch.empty(slots * self.slot_bytes, dtype=torch.uint8,
                                     device=gq_vis.device)

    def _host(self, name: str, t: torch.Tensor) -> int:
        s = name.rsplit("_", 1)[1]
        if name == "ctx_len":
            want, dt = self.B, torch.int32
        elif name.split("_")[0] in ("shift", "scale", "gate"):
            want, dt = self.B * self.C, torch.float32
        else:
            want, dt = self.B * self.N[s] * self.C, self.dtype
        if t.is_cuda or not t.is_contiguous() or t.dtype != dt or t.numel() != want:
            raise ValueError(f"step[{name!r}] must be a contiguous CPU {dt} tensor of "
                             f"{want} elements")
        return t.data_ptr()

    def run(self, steps: Sequence[dict], stream=None) -> None:
        """Enqueues every step on ``stream`` (default: the current stream);
        synchronise it before reading the outputs."""
        arr = (_lib.BlockStep * max(1, len(steps)))()
        for i, st in enumerate(steps):
            unknown = set(st) - set(_lib.BLOCK_STEP_FIELDS)
            if unknown:
                raise KeyError(f"unknown step fields {sorted(unknown)}")
            for name, t in st.items():
                if t is not None:
                    setattr(arr[i], name, self._host(name, t))
        status = _lib.lib().mmdit_block_forward_host(
            ctypes.byref(self.cfg), arr, len(steps), ctypes.c_void_p(self.workspace.data_ptr()),
            self.workspace.numel(), _stream(stream))
        check("mmdit_block_forward_host", status)
