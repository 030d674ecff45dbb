"""Float64 CPU oracle for one MMDiT block's joint-attention core.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke``
and by the CPU-baseline leg of ``bench.py``.  Nothing in the product package
imports it, and it imports nothing from the product package.

The arithmetic lives in ``oracle.c`` (plain C loops in double precision); this
module only marshals NumPy float64 arrays.  Which page and section each step
follows is stated beside each function in ``oracle.c``:
Vimoo 1.0 research page, section 2.2 (QK-RMSNorm, 3D RoPE 16/56/56 on the
visual stream, joint attention over the concatenated streams with the output
split back, adaLN modulate, gated residual); the Wan 2.1 report, sections
4.2.1 (raster flatten of the patched latent) and 4.3.1 (non-causal attention);
the Seaweed-7B report, section 3.2 (MM-RoPE text positions, 3D window
attention).

Parity status: every function is pinned by tests in tests/test_oracle_pins.py
(brute force with explicit rotation matrices and physically concatenated
sequences, library routines for the special cases that reduce to them,
closed forms and invariants).
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional, Tuple

import numpy as np

from . import build as _build

_lib = None


class _Grid(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("pos_scale", ctypes.c_double * 3), ("rope_base", ctypes.c_double),
                ("split", ctypes.c_int * 3)]


def _configure(lib):
    """Declare the C signatures on a loaded oracle library."""
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_rmsnorm.argtypes = [dp, dp, dp, ctypes.c_long, ctypes.c_int, ctypes.c_double]
    lib.oracle_rope3d.argtypes = [dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                  ctypes.POINTER(_Grid)]
    lib.oracle_rope_positions.argtypes = [dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, dp, ctypes.c_double,
                                          ctypes.POINTER(ctypes.c_int)]
    lib.oracle_joint_attention_rows.argtypes = (
        [dp] * 6 + [ctypes.POINTER(ctypes.c_int)] + [ctypes.c_int] * 5 +
        [ctypes.c_double, ctypes.POINTER(ctypes.c_long), ctypes.c_long, dp])
    lib.oracle_window_of_tokens.argtypes = [ctypes.POINTER(_Grid), ctypes.POINTER(ctypes.c_int),
                                            ctypes.POINTER(ctypes.c_int)]
    lib.oracle_window_attention_rows.argtypes = (
        [dp] * 6 + [ctypes.POINTER(ctypes.c_int)] + [ctypes.c_int] * 5 +
        [ctypes.POINTER(_Grid), ctypes.POINTER(ctypes.c_int)] +
        [ctypes.c_double, ctypes.POINTER(ctypes.c_long), ctypes.c_long, dp])
    lib.oracle_joint_attention_bwd.argtypes = (
        [dp] * 6 + [ctypes.POINTER(ctypes.c_int)] + [dp] * 2 + [ctypes.c_int] * 5 +
        [ctypes.c_double] + [dp] * 7)
    lib.oracle_window_attention_bwd.argtypes = (
        [dp] * 6 + [ctypes.POINTER(ctypes.c_int)] + [dp] * 2 + [ctypes.c_int] * 5 +
        [ctypes.POINTER(_Grid), ctypes.POINTER(ctypes.c_int), ctypes.c_double] + [dp] * 7)
    lib.oracle_joint_attention_dq_rows.argtypes = (
        [dp] * 6 + [ctypes.POINTER(ctypes.c_int)] + [dp] * 2 + [ctypes.c_int] * 5 +
        [ctypes.c_double, ctypes.POINTER(ctypes.c_long), ctypes.c_long, dp, dp])
    lib.oracle_joint_attention_dkdv_rows.argtypes = (
        [dp] * 6 + [ctypes.POINTER(ctypes.c_int)] + [dp] * 2 + [ctypes.c_int] * 5 +
        [ctypes.c_double, ctypes.POINTER(ctypes.c_long), ctypes.c_long, dp, dp])
    lib.oracle_rmsnorm_rope_bwd.argtypes = [dp, dp, dp, dp, ctypes.c_double,
                                            ctypes.POINTER(ctypes.c_int), ctypes.c_long,
                                            ctypes.c_int, ctypes.c_double, dp, dp]
    lib.oracle_e4m3_round.argtypes = [ctypes.c_double]
    lib.oracle_e4m3_round.restype = ctypes.c_double
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
    lib.oracle_e4m3_encode.restype = ctypes.c_ubyte
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_ubyte]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    i8p = ctypes.POINTER(ctypes.c_byte)
    u8p = ctypes.POINTER(ctypes.c_ubyte)
    fp = ctypes.POINTER(ctypes.c_float)
    lib.oracle_quant_int8.argtypes = [dp] + [ctypes.c_int] * 5 + [i8p, fp]
    lib.oracle_quant_v_e4m3.argtypes = [dp, dp, ctypes.POINTER(ctypes.c_int)] + \
        [ctypes.c_int] * 5 + [u8p, u8p, fp]
    lib.oracle_attention_q8_rows.argtypes = [i8p, i8p, fp, fp, i8p, i8p, fp, fp, u8p, u8p, fp,
                                             ctypes.POINTER(ctypes.c_int)] + [ctypes.c_int] * 5 + \
        [ctypes.c_double, ctypes.POINTER(ctypes.c_long), ctypes.c_long, dp, ctypes.c_double, dp]
    lib.oracle_adaln_modulate.argtypes = [dp, dp, dp, dp] + [ctypes.c_int] * 3 + [ctypes.c_double]
    lib.oracle_gated_residual.argtypes = [dp, dp, dp, dp] + [ctypes.c_int] * 3
    lib.oracle_adaln_modulate_bwd.argtypes = [dp, dp, dp] + [ctypes.c_int] * 3 + [
        ctypes.c_double, dp, dp, dp]
    lib.oracle_gated_residual_bwd.argtypes = [dp, dp, dp] + [ctypes.c_int] * 3 + [dp, dp, dp]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _configure(ctypes.CDLL(_build.build()))
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def rmsnorm(x, g, eps: float = 1e-6) -> np.ndarray:
    """RMS-normalise the last axis of ``x`` (length D) and scale by ``g`` [D]."""
    x = _f64(x)
    g = _f64(g)
    y = np.empty_like(x)
    D = x.shape[-1]
    _load().oracle_rmsnorm(_p(x), _p(y), _p(g), x.size // D, D, eps)
    return y


def rope3d(x, grid: Tuple[int, int, int], pos_scale=(1.0, 1.0, 1.0), base: float = 10000.0,
           split=(16, 56, 56)) -> np.ndarray:
    """Rotate visual rows x [B, N, H, D] by their (t, h, w) grid position."""
    x = _f64(x).copy()
    B, N, H, D = x.shape
    if N != grid[0] * grid[1] * grid[2] or sum(split) != D:
        raise ValueError("grid / split do not match x")
    gr = _Grid(grid[0], grid[1], grid[2], (ctypes.c_double * 3)(*pos_scale), base,
               (ctypes.c_int * 3)(*split))
    _load().oracle_rope3d(_p(x), B, N, H, D, ctypes.byref(gr))
    return x


def rope_positions(x, pos, base: float = 10000.0, split=(16, 56, 56)) -> np.ndarray:
    """Rotate rows x [B, N, H, D] by explicit per-axis positions pos [N, 3]."""
    x = _f64(x).copy()
    B, N, H, D = x.shape
    pos = _f64(pos).reshape(N, 3)
    if sum(split) != D:
        raise ValueError("split does not match D")
    sp = (ctypes.c_int * 3)(*split)
    _load().oracle_rope_positions(_p(x), B, N, H, D, _p(pos), base, sp)
    return x


def text_positions(N: int, offset: float = 0.0) -> np.ndarray:
    """MM-RoPE positions of N text tokens: token n at (offset + n) on all three axes."""
    p = offset + np.arange(N, dtype=np.float64)
    return np.stack([p, p, p], axis=1)


def qk_norm_rope_text(q, k, gq, gk, offset: float = 0.0, eps: float = 1e-6,
                      base: float = 10000.0, split=(16, 56, 56)):
    """QK-RMSNorm, then MM-RoPE with shared 1D text positions (Seaweed-7B report,
    section 3.2) for the conditioning stream."""
    qn = rmsnorm(q, gq, eps)
    kn = rmsnorm(k, gk, eps)
    pos = text_positions(np.shape(q)[1], offset)
    return rope_positions(qn, pos, base, split), rope_positions(kn, pos, base, split)


def qk_norm_rope(q, k, gq, gk, grid=None, pos_scale=(1.0, 1.0, 1.0), eps: float = 1e-6,
                 base: float = 10000.0, split=(16, 56, 56)):
    """QK-RMSNorm of q and k [B, N, H, D] with their own scales, then (when a
    grid is given, i.e. for the visual stream) 3D RoPE."""
    qn = rmsnorm(q, gq, eps)
    kn = rmsnorm(k, gk, eps)
    if grid is not None:
        qn = rope3d(qn, grid, pos_scale, base, split)
        kn = rope3d(kn, grid, pos_scale, base, split)
    return qn, kn


def joint_attention_rows(qv, kv, vv, qc, kc, vc, ctx_len, rows, scale: Optional[float] = None):
    """Attention output for selected query rows.  ``rows`` is an int array of
    (b, h, i) triplets with i the joint index (< Nv visual, else cond)."""
    qv, kv, vv, qc, kc, vc = (_f64(a) for a in (qv, kv, vv, qc, kc, vc))
    B, Nv, H, D = qv.shape
    Nc = qc.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    out = np.zeros((rows.shape[0], D), dtype=np.float64)
    if ctx_len is None:
        cl_p = ctypes.POINTER(ctypes.c_int)()
    else:
        cl = np.ascontiguousarray(ctx_len, dtype=np.int32)
        cl_p = cl.ctypes.data_as(ctypes.POINTER(ctypes.c_int))
    if rows.shape[0]:
        _load().oracle_joint_attention_rows(
            _p(qv), _p(kv), _p(vv), _p(qc), _p(kc), _p(vc), cl_p, B, Nv, Nc, H, D, scale,
            rows.ctypes.data_as(ctypes.POINTER(ctypes.c_long)), rows.shape[0], _p(out))
    return out


def joint_attention(qv, kv, vv, qc, kc, vc, ctx_len=None, scale: Optional[float] = None):
    """Full joint attention; returns (o_vis [B,Nv,H,D], o_ctx [B,Nc,H,D])."""
    B, Nv, H, D = np.shape(qv)
    Nc = np.shape(qc)[1]
    bb, hh, ii = np.meshgrid(np.arange(B), np.arange(H), np.arange(Nv + Nc), indexing="ij")
    rows = np.stack([bb.ravel(), hh.ravel(), ii.ravel()], axis=1)
    out = joint_attention_rows(qv, kv, vv, qc, kc, vc, ctx_len, rows, scale)
    out = out.reshape(B, H, Nv + Nc, D).transpose(0, 2, 1, 3)
    return np.ascontiguousarray(out[:, :Nv]), np.ascontiguousarray(out[:, Nv:])


def _ctx_ptr(ctx_len):
    if ctx_len is None:
        return ctypes.POINTER(ctypes.c_int)(), None
    cl = np.ascontiguousarray(ctx_len, dtype=np.int32)
    return cl.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), cl


def joint_attention_bwd(qv, kv, vv, qc, kc, vc, dov, doc, ctx_len=None,
                        scale: Optional[float] = None) -> dict:
    """Gradients of the joint attention for upstream gradients (dov, doc) on
    (o_vis, o_ctx): returns dq_vis, dk_vis, dv_vis, dq_ctx, dk_ctx, dv_ctx
    (shapes of the inputs) and lse [B, H, Nv + Nc] (natural log of the softmax
    denominator including the max; +inf for rows without an output)."""
    qv, kv, vv, qc, kc, vc, dov, doc = (_f64(a) for a in (qv, kv, vv, qc, kc, vc, dov, doc))
    B, Nv, H, D = qv.shape
    Nc = qc.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = {k: np.empty_like(qv) for k in ("dq_vis", "dk_vis", "dv_vis")}
    out.update({k: np.empty_like(qc) for k in ("dq_ctx", "dk_ctx", "dv_ctx")})
    out["lse"] = np.empty((B, H, Nv + Nc), dtype=np.float64)
    cl_p, _keep = _ctx_ptr(ctx_len)
    _load().oracle_joint_attention_bwd(
        _p(qv), _p(kv), _p(vv), _p(qc), _p(kc), _p(vc), cl_p, _p(dov), _p(doc), B, Nv, Nc, H, D,
        scale, _p(out["dq_vis"]), _p(out["dk_vis"]), _p(out["dv_vis"]), _p(out["dq_ctx"]),
        _p(out["dk_ctx"]), _p(out["dv_ctx"]), _p(out["lse"]))
    return out


def joint_attention_dq_rows(qv, kv, vv, qc, kc, vc, dov, doc, ctx_len, rows,
                            scale: Optional[float] = None):
    """(dq [nrows, D], lse [nrows]) of selected (b, h, joint row) triplets."""
    qv, kv, vv, qc, kc, vc, dov, doc = (_f64(a) for a in (qv, kv, vv, qc, kc, vc, dov, doc))
    B, Nv, H, D = qv.shape
    Nc = qc.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    dq = np.zeros((rows.shape[0], D), dtype=np.float64)
    lse = np.zeros(rows.shape[0], dtype=np.float64)
    cl_p, _keep = _ctx_ptr(ctx_len)
    if rows.shape[0]:
        _load().oracle_joint_attention_dq_rows(
            _p(qv), _p(kv), _p(vv), _p(qc), _p(kc), _p(vc), cl_p, _p(dov), _p(doc), B, Nv, Nc,
            H, D, scale, rows.ctypes.data_as(ctypes.POINTER(ctypes.c_long)), rows.shape[0],
            _p(dq), _p(lse))
    return dq, lse


def joint_attention_dkdv_rows(qv, kv, vv, qc, kc, vc, dov, doc, ctx_len, keys,
                              scale: Optional[float] = None):
    """(dk [nkeys, D], dv [nkeys, D]) of selected (b, h, joint key index)
    triplets; padded keys give zeros."""
    qv, kv, vv, qc, kc, vc, dov, doc = (_f64(a) for a in (qv, kv, vv, qc, kc, vc, dov, doc))
    B, Nv, H, D = qv.shape
    Nc = qc.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    keys = np.ascontiguousarray(keys, dtype=np.int64).reshape(-1, 3)
    dk = np.zeros((keys.shape[0], D), dtype=np.float64)
    dv = np.zeros((keys.shape[0], D), dtype=np.float64)
    cl_p, _keep = _ctx_ptr(ctx_len)
    if keys.shape[0]:
        _load().oracle_joint_attention_dkdv_rows(
            _p(qv), _p(kv), _p(vv), _p(qc), _p(kc), _p(vc), cl_p, _p(dov), _p(doc), B, Nv, Nc,
            H, D, scale, keys.ctypes.data_as(ctypes.POINTER(ctypes.c_long)), keys.shape[0],
            _p(dk), _p(dv))
    return dk, dv


def grid_positions(grid, pos_scale=(1.0, 1.0, 1.0)) -> np.ndarray:
    """Scaled (t, h, w) RoPE positions [T*H*W, 3] of the visual tokens in raster
    order (token n at t = n / (H W), h = (n / W) % H, w = n % W)."""
    T, Hg, Wg = grid
    n = np.arange(T * Hg * Wg)
    p = np.stack([n // (Hg * Wg), (n // Wg) % Hg, n % Wg], axis=1).astype(np.float64)
    return p * np.asarray(pos_scale, dtype=np.float64)


def rmsnorm_rope_bwd(x, g, dy, pos=None, eps: float = 1e-6, base: float = 10000.0,
                     split=(16, 56, 56)):
    """Backward of y = RoPE(pos)(rmsnorm(x) * g) for x, dy [B, N, H, D] and
    positions pos [N, 3] (None: no rotation).  Returns (dx, dg [D])."""
    x = _f64(x)
    dy = _f64(dy)
    g = _f64(g)
    B, N, H, D = x.shape
    dx = np.empty_like(x)
    dg = np.zeros(D, dtype=np.float64)
    if pos is not None:
        # one (t, h, w) triple per (b, n, h) row
        pr = np.ascontiguousarray(np.broadcast_to(_f64(pos).reshape(1, N, 1, 3), (B, N, H, 3)))
        pp = _p(pr)
    else:
        pr = None
        pp = ctypes.POINTER(ctypes.c_double)()
    sp = (ctypes.c_int * 3)(*split)
    _load().oracle_rmsnorm_rope_bwd(_p(x), _p(g), _p(dy), pp, base, sp, B * N * H, D, eps,
                                    _p(dx), _p(dg))
    return dx, dg


def qk_norm_rope_bwd(q, k, gq, gk, dq_out, dk_out, grid=None, pos_scale=(1.0, 1.0, 1.0),
                     eps: float = 1e-6, base: float = 10000.0, split=(16, 56, 56)):
    """Backward of qk_norm_rope: returns dq, dk (inputs' shapes), dgq, dgk [D]."""
    pos = grid_positions(grid, pos_scale) if grid is not None else None
    dq, dgq = rmsnorm_rope_bwd(q, gq, dq_out, pos, eps, base, split)
    dk, dgk = rmsnorm_rope_bwd(k, gk, dk_out, pos, eps, base, split)
    return dq, dk, dgq, dgk


def qk_norm_rope_text_bwd(q, k, gq, gk, dq_out, dk_out, offset: float = 0.0,
                          eps: float = 1e-6, base: float = 10000.0, split=(16, 56, 56)):
    """Backward of qk_norm_rope_text (MM-RoPE text positions): dq, dk, dgq, dgk."""
    pos = text_positions(np.shape(q)[1], offset)
    dq, dgq = rmsnorm_rope_bwd(q, gq, dq_out, pos, eps, base, split)
    dk, dgk = rmsnorm_rope_bwd(k, gk, dk_out, pos, eps, base, split)
    return dq, dk, dgq, dgk


# ------------------------------------------------------------ 8-bit attention

def e4m3_round(x) -> np.ndarray:
    """Round to the nearest E4M3 value (half-even, saturating at +-448)."""
    f = _load().oracle_e4m3_round
    a = np.asarray(x, dtype=np.float64)
    return np.array([f(float(v)) for v in a.ravel()]).reshape(a.shape)


def e4m3_encode(x) -> np.ndarray:
    f = _load().oracle_e4m3_encode
    a = np.asarray(x, dtype=np.float64)
    return np.array([f(float(v)) for v in a.ravel()], dtype=np.uint8).reshape(a.shape)


def e4m3_decode(c) -> np.ndarray:
    f = _load().oracle_e4m3_decode
    a = np.asarray(c, dtype=np.uint8)
    return np.array([f(int(v)) for v in a.ravel()]).reshape(a.shape)


def quant_int8(x, block: int):
    """Symmetric int8 codes of x [B, N, H, D] with one fp32 scale per block of
    ``block`` consecutive tokens of a (sample, head): (codes, scales [B, H, nblk])."""
    x = _f64(x)
    B, N, H, D = x.shape
    nblk = (N + block - 1) // block
    codes = np.zeros(x.shape, dtype=np.int8)
    scales = np.zeros((B, H, max(nblk, 0)), dtype=np.float32)
    if x.size:
        _load().oracle_quant_int8(_p(x), B, N, H, D, block,
                                  codes.ctypes.data_as(ctypes.POINTER(ctypes.c_byte)),
                                  scales.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    return codes, scales


def quant_v_e4m3(vv, vc, ctx_len=None):
    """E4M3 codes of v (both streams) with one fp32 scale per (sample, head,
    channel) over the valid tokens: (codes_vis, codes_ctx, scales [B, H, D])."""
    vv, vc = _f64(vv), _f64(vc)
    B, Nv, H, D = vv.shape
    Nc = vc.shape[1]
    cv = np.zeros(vv.shape, dtype=np.uint8)
    cc = np.zeros(vc.shape, dtype=np.uint8)
    sv = np.zeros((B, H, D), dtype=np.float32)
    cl_p, _keep = _ctx_ptr(ctx_len)
    u8 = ctypes.POINTER(ctypes.c_ubyte)
    _load().oracle_quant_v_e4m3(_p(vv), _p(vc), cl_p, B, Nv, Nc, H, D, cv.ctypes.data_as(u8),
                                cc.ctypes.data_as(u8),
                                sv.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    return cv, cc, sv


def attention_q8_rows(qv8, qc8, sqv, sqc, kv8, kc8, skv, skc, vv8, vc8, sv, ctx_len, rows,
                      scale: Optional[float] = None, rel: Optional[float] = None):
    """Output rows (b, h, joint i) of the 8-bit joint attention (Wan 2.1
    report, section 4.4.3) from quantised operands (see oracle.c).  With
    ``rel``, also the bound on how far rounding the P' that lie within a
    relative ``rel`` of an E4M3 midpoint the other way can move each output
    element: returns (out, amb)."""
    arrs = [np.ascontiguousarray(a) for a in (qv8, qc8, kv8, kc8)]
    qv8, qc8, kv8, kc8 = (a.astype(np.int8, copy=False) for a in arrs)
    vv8 = np.ascontiguousarray(vv8, dtype=np.uint8)
    vc8 = np.ascontiguousarray(vc8, dtype=np.uint8)
    sqv, sqc, skv, skc, sv = (np.ascontiguousarray(a, dtype=np.float32)
                              for a in (sqv, sqc, skv, skc, sv))
    B, Nv, H, D = qv8.shape
    Nc = qc8.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    out = np.zeros((rows.shape[0], D), dtype=np.float64)
    amb = np.zeros_like(out) if rel is not None else None
    cl_p, _keep = _ctx_ptr(ctx_len)
    i8 = ctypes.POINTER(ctypes.c_byte)
    u8 = ctypes.POINTER(ctypes.c_ubyte)
    f = ctypes.POINTER(ctypes.c_float)
    if rows.shape[0]:
        _load().oracle_attention_q8_rows(
            qv8.ctypes.data_as(i8), qc8.ctypes.data_as(i8), sqv.ctypes.data_as(f),
            sqc.ctypes.data_as(f), kv8.ctypes.data_as(i8), kc8.ctypes.data_as(i8),
            skv.ctypes.data_as(f), skc.ctypes.data_as(f), vv8.ctypes.data_as(u8),
            vc8.ctypes.data_as(u8), sv.ctypes.data_as(f), cl_p, B, Nv, Nc, H, D, scale,
            rows.ctypes.data_as(ctypes.POINTER(ctypes.c_long)), rows.shape[0], _p(out),
            float(rel or 0.0), _p(amb) if amb is not None else None)
    return out if rel is None else (out, amb)


def attention_q8(qv, kv, vv, qc, kc, vc, ctx_len=None, rows=None, scale=None, rel=None):
    """The whole 8-bit method from unquantised q, k, v: quantise (q per token,
    k per 128-token block, v per channel), then attend.  Returns (o_vis, o_ctx)
    when ``rows`` is None, else the requested rows; with ``rel``, each output
    comes with its rounding-ambiguity bound (attention_q8_rows):
    (o_vis, o_ctx, amb_vis, amb_ctx), or (rows, amb)."""
    qv8, sqv = quant_int8(qv, 1)
    qc8, sqc = quant_int8(qc, 1)
    kv8, skv = quant_int8(kv, 128)
    kc8, skc = quant_int8(kc, 128)
    vv8, vc8, sv = quant_v_e4m3(vv, vc, ctx_len)
    B, Nv, H, D = np.shape(qv)
    Nc = np.shape(qc)[1]
    full = rows is None
    if full:
        bb, hh, ii = np.meshgrid(np.arange(B), np.arange(H), np.arange(Nv + Nc), indexing="ij")
        rows = np.stack([bb.ravel(), hh.ravel(), ii.ravel()], axis=1)
    res = attention_q8_rows(qv8, qc8, sqv.reshape(B, H, -1), sqc.reshape(B, H, -1), kv8, kc8,
                            skv, skc, vv8, vc8, sv, ctx_len, rows, scale, rel)
    if not full:
        return res
    parts = []
    for a in (res if rel is not None else (res,)):
        a = a.reshape(B, H, Nv + Nc, D).transpose(0, 2, 1, 3)
        parts += [np.ascontiguousarray(a[:, :Nv]), np.ascontiguousarray(a[:, Nv:])]
    return tuple(parts)


def _grid_struct(grid) -> _Grid:
    return _Grid(grid[0], grid[1], grid[2], (ctypes.c_double * 3)(1.0, 1.0, 1.0), 10000.0,
                 (ctypes.c_int * 3)(16, 56, 56))


def window_of_tokens(grid: Tuple[int, int, int], parts: Tuple[int, int, int]) -> np.ndarray:
    """Window index of every visual token (raster order) when the (T, H, W) grid
    is split into parts[a] windows along axis a (Seaweed-7B report, section 3.2;
    the first extent % parts windows of an axis are one position longer)."""
    if any(p < 1 or p > e for p, e in zip(parts, grid)):
        raise ValueError("each axis needs 1 <= parts <= extent")
    win = np.empty(grid[0] * grid[1] * grid[2], dtype=np.int32)
    pa = (ctypes.c_int * 3)(*parts)
    gr = _grid_struct(grid)
    _load().oracle_window_of_tokens(ctypes.byref(gr), pa,
                                    win.ctypes.data_as(ctypes.POINTER(ctypes.c_int)))
    return win


def window_attention_rows(qv, kv, vv, qc, kc, vc, ctx_len, grid, parts, rows,
                          scale: Optional[float] = None):
    """3D window joint attention for selected query rows (inputs and joint
    indices in raster order): a visual query sees the visual keys of its own
    window and every valid conditioning key; a conditioning query sees every
    valid key."""
    qv, kv, vv, qc, kc, vc = (_f64(a) for a in (qv, kv, vv, qc, kc, vc))
    B, Nv, H, D = qv.shape
    Nc = qc.shape[1]
    if Nv != grid[0] * grid[1] * grid[2]:
        raise ValueError("grid does not match Nv")
    if any(p < 1 or p > e for p, e in zip(parts, grid)):
        raise ValueError("each axis needs 1 <= parts <= extent")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    out = np.zeros((rows.shape[0], D), dtype=np.float64)
    if ctx_len is None:
        cl_p = ctypes.POINTER(ctypes.c_int)()
    else:
        cl = np.ascontiguousarray(ctx_len, dtype=np.int32)
        cl_p = cl.ctypes.data_as(ctypes.POINTER(ctypes.c_int))
    gr = _grid_struct(grid)
    pa = (ctypes.c_int * 3)(*parts)
    if rows.shape[0]:
        _load().oracle_window_attention_rows(
            _p(qv), _p(kv), _p(vv), _p(qc), _p(kc), _p(vc), cl_p, B, Nv, Nc, H, D,
            ctypes.byref(gr), pa, scale, rows.ctypes.data_as(ctypes.POINTER(ctypes.c_long)),
            rows.shape[0], _p(out))
    return out


def window_attention(qv, kv, vv, qc, kc, vc, grid, parts, ctx_len=None,
                     scale: Optional[float] = None):
    """Full 3D window joint attention; returns (o_vis, o_ctx) in raster order."""
    B, Nv, H, D = np.shape(qv)
    Nc = np.shape(qc)[1]
    bb, hh, ii = np.meshgrid(np.arange(B), np.arange(H), np.arange(Nv + Nc), indexing="ij")
    rows = np.stack([bb.ravel(), hh.ravel(), ii.ravel()], axis=1)
    out = window_attention_rows(qv, kv, vv, qc, kc, vc, ctx_len, grid, parts, rows, scale)
    out = out.reshape(B, H, Nv + Nc, D).transpose(0, 2, 1, 3)
    return np.ascontiguousarray(out[:, :Nv]), np.ascontiguousarray(out[:, Nv:])


def window_attention_bwd(qv, kv, vv, qc, kc, vc, dov, doc, grid, parts, ctx_len=None,
                         scale: Optional[float] = None) -> dict:
    """Gradients of the 3D window joint attention (raster order in and out):
    dq/dk/dv of both streams and lse [B, H, Nv + Nc] (+inf for rows without
    an output)."""
    qv, kv, vv, qc, kc, vc, dov, doc = (_f64(a) for a in (qv, kv, vv, qc, kc, vc, dov, doc))
    B, Nv, H, D = qv.shape
    Nc = qc.shape[1]
    if Nv != grid[0] * grid[1] * grid[2]:
        raise ValueError("grid does not match Nv")
    if any(p < 1 or p > e for p, e in zip(parts, grid)):
        raise ValueError("each axis needs 1 <= parts <= extent")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = {k: np.empty_like(qv) for k in ("dq_vis", "dk_vis", "dv_vis")}
    out.update({k: np.empty_like(qc) for k in ("dq_ctx", "dk_ctx", "dv_ctx")})
    out["lse"] = np.empty((B, H, Nv + Nc), dtype=np.float64)
    cl_p, _keep = _ctx_ptr(ctx_len)
    gr = _grid_struct(grid)
    pa = (ctypes.c_int * 3)(*parts)
    _load().oracle_window_attention_bwd(
        _p(qv), _p(kv), _p(vv), _p(qc), _p(kc), _p(vc), cl_p, _p(dov), _p(doc), B, Nv, Nc, H, D,
        ctypes.byref(gr), pa, scale, _p(out["dq_vis"]), _p(out["dk_vis"]), _p(out["dv_vis"]),
        _p(out["dq_ctx"]), _p(out["dk_ctx"]), _p(out["dv_ctx"]), _p(out["lse"]))
    return out


def adaln_modulate(x, shift, scale, eps: float = 1e-6) -> np.ndarray:
    """LN(x) * (1 + scale) + shift for x [B, N, C], shift/scale [B, C]."""
    x = _f64(x)
    shift = _f64(shift)
    scale = _f64(scale)
    B, N, C = x.shape
    y = np.empty_like(x)
    _load().oracle_adaln_modulate(_p(x), _p(shift), _p(scale), _p(y), B, N, C, eps)
    return y


def gated_residual(x, branch, gate) -> np.ndarray:
    """x + gate * branch for x, branch [B, N, C], gate [B, C]."""
    x = _f64(x)
    branch = _f64(branch)
    gate = _f64(gate)
    B, N, C = x.shape
    out = np.empty_like(x)
    _load().oracle_gated_residual(_p(x), _p(branch), _p(gate), _p(out), B, N, C)
    return out


def adaln_modulate_bwd(x, scale, dy, eps: float = 1e-6) -> dict:
    """Backward of adaln_modulate for the upstream gradient dy [B, N, C]:
    dx [B, N, C], dshift and dscale [B, C] (the shift does not enter any of
    them)."""
    x, scale, dy = _f64(x), _f64(scale), _f64(dy)
    B, N, C = x.shape
    out = {"dx": np.empty_like(x), "dshift": np.empty((B, C)), "dscale": np.empty((B, C))}
    _load().oracle_adaln_modulate_bwd(_p(x), _p(scale), _p(dy), B, N, C, eps, _p(out["dx"]),
                                      _p(out["dshift"]), _p(out["dscale"]))
    return out


def gated_residual_bwd(branch, gate, dout) -> dict:
    """Backward of gated_residual for the upstream gradient dout [B, N, C]:
    dx, dbranch [B, N, C] and dgate [B, C]."""
    branch, gate, dout = _f64(branch), _f64(gate), _f64(dout)
    B, N, C = branch.shape
    out = {"dx": np.empty_like(branch), "dbranch": np.empty_like(branch),
           "dgate": np.empty((B, C))}
    _load().oracle_gated_residual_bwd(_p(branch), _p(gate), _p(dout), B, N, C, _p(out["dx"]),
                                      _p(out["dbranch"]), _p(out["dgate"]))
    return out


def residual_modulate(x, branch, gate, shift, scale, eps: float = 1e-6, round_to=None):
    """Gated residual, then the adaLN modulate of the next branch on its result.
    ``round_to`` (a function) rounds x' to the storage type before the
    LayerNorm, as a pipeline that stores x' and reads it back does."""
    xo = gated_residual(x, branch, gate)
    xs = round_to(xo) if round_to is not None else xo
    return xo, adaln_modulate(xs, shift, scale, eps)


def block(inp: dict, eps: float = 1e-6):
    """One pass of the whole path on the arrays of ``mmdit_joint_attention_b200.inputs
    .make_inputs``: modulate both streams, QK-norm (+RoPE on the visual stream),
    joint attention, and the gated residual with the attention output as the
    branch (the projections around attention are outside this path).

    Returns a dict with y_vis, y_ctx, q_vis, k_vis, q_ctx, k_ctx (normalised),
    o_vis, o_ctx, x_vis, x_ctx (after the residual)."""
    w = inp["workload"]
    B, Nv, Nc, H, D = w.B, w.Nv, w.Nc, w.H, w.D
    r = {}
    for s in ("vis", "ctx"):
        r["y_" + s] = adaln_modulate(inp["x_" + s].f64, inp["shift_" + s], inp["scale_" + s], eps)
    r["q_vis"], r["k_vis"] = qk_norm_rope(inp["q_vis"].f64, inp["k_vis"].f64, inp["gq_vis"],
                                          inp["gk_vis"], grid=w.grid, pos_scale=w.pos_scale,
                                          eps=eps)
    r["q_ctx"], r["k_ctx"] = qk_norm_rope(inp["q_ctx"].f64, inp["k_ctx"].f64, inp["gq_ctx"],
                                          inp["gk_ctx"], grid=None, eps=eps)
    r["o_vis"], r["o_ctx"] = joint_attention(r["q_vis"], r["k_vis"], inp["v_vis"].f64,
                                             r["q_ctx"], r["k_ctx"], inp["v_ctx"].f64,
                                             inp["ctx_len"])
    r["x_vis"] = gated_residual(inp["x_vis"].f64, r["o_vis"].reshape(B, Nv, H * D), inp["gate_vis"])
    r["x_ctx"] = gated_residual(inp["x_ctx"].f64, r["o_ctx"].reshape(B, Nc, H * D), inp["gate_ctx"])
    return r
