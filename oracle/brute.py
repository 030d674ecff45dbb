"""Brute-force float64 restatement of the block, for tiny inputs only.

TEST INFRASTRUCTURE ONLY: a second, structurally different formulation used
to pin the C oracle (``oracle.c``).  It shares no code with it:

  * RoPE is built as an explicit D x D block-diagonal rotation matrix per token
    (one 2x2 rotation block per pair) and applied as a matrix product;
  * joint attention physically concatenates [visual ; cond] Q, K, V, forms the
    whole score matrix with one matrix product, applies an additive -inf key
    mask, and normalises every row of exp(S - rowmax);
  * LayerNorm uses numpy's mean / var;
  * window attention physically gathers each window's tokens (numpy's
    array_split of the (T, H, W) grid along each axis) and runs the
    concatenated-sequence attention above on every window separately;
  * the 8-bit attention quantises with numpy float32 arithmetic and torch's
    float8_e4m3fn conversion, dequantises k block by block, and forms each
    row's whole score vector with one matrix product.

Sources: Vimoo 1.0 research page, section 2.2 (dual-stream joint attention,
QK-RMSNorm, 3D RoPE 16/56/56, adaLN, gated residual); Wan 2.1 report section
4.2.1 (raster flatten of the patched latent).
"""
from __future__ import annotations

import numpy as np


def rotation_matrix(pos_thw, D=128, split=(16, 56, 56), base=10000.0, pos_scale=(1.0, 1.0, 1.0)):
    """D x D block-diagonal rotation for a token at grid position (t, h, w)."""
    R = np.zeros((D, D))
    off = 0
    for a in range(3):
        d_a = split[a]
        p = pos_thw[a] * pos_scale[a]
        for j in range(d_a // 2):
            ang = p * base ** (-2.0 * j / d_a)
            c, s = np.cos(ang), np.sin(ang)
            i0 = off + 2 * j
            R[i0:i0 + 2, i0:i0 + 2] = [[c, -s], [s, c]]
        off += d_a
    return R


def grid_positions(grid):
    T, Hp, Wp = grid
    t, h, w = np.meshgrid(np.arange(T), np.arange(Hp), np.arange(Wp), indexing="ij")
    return np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1)   # [N, 3] raster order


def rope3d(x, grid, pos_scale=(1.0, 1.0, 1.0), base=10000.0, split=(16, 56, 56)):
    x = np.asarray(x, dtype=np.float64)
    B, N, H, D = x.shape
    out = np.empty_like(x)
    for n, pos in enumerate(grid_positions(grid)):
        R = rotation_matrix(pos, D, split, base, pos_scale)
        out[:, n] = x[:, n] @ R.T
    return out


def rmsnorm(x, g, eps=1e-6):
    x = np.asarray(x, dtype=np.float64)
    norm = np.linalg.norm(x, axis=-1, keepdims=True)
    D = x.shape[-1]
    return x * (np.sqrt(D) / np.sqrt(norm ** 2 + D * eps)) * np.asarray(g, dtype=np.float64)


def joint_attention(qv, kv, vv, qc, kc, vc, ctx_len=None, scale=None):
    qv, kv, vv, qc, kc, vc = (np.asarray(a, dtype=np.float64) for a in (qv, kv, vv, qc, kc, vc))
    B, Nv, H, D = qv.shape
    Nc = qc.shape[1]
    if scale is None:
        scale = D ** -0.5
    if ctx_len is None:
        ctx_len = [Nc] * B
    Q = np.concatenate([qv, qc], axis=1)       # [B, N, H, D]
    K = np.concatenate([kv, kc], axis=1)
    V = np.concatenate([vv, vc], axis=1)
    O = np.zeros_like(Q)
    for b in range(B):
        valid = np.concatenate([np.ones(Nv, bool), np.arange(Nc) < ctx_len[b]])
        bias = np.where(valid, 0.0, -np.inf)
        for h in range(H):
            S = Q[b, :, h] @ K[b, :, h].T * scale + bias[None, :]
            P = np.exp(S - S.max(axis=1, keepdims=True))
            P /= P.sum(axis=1, keepdims=True)
            O[b, :, h] = P @ V[b, :, h]
        O[b, Nv:][~valid[Nv:]] = 0.0
    return O[:, :Nv], O[:, Nv:]


def window_token_lists(grid, parts):
    """Raster indices of the visual tokens of each window, window-major
    (T part slowest), each list in raster order."""
    T, Hp, Wp = grid
    idx = np.arange(T * Hp * Wp).reshape(T, Hp, Wp)
    out = []
    for ts in np.array_split(np.arange(T), parts[0]):
        for hs in np.array_split(np.arange(Hp), parts[1]):
            for ws in np.array_split(np.arange(Wp), parts[2]):
                out.append(idx[np.ix_(ts, hs, ws)].ravel())
    return out


def window_attention(qv, kv, vv, qc, kc, vc, grid, parts, ctx_len=None, scale=None):
    """Each window's visual rows attend to [window visual ; cond]; cond rows
    attend to the whole joint sequence."""
    qv, kv, vv = (np.asarray(a, dtype=np.float64) for a in (qv, kv, vv))
    ov = np.zeros_like(qv)
    for toks in window_token_lists(grid, parts):
        o, _ = joint_attention(qv[:, toks], kv[:, toks], vv[:, toks], qc, kc, vc, ctx_len, scale)
        ov[:, toks] = o
    _, oc = joint_attention(qv, kv, vv, qc, kc, vc, ctx_len, scale)
    return ov, oc


def adaln_modulate(x, shift, scale, eps=1e-6):
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = x.var(axis=-1, keepdims=True)
    ln = (x - mu) / np.sqrt(var + eps)
    return ln * (1.0 + np.asarray(scale, np.float64)[:, None, :]) + np.asarray(shift, np.float64)[:, None, :]


def gated_residual(x, branch, gate):
    return np.asarray(x, np.float64) + np.asarray(gate, np.float64)[:, None, :] * np.asarray(branch, np.float64)


# ------------------------------------------------------------ 8-bit attention

def e4m3(x):
    """Nearest E4M3 value through torch's float8_e4m3fn (half-even), after
    saturating to +-448."""
    import torch
    a = np.clip(np.asarray(x, dtype=np.float64), -448.0, 448.0)
    return torch.from_numpy(a).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def quant_int8(x, block):
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    B, N, H, D = x32.shape
    codes = np.zeros(x32.shape, dtype=np.float64)
    nblk = -(-N // block)
    scales = np.zeros((B, H, nblk), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            for k in range(nblk):
                blk = x32[b, k * block:(k + 1) * block, h]
                s = np.float32(np.abs(blk).max()) / np.float32(127.0)
                scales[b, h, k] = s
                if s > 0:
                    codes[b, k * block:(k + 1) * block, h] = np.clip(np.rint(blk / s), -127, 127)
    return codes, scales


def attention_q8(qv, kv, vv, qc, kc, vc, ctx_len=None, scale=None, round_input=None):
    """The 8-bit method with numpy arrays: float32 quantisation, torch's E4M3
    conversion, and for each (row, head) the whole score vector at once (the
    concatenated valid keys), m = ceil of its maximum, P' = 2^(x - m + 6).
    round_input (optional): maps the vector P' to the values that are rounded
    to E4M3 for the P V product (the row sum keeps P')."""
    qv, kv, vv, qc, kc, vc = (np.asarray(a, dtype=np.float64) for a in (qv, kv, vv, qc, kc, vc))
    B, Nv, H, D = qv.shape
    Nc = qc.shape[1]
    if scale is None:
        scale = D ** -0.5
    if ctx_len is None:
        ctx_len = [Nc] * B
    q8v, sqv = quant_int8(qv, 1)
    q8c, sqc = quant_int8(qc, 1)
    k8v, skv = quant_int8(kv, 128)
    k8c, skc = quant_int8(kc, 128)
    out_v = np.zeros_like(qv)
    out_c = np.zeros_like(qc)
    for b in range(B):
        L = ctx_len[b]
        vals = np.concatenate([vv[b], vc[b, :L]], axis=0).astype(np.float32)     # [Nk, H, D]
        sv = np.abs(vals).max(axis=0) / np.float32(448.0)                          # [H, D]
        v8 = np.where(sv > 0, e4m3(np.where(sv > 0, vals / np.where(sv > 0, sv, 1), 0)), 0)
        # dequantised keys: codes times the scale of their 128-token block
        kd = np.concatenate([k8v[b] * np.repeat(skv[b].T, 128, axis=0)[:Nv, :, None],
                             k8c[b, :L] * np.repeat(skc[b].T, 128, axis=0)[:L, :, None]], axis=0)
        for i in range(Nv + L):
            q8 = q8v[b, i] if i < Nv else q8c[b, i - Nv]
            sq = sqv[b, :, i] if i < Nv else sqc[b, :, i - Nv]
            for h in range(H):
                x = (kd[:, h] @ q8[h]) * float(sq[h]) * scale * np.log2(np.e)
                m = np.ceil(x.max())
                p = 2.0 ** (x - m + 6)
                pr = p if round_input is None else round_input(p)
                o = (e4m3(pr) @ v8[:, h]) * sv[h] / p.sum()
                if i < Nv:
                    out_v[b, i, h] = o
                else:
                    out_c[b, i - Nv, h] = o
    return out_v, out_c
