"""Pins for the float64 oracle, independent of the oracle itself.

Each pin checks the oracle against something the pages or mathematics fix:
a brute-force restatement with explicit rotation matrices and physically
concatenated sequences (oracle/brute.py), a library routine in a special case
the definition reduces to (torch float64 scaled_dot_product_attention and
layer_norm), closed forms (tests/golden/rope_closed_form.json) and invariants
(RoPE preserves norms and is relative; softmax rows sum to one; identical keys
give mean(V); masked keys have no influence; constant-scale RMSNorm has RMS
equal to the scale; a window sees nothing outside itself), and for the
attention backward: central finite differences of sum(dO * O), torch float64
autograd, scipy's logsumexp, and the gradient sums fixed by softmax rows
summing to one; for the QK-norm + RoPE backward: finite differences through
the forward oracle and torch autograd through the brute-force rotations.  Sources: Vimoo
1.0 research page, section 2.2; Wan 2.1 report sections 4.2.1 and 4.3.1;
Seaweed-7B report, section 3.2.

``test_mutants_are_caught`` plants plausible mistakes in copies of the
oracle's C source and checks that at least one pin fails for each.
"""
import ctypes
import json
import math
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from mmdit_joint_attention_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = lambda s: np.random.Generator(np.random.PCG64(s))  # noqa: E731

PINS = {}


def pin(f):
    PINS[f.__name__] = f
    return f


def _close(a, b, tol=1e-12):
    a, b = np.asarray(a), np.asarray(b)
    assert a.shape == b.shape, (a.shape, b.shape)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert err <= tol, f"max abs err {err} > {tol}"


# --------------------------------------------------------------------- RMSNorm

@pin
def pin_rmsnorm_constant_scale_rms():
    """A constant scale g*1 gives output RMS g * sqrt(ms / (ms + eps))."""
    x = RNG(1).standard_normal((3, 7, 2, 128))
    for g, eps in ((0.7, 1e-6), (1.3, 0.0), (2.0, 0.5)):
        y = oracle.rmsnorm(x, np.full(128, g), eps)
        ms = np.mean(x * x, axis=-1)
        _close(np.sqrt(np.mean(y * y, axis=-1)), g * np.sqrt(ms / (ms + eps)))


@pin
def pin_rmsnorm_closed_form():
    """x = a*1 -> y = a / sqrt(a^2 + eps) * g, element by element."""
    g = RNG(2).uniform(0.5, 1.5, 128)
    for a in (1.0, -3.0, 0.25):
        y = oracle.rmsnorm(np.full((1, 128), a), g, 1e-6)
        _close(y[0], a / math.sqrt(a * a + 1e-6) * g)


@pin
def pin_rmsnorm_per_dim_scale_and_homogeneity():
    """With eps = 0: y(x; g) = y(x; 1) * g per dim, and y(c x) = y(x) for c > 0."""
    r = RNG(3)
    x = r.standard_normal((5, 128))
    g = r.uniform(0.5, 1.5, 128)
    y1 = oracle.rmsnorm(x, np.ones(128), 0.0)
    _close(oracle.rmsnorm(x, g, 0.0), y1 * g)
    _close(oracle.rmsnorm(3.5 * x, np.ones(128), 0.0), y1)


@pin
def pin_rmsnorm_brute():
    r = RNG(4)
    x = r.standard_normal((2, 9, 3, 128))
    g = r.uniform(0.5, 1.5, 128)
    _close(oracle.rmsnorm(x, g, 1e-6), brute.rmsnorm(x, g, 1e-6))


# ------------------------------------------------------------------------ RoPE

GRID = (4, 5, 6)


def _unit_rows(grid, D=128, H=1, seed=5):
    N = grid[0] * grid[1] * grid[2]
    return RNG(seed).standard_normal((2, N, H, D))


@pin
def pin_rope_norm_preserved():
    """A rotation keeps the norm of every head vector and of every pair."""
    x = _unit_rows(GRID, H=2)
    y = oracle.rope3d(x, GRID, pos_scale=(1.0, 0.5, 2.0))
    _close(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), 1e-11)
    xp = x.reshape(*x.shape[:-1], 64, 2)
    yp = y.reshape(*y.shape[:-1], 64, 2)
    _close(np.linalg.norm(yp, axis=-1), np.linalg.norm(xp, axis=-1), 1e-11)


@pin
def pin_rope_identity_at_origin():
    x = _unit_rows(GRID)
    y = oracle.rope3d(x, GRID)
    _close(y[:, 0], x[:, 0], 0.0)


@pin
def pin_rope_relative_position():
    """<R(p1) q, R(p2) k> depends only on p1 - p2: shifting both tokens by the
    same grid offset leaves every score unchanged."""
    T, Hp, Wp = GRID
    r = RNG(6)
    q = r.standard_normal(128)
    k = r.standard_normal(128)
    N = T * Hp * Wp
    xq = np.broadcast_to(q, (1, N, 1, 128)).copy()
    xk = np.broadcast_to(k, (1, N, 1, 128)).copy()
    rq = oracle.rope3d(xq, GRID, pos_scale=(1.0, 0.75, 1.25))[0, :, 0]
    rk = oracle.rope3d(xk, GRID, pos_scale=(1.0, 0.75, 1.25))[0, :, 0]
    idx = lambda t, h, w: (t * Hp + h) * Wp + w  # noqa: E731
    pairs = [((0, 0, 0), (1, 2, 3)), ((2, 1, 0), (0, 4, 5)), ((1, 3, 2), (1, 0, 4))]
    for p1, p2 in pairs:
        base_score = rq[idx(*p1)] @ rk[idx(*p2)]
        for d in ((1, 0, 0), (0, 1, 0), (0, 0, 1), (1, 1, 0)):
            s1 = tuple(a + b for a, b in zip(p1, d))
            s2 = tuple(a + b for a, b in zip(p2, d))
            if all(s1[i] < GRID[i] and s2[i] < GRID[i] for i in range(3)):
                assert abs(rq[idx(*s1)] @ rk[idx(*s2)] - base_score) < 1e-10


@pin
def pin_rope_axis_chunks():
    """Moving along one axis only changes that axis's chunk of dims:
    T -> [0, 16), H -> [16, 72), W -> [72, 128)."""
    T, Hp, Wp = GRID
    x = _unit_rows(GRID)
    y = oracle.rope3d(x, GRID)
    idx = lambda t, h, w: (t * Hp + h) * Wp + w  # noqa: E731
    chunks = {0: (0, 16), 1: (16, 72), 2: (72, 128)}
    for axis, pos in ((0, (2, 0, 0)), (1, (0, 3, 0)), (2, (0, 0, 4))):
        n = idx(*pos)
        lo, hi = chunks[axis]
        changed = np.any(np.abs(y[:, n, 0] - x[:, n, 0]) > 0, axis=0)
        assert changed[lo:hi].sum() >= (hi - lo) - 2
        assert not changed[:lo].any() and not changed[hi:].any()


def _eval(expr):
    return eval(expr, {"cos": math.cos, "sin": math.sin})


@pin
def pin_rope_golden_closed_form():
    with open(os.path.join(GOLDEN, "rope_closed_form.json")) as f:
        gold = json.load(f)
    grid = tuple(gold["grid"])
    T, Hp, Wp = grid
    N = T * Hp * Wp
    for block, scale in ((gold["cases"], (1.0, 1.0, 1.0)),
                         (gold["scaled"]["cases"], tuple(gold["scaled"]["pos_scale"]))):
        for c in block:
            x = np.zeros((1, N, 1, 128))
            n = (c["pos"][0] * Hp + c["pos"][1]) * Wp + c["pos"][2]
            x[0, n, 0, c["in_dim"]] = 1.0
            y = oracle.rope3d(x, grid, pos_scale=scale)[0, n, 0]
            want = [_eval(e) for e in c["expect"]]
            _close(y[c["out_dims"]], want, 1e-13)
            rest = np.delete(y, c["out_dims"])
            _close(rest, np.zeros_like(rest), 0.0)


@pin
def pin_rope_brute():
    x = _unit_rows((2, 3, 4), H=2)
    for ps in ((1.0, 1.0, 1.0), (1.0, 1 / 1.5, 1 / 1.5)):
        _close(oracle.rope3d(x, (2, 3, 4), pos_scale=ps), brute.rope3d(x, (2, 3, 4), pos_scale=ps),
               1e-12)


@pin
def pin_rope_positions_matches_grid_and_brute():
    """Explicit-position RoPE equals the grid RoPE at the grid's (scaled)
    positions, and brute-force rotation matrices at arbitrary positions."""
    g = (2, 3, 4)
    ps = (1.0, 0.5, 1.5)
    x = _unit_rows(g, H=2)
    pos = brute.grid_positions(g) * np.asarray(ps)
    _close(oracle.rope_positions(x, pos), oracle.rope3d(x, g, pos_scale=ps), 1e-12)
    rnd = RNG(31).uniform(-20, 60, size=(g[0] * g[1] * g[2], 3))
    want = np.stack([x[:, n] @ brute.rotation_matrix(rnd[n]).T for n in range(len(rnd))], axis=1)
    _close(oracle.rope_positions(x, rnd), want, 1e-11)


@pin
def pin_text_rope_shared_position():
    """MM-RoPE text tokens: position offset + n on all three axes.  Pair 0 of
    each chunk (dims 0, 16, 72) turns by exactly that position; pair d/4 of the
    H and W chunks by 0.01 of it; scores depend only on position differences."""
    N, off = 6, 7.0
    pos = oracle.text_positions(N, off)
    assert np.array_equal(pos[:, 0], pos[:, 1]) and np.array_equal(pos[:, 0], pos[:, 2])
    for d0, dd in ((0, 0), (16, 0), (72, 0), (44, 0.01), (100, 0.01)):
        x = np.zeros((1, N, 1, 128))
        x[0, :, 0, d0] = 1.0
        y = oracle.rope_positions(x, pos)[0, :, 0]
        for n in range(N):
            p = (off + n) * (dd if dd else 1.0)
            _close(y[n, d0:d0 + 2], [math.cos(p), math.sin(p)], 1e-13)
    r = RNG(32)
    q, k = r.standard_normal(128), r.standard_normal(128)
    xq = np.broadcast_to(q, (1, N, 1, 128)).copy()
    xk = np.broadcast_to(k, (1, N, 1, 128)).copy()
    rq = oracle.rope_positions(xq, pos)[0, :, 0]
    rk = oracle.rope_positions(xk, pos)[0, :, 0]
    for d in (1, 2, 3):
        s0 = rq[d] @ rk[0]
        for a in range(1, N - d):
            assert abs(rq[a + d] @ rk[a] - s0) < 1e-10


# ------------------------------------------------------------------- attention

def _qkv(B, Nv, Nc, H, seed, D=128):
    r = RNG(seed)
    return [r.standard_normal((B, n, H, D)) for n in (Nv, Nv, Nv, Nc, Nc, Nc)]


def _sdpa(Q, K, V, mask=None):
    """torch float64 SDPA on [B, N, H, D] tensors (heads moved to dim 1)."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).permute(0, 2, 1, 3)  # noqa: E731
    o = torch.nn.functional.scaled_dot_product_attention(t(Q), t(K), t(V), attn_mask=mask)
    return o.permute(0, 2, 1, 3).numpy()


@pin
def pin_attention_brute():
    for (B, Nv, Nc, H, cl) in ((1, 32, 8, 2, None), (2, 20, 9, 3, [0, 5]), (2, 17, 6, 1, [6, 1])):
        a = _qkv(B, Nv, Nc, H, seed=7 + B + Nv)
        ov, oc = oracle.joint_attention(*a, ctx_len=cl)
        bv, bc = brute.joint_attention(*a, ctx_len=cl)
        _close(ov, bv, 1e-12)
        _close(oc, bc, 1e-12)


@pin
def pin_attention_sdpa_on_concatenation():
    """With every cond token valid, joint attention is plain attention over
    the physically concatenated sequence (torch float64 SDPA, scale 1/sqrt(D))."""
    qv, kv, vv, qc, kc, vc = _qkv(2, 24, 10, 3, seed=11)
    ov, oc = oracle.joint_attention(qv, kv, vv, qc, kc, vc)
    o = _sdpa(*(np.concatenate(p, axis=1) for p in ((qv, qc), (kv, kc), (vv, vc))))
    _close(np.concatenate([ov, oc], axis=1), o, 1e-12)


@pin
def pin_attention_sdpa_key_padding():
    """Ragged cond lengths equal SDPA with a boolean key mask, per sample."""
    B, Nv, Nc, H = 2, 16, 12, 2
    a = _qkv(B, Nv, Nc, H, seed=12)
    cl = [3, 12]
    ov, oc = oracle.joint_attention(*a, ctx_len=cl)
    for b in range(B):
        Q, K, V = (np.concatenate([a[i][b:b + 1], a[i + 3][b:b + 1]], axis=1) for i in range(3))
        keep = torch.tensor(np.concatenate([np.ones(Nv, bool), np.arange(Nc) < cl[b]]))
        o = _sdpa(Q, K, V, mask=keep[None, None, None, :])
        _close(ov[b], o[0, :Nv], 1e-12)
        _close(oc[b, :cl[b]], o[0, Nv:Nv + cl[b]], 1e-12)
        _close(oc[b, cl[b]:], np.zeros_like(oc[b, cl[b]:]), 0.0)


@pin
def pin_attention_self_when_no_cond():
    """Nc = 0 reduces joint attention to self-attention over the visual stream."""
    qv, kv, vv = _qkv(1, 30, 0, 2, seed=13)[:3]
    empty = np.zeros((1, 0, 2, 128))
    ov, oc = oracle.joint_attention(qv, kv, vv, empty, empty, empty)
    _close(ov, _sdpa(qv, kv, vv), 1e-12)
    assert oc.shape == (1, 0, 2, 128)


@pin
def pin_attention_rows_sum_to_one():
    """V = 1 for every key: each valid output row is exactly the weight sum, 1."""
    qv, kv, vv, qc, kc, vc = _qkv(2, 19, 7, 2, seed=14)
    ov, oc = oracle.joint_attention(qv, kv, np.ones_like(vv), qc, kc, np.ones_like(vc),
                                    ctx_len=[7, 2])
    _close(ov, np.ones_like(ov), 1e-13)
    _close(oc[0], np.ones_like(oc[0]), 1e-13)
    _close(oc[1, :2], np.ones_like(oc[1, :2]), 1e-13)


@pin
def pin_attention_identical_keys_mean_v():
    """All keys equal -> uniform weights -> output = mean of the valid V rows."""
    B, Nv, Nc, H = 2, 13, 6, 2
    qv, kv, vv, qc, kc, vc = _qkv(B, Nv, Nc, H, seed=15)
    kvec = RNG(16).standard_normal((1, 1, H, 128))
    kv = np.broadcast_to(kvec, kv.shape).copy()
    kc = np.broadcast_to(kvec, kc.shape).copy()
    cl = [6, 4]
    ov, oc = oracle.joint_attention(qv, kv, vv, qc, kc, vc, ctx_len=cl)
    for b in range(B):
        m = np.concatenate([vv[b], vc[b, :cl[b]]], axis=0).mean(axis=0)  # [H, D]
        _close(ov[b], np.broadcast_to(m, ov[b].shape), 1e-12)
        _close(oc[b, :cl[b]], np.broadcast_to(m, oc[b, :cl[b]].shape), 1e-12)


@pin
def pin_attention_mask_no_influence():
    """Changing padded cond keys / values leaves every output bit-identical."""
    B, Nv, Nc, H = 2, 11, 9, 2
    a = _qkv(B, Nv, Nc, H, seed=17)
    cl = [4, 0]
    ov, oc = oracle.joint_attention(*a, ctx_len=cl)
    a2 = [x.copy() for x in a]
    for b in range(B):
        a2[4][b, cl[b]:] = 1e3 * RNG(18).standard_normal(a2[4][b, cl[b]:].shape)
        a2[5][b, cl[b]:] = -7.0
    ov2, oc2 = oracle.joint_attention(*a2, ctx_len=cl)
    assert np.array_equal(ov, ov2) and np.array_equal(oc, oc2)


@pin
def pin_attention_two_keys_closed_form():
    """One query, two keys: o = (e^s1 v1 + e^s2 v2) / (e^s1 + e^s2), s = q.k / sqrt(128)."""
    r = RNG(19)
    q = r.standard_normal((1, 1, 1, 128))
    k1, k2 = r.standard_normal((2, 128))
    v1, v2 = r.standard_normal((2, 128))
    kv = k1.reshape(1, 1, 1, 128)
    vv = v1.reshape(1, 1, 1, 128)
    kc = k2.reshape(1, 1, 1, 128)
    vc = v2.reshape(1, 1, 1, 128)
    ov, _ = oracle.joint_attention(q, kv, vv, q, kc, vc)
    s1 = float(q.ravel() @ k1) / math.sqrt(128)
    s2 = float(q.ravel() @ k2) / math.sqrt(128)
    want = (math.exp(s1) * v1 + math.exp(s2) * v2) / (math.exp(s1) + math.exp(s2))
    _close(ov[0, 0, 0], want, 1e-13)


@pin
def pin_attention_large_scores_stable():
    """Scores in the thousands (the softmax is shift-invariant, so the exact
    result is well defined) must come out finite and equal brute force,
    which subtracts the row maximum."""
    a = _qkv(1, 12, 5, 2, seed=25)
    a[0] = a[0] * 1000.0
    a[3] = a[3] * 1000.0
    ov, oc = oracle.joint_attention(*a)
    bv, bc = brute.joint_attention(*a)
    assert np.all(np.isfinite(ov)) and np.all(np.isfinite(oc))
    _close(ov, bv, 1e-9)
    _close(oc, bc, 1e-9)


@pin
def pin_attention_rows_subset_matches_full():
    """The row-subset entry point returns the same rows as the full call."""
    w = I.Workload("t", "f32", B=2, H=2, grid=(2, 3, 5), Nc=9, ctx_len=(9, 3))
    a = _qkv(2, w.Nv, w.Nc, 2, seed=20)
    ov, oc = oracle.joint_attention(*a, ctx_len=w.ctx_lengths())
    full = np.concatenate([ov, oc], axis=1)
    for b in range(2):
        for h in range(2):
            rows = I.parity_rows(w, b, h, n_random=8)
            trip = np.stack([np.full_like(rows, b), np.full_like(rows, h), rows], axis=1)
            got = oracle.joint_attention_rows(*a, w.ctx_lengths(), trip)
            _close(got, full[b, rows, h], 0.0)


# ------------------------------------------------------------- adaLN / residual

@pin
def pin_modulate_zero_is_layer_norm():
    """scale = shift = 0 leaves plain LayerNorm (torch float64 layer_norm)."""
    x = RNG(21).standard_normal((2, 7, 3072)) * 3.0 + 1.5
    z = np.zeros((2, 3072))
    y = oracle.adaln_modulate(x, z, z, 1e-6)
    ln = torch.nn.functional.layer_norm(torch.from_numpy(x), (3072,), eps=1e-6).numpy()
    _close(y, ln, 1e-12)
    _close(y.mean(axis=-1), np.zeros((2, 7)), 1e-12)


@pin
def pin_modulate_closed_form():
    """Row (a, -a, a, -a, ...) + m: mean m, variance a^2, so
    y = +-a / sqrt(a^2 + eps) * (1 + scale) + shift."""
    C = 3072
    a, m, eps = 2.0, 0.75, 1e-6
    x = (np.where(np.arange(C) % 2 == 0, a, -a) + m).reshape(1, 1, C)
    r = RNG(22)
    shift = r.standard_normal((1, C)) * 0.1
    scale = r.standard_normal((1, C)) * 0.1
    sign = np.where(np.arange(C) % 2 == 0, 1.0, -1.0)
    want = sign * a / math.sqrt(a * a + eps) * (1 + scale[0]) + shift[0]
    _close(oracle.adaln_modulate(x, shift, scale, eps)[0, 0], want, 1e-12)


@pin
def pin_modulate_brute():
    r = RNG(23)
    x = r.standard_normal((2, 5, 256))
    shift = r.standard_normal((2, 256)) * 0.1
    scale = r.standard_normal((2, 256)) * 0.1
    _close(oracle.adaln_modulate(x, shift, scale), brute.adaln_modulate(x, shift, scale), 1e-12)


@pin
def pin_residual_special_gates():
    r = RNG(24)
    x = r.standard_normal((2, 5, 64))
    br = r.standard_normal((2, 5, 64))
    _close(oracle.gated_residual(x, br, np.zeros((2, 64))), x, 0.0)
    _close(oracle.gated_residual(x, br, np.ones((2, 64))), x + br, 0.0)
    g = r.standard_normal((2, 64))
    _close(oracle.gated_residual(x, x, g), x * (1.0 + g[:, None, :]), 1e-14)
    g2 = np.zeros((2, 64))
    g2[1] = 1.0
    out = oracle.gated_residual(x, br, g2)
    _close(out[0], x[0], 0.0)
    _close(out[1], x[1] + br[1], 0.0)


@pin
def pin_block_brute():
    """The composed block equals the brute-force composition on the tiny workload."""
    w = I.WORKLOADS["tiny"]
    inp = I.make_inputs(w, seed=0)
    r = oracle.block(inp)
    qv, kv = brute.rmsnorm(inp["q_vis"].f64, inp["gq_vis"]), brute.rmsnorm(inp["k_vis"].f64, inp["gk_vis"])
    qv, kv = brute.rope3d(qv, w.grid), brute.rope3d(kv, w.grid)
    qc, kc = brute.rmsnorm(inp["q_ctx"].f64, inp["gq_ctx"]), brute.rmsnorm(inp["k_ctx"].f64, inp["gk_ctx"])
    ov, oc = brute.joint_attention(qv, kv, inp["v_vis"].f64, qc, kc, inp["v_ctx"].f64)
    _close(r["o_vis"], ov, 1e-12)
    _close(r["o_ctx"], oc, 1e-12)
    _close(r["x_vis"], brute.gated_residual(inp["x_vis"].f64, ov.reshape(1, w.Nv, w.C), inp["gate_vis"]), 1e-12)
    _close(r["y_ctx"], brute.adaln_modulate(inp["x_ctx"].f64, inp["shift_ctx"], inp["scale_ctx"]), 1e-12)


# ------------------------------------------------------- 3D window attention

def _window_case(seed, grid, Nc=6, B=2, H=2, ctx_len=(6, 3)):
    r = RNG(seed)
    Nv = grid[0] * grid[1] * grid[2]
    qv, kv, vv = (r.standard_normal((B, Nv, H, 128)) for _ in range(3))
    qc, kc, vc = (r.standard_normal((B, Nc, H, 128)) for _ in range(3))
    return (qv, kv, vv, qc, kc, vc), (None if ctx_len is None else np.array(ctx_len, np.int32))


@pin
def pin_window_brute():
    """Seaweed-7B section 3.2 windows against a brute force that gathers each
    window with numpy's array_split and attends over [window ; cond]."""
    grid = (5, 6, 7)
    t, cl = _window_case(40, grid)
    for parts in ((1, 2, 2), (4, 1, 1), (2, 3, 2), (5, 1, 3)):
        ov, oc = oracle.window_attention(*t, grid, parts, cl)
        bv, bc = brute.window_attention(*t, grid, parts, cl)
        _close(ov, bv, 1e-12)
        _close(oc, bc, 1e-12)


@pin
def pin_window_single_is_joint():
    """One window over the whole grid is plain joint attention."""
    grid = (3, 4, 5)
    t, cl = _window_case(41, grid)
    ov, oc = oracle.window_attention(*t, grid, (1, 1, 1), cl)
    jv, jc = brute.joint_attention(*t, cl)
    _close(ov, jv, 1e-12)
    _close(oc, jc, 1e-12)


@pin
def pin_window_singletons():
    """parts = grid extents puts every token in its own window: with no
    conditioning keys a visual row sees only itself, so its output is its V."""
    grid = (2, 3, 4)
    t, _ = _window_case(42, grid, Nc=0, ctx_len=None)
    ov, _ = oracle.window_attention(*t, grid, grid)
    _close(ov, t[2], 1e-15)


@pin
def pin_window_locality():
    """Changing K and V of the tokens outside a window leaves that window's
    visual rows unchanged but changes the conditioning rows."""
    grid = (4, 6, 6)
    parts = (2, 2, 3)
    t, cl = _window_case(43, grid)
    win = brute.window_token_lists(grid, parts)
    inside = win[5]
    outside = np.setdiff1d(np.arange(grid[0] * grid[1] * grid[2]), inside)
    qv, kv, vv, qc, kc, vc = t
    kv2, vv2 = kv.copy(), vv.copy()
    kv2[:, outside] += 3.0
    vv2[:, outside] *= -2.0
    a_v, a_c = oracle.window_attention(qv, kv, vv, qc, kc, vc, grid, parts, cl)
    b_v, b_c = oracle.window_attention(qv, kv2, vv2, qc, kc, vc, grid, parts, cl)
    _close(a_v[:, inside], b_v[:, inside], 0.0)
    assert np.max(np.abs(a_c - b_c)) > 1e-3
    assert np.max(np.abs(a_v[:, outside] - b_v[:, outside])) > 1e-3


@pin
def pin_window_sizes():
    """Window sizes of the pages' 480p latent grid (21 x 30 x 52): 1x2x2 gives
    four windows of 21*15*26 tokens; 4x1x1 splits the 21 frames 6/5/5/5."""
    win = oracle.window_of_tokens((21, 30, 52), (1, 2, 2))
    assert win.min() == 0 and win.max() == 3
    assert np.bincount(win).tolist() == [8190] * 4
    win = oracle.window_of_tokens((21, 30, 52), (4, 1, 1))
    assert win.min() == 0
    assert np.bincount(win).tolist() == [6 * 1560, 5 * 1560, 5 * 1560, 5 * 1560]
    assert win[0] == 0 and win[6 * 1560 - 1] == 0 and win[6 * 1560] == 1
    # 720p: 45 rows split 23/22, 80 columns 40/40; raster token (t, h, w) = (0, 23, 40)
    win = oracle.window_of_tokens((21, 45, 80), (1, 2, 2))
    assert win.min() == 0
    assert np.bincount(win).tolist() == [21 * 23 * 40, 21 * 23 * 40, 21 * 22 * 40, 21 * 22 * 40]
    assert win[23 * 80 + 40] == 3 and win[22 * 80 + 39] == 0


# ------------------------------------------------------------ attention backward

def _bwd_case(seed, B=2, Nv=5, Nc=3, H=2, D=8, ctx_len=(3, 1)):
    r = RNG(seed)
    t = [r.standard_normal((B, Nv, H, D)) for _ in range(3)] + \
        [r.standard_normal((B, Nc, H, D)) for _ in range(3)]
    do = (r.standard_normal((B, Nv, H, D)), r.standard_normal((B, Nc, H, D)))
    return t, do, (None if ctx_len is None else np.array(ctx_len, np.int32))


@pin
def pin_bwd_finite_differences():
    """Every gradient entry equals the central difference of L = sum(dO * O)
    computed with the forward oracle (step 1e-6)."""
    t, (dov, doc), cl = _bwd_case(50)
    g = oracle.joint_attention_bwd(*t, dov, doc, cl)

    def loss(tt):
        ov, oc = oracle.joint_attention(*tt, cl)
        return float(np.sum(ov * dov) + np.sum(oc * doc))

    names = ["dq_vis", "dk_vis", "dv_vis", "dq_ctx", "dk_ctx", "dv_ctx"]
    h = 1e-6
    for a, name in enumerate(names):
        num = np.zeros_like(t[a])
        for idx in np.ndindex(t[a].shape):
            tp = [x.copy() for x in t]
            tm = [x.copy() for x in t]
            tp[a][idx] += h
            tm[a][idx] -= h
            num[idx] = (loss(tp) - loss(tm)) / (2 * h)
        _close(g[name], num, 1e-7)


@pin
def pin_window_bwd_finite_differences():
    """Every gradient of the 3D window attention equals the central difference
    of L = sum(dO * O) through the window forward oracle (grid 2x2x3 in 1x2x2
    windows of uneven size, ragged conditioning), and the row log-sum-exp is
    scipy's logsumexp over each row's visible keys."""
    from scipy.special import logsumexp
    grid, parts = (2, 2, 3), (1, 2, 2)
    t, (dov, doc), cl = _bwd_case(53, Nv=12, Nc=3, H=2, D=8, ctx_len=(3, 1))
    g = oracle.window_attention_bwd(*t, dov, doc, grid, parts, cl)

    def loss(tt):
        ov, oc = oracle.window_attention(*tt, grid, parts, cl)
        return float(np.sum(ov * dov) + np.sum(oc * doc))

    names = ["dq_vis", "dk_vis", "dv_vis", "dq_ctx", "dk_ctx", "dv_ctx"]
    h = 1e-6
    for a, name in enumerate(names):
        num = np.zeros_like(t[a])
        for idx in np.ndindex(t[a].shape):
            tp = [x.copy() for x in t]
            tm = [x.copy() for x in t]
            tp[a][idx] += h
            tm[a][idx] -= h
            num[idx] = (loss(tp) - loss(tm)) / (2 * h)
        _close(g[name], num, 1e-7)
    win = oracle.window_of_tokens(grid, parts)
    B, Nv, H, D = t[0].shape
    for b in range(B):
        for hh in range(H):
            q = np.concatenate([t[0][b, :, hh], t[3][b, :, hh]])
            k = np.concatenate([t[1][b, :, hh], t[4][b, :cl[b], hh]])
            for i in range(Nv + 3):
                if i >= Nv + cl[b]:
                    assert np.isinf(g["lse"][b, hh, i])
                    continue
                vis_ok = (win == win[i]) if i < Nv else np.ones(Nv, bool)
                sel = np.concatenate([vis_ok, np.ones(cl[b], bool)])
                want = logsumexp(k[sel] @ q[i] / math.sqrt(D))
                assert abs(g["lse"][b, hh, i] - want) <= 1e-12


@pin
def pin_window_bwd_one_window_is_joint():
    """With one window over the whole grid the window backward is the joint
    attention backward."""
    t, (dov, doc), cl = _bwd_case(54, Nv=12, Nc=5, H=2, D=16, ctx_len=(5, 2))
    g = oracle.window_attention_bwd(*t, dov, doc, (2, 3, 2), (1, 1, 1), cl)
    j = oracle.joint_attention_bwd(*t, dov, doc, cl)
    for k in ("dq_vis", "dk_vis", "dv_vis", "dq_ctx", "dk_ctx", "dv_ctx"):
        _close(g[k], j[k], 1e-12)
    assert np.array_equal(np.isinf(g["lse"]), np.isinf(j["lse"]))


@pin
def pin_bwd_torch_autograd():
    """torch float64 autograd through scaled_dot_product_attention on the
    concatenated sequence with a boolean key mask; the padded cond query rows
    get dO = 0 (their output is a constant).  Also the row log-sum-exp
    against scipy's logsumexp of the masked scores."""
    from scipy.special import logsumexp
    t, (dov, doc), cl = _bwd_case(51, B=2, Nv=7, Nc=4, H=3, D=16, ctx_len=(4, 2))
    g = oracle.joint_attention_bwd(*t, dov, doc, cl)
    B, Nv, H, D = t[0].shape
    Nc = t[3].shape[1]
    qkv = [torch.tensor(np.concatenate([t[i], t[i + 3]], axis=1).transpose(0, 2, 1, 3),
                        requires_grad=True) for i in range(3)]
    valid = np.concatenate([np.ones((B, Nv), bool), np.arange(Nc)[None, :] < cl[:, None]], 1)
    mask = torch.from_numpy(valid)[:, None, None, :]
    out = torch.nn.functional.scaled_dot_product_attention(*qkv, attn_mask=mask)
    dO = np.concatenate([dov, doc], axis=1).transpose(0, 2, 1, 3) * valid[:, None, :, None]
    out.backward(torch.from_numpy(dO))
    for i, n in enumerate("qkv"):
        grad = qkv[i].grad.numpy().transpose(0, 2, 1, 3)
        _close(g["d%s_vis" % n], grad[:, :Nv], 1e-12)
        _close(g["d%s_ctx" % n], grad[:, Nv:], 1e-12)
    q = np.concatenate([t[0], t[3]], 1).transpose(0, 2, 1, 3)
    k = np.concatenate([t[1], t[4]], 1).transpose(0, 2, 1, 3)
    sc = q @ k.transpose(0, 1, 3, 2) / math.sqrt(D)
    sc = np.where(valid[:, None, None, :], sc, -np.inf)
    want = logsumexp(sc, axis=-1)
    want = np.where(valid[:, None, :], want, np.inf)
    _close(np.where(np.isinf(g["lse"]), 0, g["lse"]), np.where(np.isinf(want), 0, want), 1e-12)
    assert np.array_equal(np.isinf(g["lse"]), np.isinf(want))
    # the row function gives the same dq and lse as autograd and scipy
    rows = np.array([[b, h, i] for b in range(B) for h in range(H) for i in range(Nv + Nc)])
    dq, lse = oracle.joint_attention_dq_rows(*t, dov, doc, cl, rows)
    gq = qkv[0].grad.numpy()
    _close(dq, gq[rows[:, 0], rows[:, 1], rows[:, 2]], 1e-12)
    _close(np.where(np.isinf(lse), 0, lse),
           np.where(np.isinf(want), 0, want)[rows[:, 0], rows[:, 1], rows[:, 2]], 1e-12)
    # the key-row function gives autograd's dk and dv (zero on padded keys)
    dk, dv = oracle.joint_attention_dkdv_rows(*t, dov, doc, cl, rows)
    gk, gv = qkv[1].grad.numpy(), qkv[2].grad.numpy()
    _close(dk, gk[rows[:, 0], rows[:, 1], rows[:, 2]], 1e-12)
    _close(dv, gv[rows[:, 0], rows[:, 1], rows[:, 2]], 1e-12)


@pin
def pin_bwd_invariants():
    """Softmax rows sum to one, so sum_j dv_j = sum of dO over the rows with
    an output; sum_j dS_ij = 0, so sum_j dk_j = 0; identical keys make every
    dq zero."""
    t, (dov, doc), cl = _bwd_case(52, B=2, Nv=9, Nc=5, H=2, D=16, ctx_len=(5, 2))
    g = oracle.joint_attention_bwd(*t, dov, doc, cl)
    for b in range(2):
        L = cl[b]
        want = dov[b].sum(axis=0) + doc[b, :L].sum(axis=0)
        got = g["dv_vis"][b].sum(axis=0) + g["dv_ctx"][b].sum(axis=0)
        _close(got, want, 1e-12)
        _close(g["dk_vis"][b].sum(axis=0) + g["dk_ctx"][b].sum(axis=0), np.zeros((2, 16)), 1e-12)
        assert np.all(g["dk_ctx"][b, L:] == 0) and np.all(g["dv_ctx"][b, L:] == 0)
        assert np.all(g["dq_ctx"][b, L:] == 0)
    t2 = [x.copy() for x in t]
    t2[1][:] = t2[1][:, :1]
    t2[4][:] = t2[1][:, :1]
    g2 = oracle.joint_attention_bwd(*t2, dov, doc, cl)
    _close(g2["dq_vis"], np.zeros_like(g2["dq_vis"]), 1e-12)


# ------------------------------------------------- QK-RMSNorm + RoPE backward

@pin
def pin_norm_rope_bwd_finite_differences():
    """dx and dg equal central differences of L = sum(dy * y), y the forward
    oracle (RMSNorm then 3D RoPE, and RMSNorm alone for the cond stream)."""
    r = RNG(60)
    grid = (1, 2, 2)
    x = r.standard_normal((1, 4, 1, 128))
    dy = r.standard_normal((1, 4, 1, 128))
    g = r.uniform(0.5, 1.5, 128)
    for pos_grid in (grid, None):
        def loss(xx, gg):
            y = oracle.rmsnorm(xx, gg, 1e-6)
            if pos_grid is not None:
                y = oracle.rope3d(y, pos_grid, (1.0, 1.0, 1.0))
            return float(np.sum(y * dy))
        pos = oracle.grid_positions(grid) if pos_grid is not None else None
        dx, dg = oracle.rmsnorm_rope_bwd(x, g, dy, pos)
        h = 1e-6
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            num[idx] = (loss(xp, g) - loss(xm, g)) / (2 * h)
        _close(dx, num, 1e-7)
        numg = np.zeros_like(g)
        for d in range(128):
            gp, gm = g.copy(), g.copy()
            gp[d] += h
            gm[d] -= h
            numg[d] = (loss(x, gp) - loss(x, gm)) / (2 * h)
        _close(dg, numg, 1e-7)


@pin
def pin_norm_rope_bwd_torch_autograd():
    """torch float64 autograd through RMSNorm and the explicit rotation
    matrices of the brute force, at 720p-style scaled positions."""
    r = RNG(61)
    grid, ps = (2, 3, 2), (1.0, 1 / 1.5, 1 / 1.5)
    B, N, H = 2, 12, 3
    x = r.standard_normal((B, N, H, 128)) * 2.0
    dy = r.standard_normal((B, N, H, 128))
    g = r.uniform(0.5, 1.5, 128)
    R = np.stack([brute.rotation_matrix(p, pos_scale=ps) for p in brute.grid_positions(grid)])
    xt = torch.tensor(x, requires_grad=True)
    gt = torch.tensor(g, requires_grad=True)
    rms = torch.sqrt((xt * xt).mean(-1, keepdim=True) + 1e-6)
    y = torch.einsum("nde,bnhe->bnhd", torch.from_numpy(R), xt / rms * gt)
    y.backward(torch.from_numpy(dy))
    dx, dg = oracle.rmsnorm_rope_bwd(x, g, dy, oracle.grid_positions(grid, ps))
    _close(dx, xt.grad.numpy(), 1e-12)
    _close(dg, gt.grad.numpy(), 1e-11)


@pin
def pin_text_rope_bwd_torch_autograd():
    """The backward with MM-RoPE text positions (token n at offset + n on all
    three axes) equals torch float64 autograd through RMSNorm and the brute
    force's explicit rotation matrices at those positions."""
    r = RNG(62)
    B, N, H, off = 2, 9, 2, 31.0
    q = r.standard_normal((B, N, H, 128)) * 1.5
    k = r.standard_normal((B, N, H, 128))
    dq_o, dk_o = r.standard_normal((B, N, H, 128)), r.standard_normal((B, N, H, 128))
    gq, gk = r.uniform(0.5, 1.5, 128), r.uniform(0.5, 1.5, 128)
    R = torch.from_numpy(np.stack([brute.rotation_matrix((off + n, off + n, off + n))
                                   for n in range(N)]))
    got = oracle.qk_norm_rope_text_bwd(q, k, gq, gk, dq_o, dk_o, offset=off)
    for x, g, dy, dx_got, dg_got in ((q, gq, dq_o, got[0], got[2]), (k, gk, dk_o, got[1], got[3])):
        xt = torch.tensor(x, requires_grad=True)
        gt = torch.tensor(g, requires_grad=True)
        rms = torch.sqrt((xt * xt).mean(-1, keepdim=True) + 1e-6)
        y = torch.einsum("nde,bnhe->bnhd", R, xt / rms * gt)
        y.backward(torch.from_numpy(dy))
        _close(dx_got, xt.grad.numpy(), 1e-12)
        _close(dg_got, gt.grad.numpy(), 1e-11)


# ------------------------------------------------ modulate / residual backward

@pin
def pin_modulate_bwd_finite_differences():
    """dx, dshift and dscale equal central differences of L = sum(dy * y),
    y the forward modulate oracle, for every entry."""
    r = RNG(70)
    B, N, C = 2, 3, 16
    x = r.standard_normal((B, N, C)) * 1.5 + 0.3
    sh, sc = r.standard_normal((B, C)) * 0.1, r.standard_normal((B, C)) * 0.1
    dy = r.standard_normal((B, N, C))
    got = oracle.adaln_modulate_bwd(x, sc, dy)
    loss = lambda xx, hh, ss: float(np.sum(dy * oracle.adaln_modulate(xx, hh, ss)))  # noqa: E731
    h = 1e-6
    for name, arr, f in (("dx", x, lambda a: loss(a, sh, sc)),
                         ("dshift", sh, lambda a: loss(x, a, sc)),
                         ("dscale", sc, lambda a: loss(x, sh, a))):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            ap, am = arr.copy(), arr.copy()
            ap[idx] += h
            am[idx] -= h
            num[idx] = (f(ap) - f(am)) / (2 * h)
        _close(got[name], num, 1e-7)


@pin
def pin_modulate_bwd_torch_autograd():
    """torch float64 autograd through layer_norm (no affine), the (1 + scale)
    multiply and the shift."""
    r = RNG(71)
    B, N, C = 2, 5, 64
    x = r.standard_normal((B, N, C)) * 2.0
    sh, sc = r.standard_normal((B, C)) * 0.1, r.standard_normal((B, C)) * 0.1
    dy = r.standard_normal((B, N, C))
    xt, sht, sct = (torch.tensor(a, requires_grad=True) for a in (x, sh, sc))
    y = torch.nn.functional.layer_norm(xt, (C,), eps=1e-6) * (1 + sct[:, None, :]) + sht[:, None, :]
    y.backward(torch.from_numpy(dy))
    got = oracle.adaln_modulate_bwd(x, sc, dy, 1e-6)
    _close(got["dx"], xt.grad.numpy(), 1e-12)
    _close(got["dshift"], sht.grad.numpy(), 1e-12)
    _close(got["dscale"], sct.grad.numpy(), 1e-12)


@pin
def pin_modulate_bwd_invariants():
    """LayerNorm ignores adding a constant to a row and, with eps = 0,
    scaling it: so dx is orthogonal to the ones vector and to x - mean; an
    upstream gradient constant along a row (scale 0) gives dx = 0."""
    r = RNG(72)
    B, N, C = 2, 4, 32
    x = r.standard_normal((B, N, C))
    sc = r.standard_normal((B, C)) * 0.2
    dy = r.standard_normal((B, N, C))
    dx = oracle.adaln_modulate_bwd(x, sc, dy, 0.0)["dx"]
    xc = x - x.mean(-1, keepdims=True)
    assert np.max(np.abs(dx.sum(-1))) < 1e-12
    assert np.max(np.abs((dx * xc).sum(-1))) < 1e-12
    const = np.repeat(r.standard_normal((B, N, 1)), C, axis=-1)
    dx0 = oracle.adaln_modulate_bwd(x, np.zeros((B, C)), const, 1e-6)["dx"]
    assert np.max(np.abs(dx0)) < 1e-13


@pin
def pin_residual_bwd_finite_differences():
    """dx, dbranch and dgate equal central differences of L = sum(dout * out),
    out the forward gated-residual oracle."""
    r = RNG(73)
    B, N, C = 2, 3, 8
    x, br, dout = (r.standard_normal((B, N, C)) for _ in range(3))
    g = r.standard_normal((B, C)) * 0.5
    got = oracle.gated_residual_bwd(br, g, dout)
    loss = lambda xx, bb, gg: float(np.sum(dout * oracle.gated_residual(xx, bb, gg)))  # noqa: E731
    h = 1e-6
    for name, arr, f in (("dx", x, lambda a: loss(a, br, g)), ("dbranch", br, lambda a: loss(x, a, g)),
                         ("dgate", g, lambda a: loss(x, br, a))):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            ap, am = arr.copy(), arr.copy()
            ap[idx] += h
            am[idx] -= h
            num[idx] = (f(ap) - f(am)) / (2 * h)
        _close(got[name], num, 1e-8)


# ---------------------------------------------------------------- 8-bit attention

@pin
def pin_e4m3_against_torch():
    """E4M3 rounding equals torch's float8_e4m3fn conversion below the
    saturation point (including the subnormal range and halfway cases); every
    finite code decodes to torch's value and encodes back to itself; larger
    magnitudes saturate to 448."""
    r = RNG(70)
    x = np.concatenate([r.standard_normal(3000) * 60, r.standard_normal(1000) * 0.01,
                        (np.arange(-64, 64) + 0.5) * 2.0 ** -9,          # subnormal halfway
                        (8 + np.arange(8) + 0.5) * 2.0 ** -3])            # halfway at 1..2
    x = x[np.abs(x) < 448]
    want = torch.tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    _close(oracle.e4m3_round(x), want, 0.0)
    codes = np.arange(256, dtype=np.uint8)
    tv = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    fin = ~np.isnan(tv)
    _close(oracle.e4m3_decode(codes)[fin], tv[fin], 0.0)
    assert np.array_equal(oracle.e4m3_encode(tv[fin]), codes[fin])
    _close(oracle.e4m3_round([448.0, 460.0, 1e6, -500.0]), [448.0, 448.0, 448.0, -448.0], 0.0)


@pin
def pin_int8_quantisation():
    """Codes equal torch's half-even rounding of x / scale in float32 with
    scale = max|x| / 127; the largest entry of a block maps to +-127; the
    reconstruction error is at most half a step (plus the rounding of the
    float32 quotient)."""
    r = RNG(71)
    x = I.round_f64_to_bf16(r.standard_normal((2, 300, 3, 128)) * 2.0)
    for block in (1, 128):
        codes, scales = oracle.quant_int8(x, block)
        x32 = torch.from_numpy(x).float()
        for b in range(2):
            for h in range(3):
                for k in range(scales.shape[2]):
                    blk = x32[b, k * block:(k + 1) * block, h]
                    s = torch.tensor(blk.abs().max().item(), dtype=torch.float32) / 127.0
                    assert np.float32(scales[b, h, k]) == np.float32(s.item())
                    want = torch.clamp(torch.round(blk / s), -127, 127).numpy()
                    got = codes[b, k * block:(k + 1) * block, h]
                    assert np.array_equal(got, want)
                    assert np.abs(got).max() == 127
                    # half a step, plus the float32 rounding of x / scale
                    # (at most 127 * 2^-24 of a step)
                    err = np.abs(got * float(s) - blk.double().numpy()).max()
                    assert err <= float(s) * (0.5 + 127 * 2.0 ** -24)


@pin
def pin_q8_uniform_scores():
    """q = 0 makes every score 0, so every P' is exactly 2^6 and the output is
    the mean of the dequantised v over the valid keys; v built from E4M3 values
    with a channel maximum of 448 dequantises exactly, so that mean is the mean
    of v itself."""
    r = RNG(72)
    B, Nv, Nc, H, D = 2, 200, 40, 2, 128
    vals = oracle.e4m3_round(r.standard_normal((B, Nv + Nc, H, D)) * 40)
    vals[:, 0] = 448.0                        # channel maximum 448 -> scale 1
    vv, vc = vals[:, :Nv], vals[:, Nv:]
    z = np.zeros((B, Nv, H, D)), np.zeros((B, Nc, H, D))
    k = r.standard_normal((B, Nv, H, D)), r.standard_normal((B, Nc, H, D))
    cl = np.array([40, 7], np.int32)
    ov, oc = oracle.attention_q8(z[0], k[0], vv, z[1], k[1], vc, cl)
    for b in range(B):
        mean = np.concatenate([vv[b], vc[b, :cl[b]]], 0).mean(0)
        _close(ov[b], np.broadcast_to(mean, ov[b].shape), 1e-12)
        _close(oc[b, :cl[b]], np.broadcast_to(mean, oc[b, :cl[b]].shape), 1e-12)
        assert np.all(oc[b, cl[b]:] == 0)


@pin
def pin_q8_brute():
    """The 8-bit method equals a numpy restatement (float32 quantisation,
    torch E4M3 conversion, whole score vectors as matrix products) on ragged
    small inputs."""
    r = RNG(73)
    B, Nv, Nc, H, D = 2, 300, 140, 2, 128
    t = [I.round_f64_to_bf16(r.standard_normal((B, n, H, D)) * sd)
         for n, sd in ((Nv, 1.5), (Nv, 1.5), (Nv, 1.0), (Nc, 1.5), (Nc, 1.5), (Nc, 1.0))]
    cl = np.array([140, 70], np.int32)
    ov, oc = oracle.attention_q8(t[0], t[1], t[2], t[3], t[4], t[5], cl)
    bv, bc = brute.attention_q8(t[0], t[1], t[2], t[3], t[4], t[5], cl)
    _close(ov, bv, 1e-12)
    _close(oc, bc, 1e-12)


@pin
def pin_q8_rounding_ambiguity_bound():
    """The bound on choosing the other E4M3 rounding for every P' within a
    relative rel of a midpoint: zero at rel = 0; at rel = 2^-10, outputs of the
    numpy restatement whose P' are each moved by a relative amount up to rel
    before rounding (random factors, and the two extremes) stay within it of
    the oracle's, and some do move (the bound is not vacuous)."""
    r = RNG(75)
    B, Nv, Nc, H, D = 2, 300, 140, 2, 128
    t = [I.round_f64_to_bf16(r.standard_normal((B, n, H, D)) * sd)
         for n, sd in ((Nv, 1.5), (Nv, 1.5), (Nv, 1.0), (Nc, 1.5), (Nc, 1.5), (Nc, 1.0))]
    cl = np.array([140, 70], np.int32)
    _, _, z0, z1 = oracle.attention_q8(*t, cl, rel=0.0)
    assert not z0.any() and not z1.any()
    rel = 2.0 ** -10
    ov, oc, av, ac = oracle.attention_q8(*t, cl, rel=rel)
    assert av.max() > 0
    moved = 0.0
    factors = [lambda p, g=RNG(76 + k): p * (1.0 + rel * g.uniform(-1.0, 1.0, p.shape))
               for k in range(2)]
    factors += [lambda p: p * (1.0 + rel), lambda p: p * (1.0 - rel)]
    for f in factors:
        bv, bc = brute.attention_q8(*t, cl, round_input=f)
        for got, ref, bound in ((bv, ov, av), (bc, oc, ac)):
            dev = np.abs(got - ref)
            assert np.all(dev <= bound + 1e-12 * (1.0 + np.abs(ref)))
            moved = max(moved, float(dev.max()))
    assert moved > 1e-6


@pin
def pin_q8_close_to_exact():
    """The 8-bit method stays within its own rounding-error model of the exact
    attention (tests/helpers.py: every element within 6 sigma of the error
    that int8 scores and E4M3 rounding of P' and v allow, and a mean of
    |error| / sigma at most 1), on N(0,1) inputs with ragged conditioning."""
    from helpers import q8_close_to_exact, q8_exact_rows
    r = RNG(74)
    B, Nv, Nc, H, D = 2, 400, 100, 2, 128
    t = [I.round_f64_to_bf16(r.standard_normal((B, n, H, D))) for n in (Nv, Nv, Nv, Nc, Nc, Nc)]
    cl = np.array([100, 37], np.int32)
    ov, oc = oracle.attention_q8(t[0], t[1], t[2], t[3], t[4], t[5], cl)
    got = np.concatenate([ov, oc], 1)
    trip = np.array([(b, h, i) for b in range(B) for h in range(H) for i in range(Nv + Nc)])
    o, sig = q8_exact_rows(*t, cl, trip)
    q8_close_to_exact(got[trip[:, 0], trip[:, 2], trip[:, 1]], o, sig, "q8 vs exact")


@pytest.mark.parametrize("name", sorted(PINS))
def test_pin(name):
    PINS[name]()


# --------------------------------------------------------------- mutation check

MUTANTS = {
    "rope_sign": ("row[offset + 2 * j]     = u * c - v * s;", "row[offset + 2 * j]     = u * c + v * s;"),
    "rope_freq": ("double freq = pow(grid->rope_base, -2.0 * (double)j / (double)d_a);",
                  "double freq = pow(grid->rope_base, -1.0 * (double)j / (double)d_a);"),
    "rope_axis_order": ("pos[0] = n / HW;", "pos[0] = n % grid->W;"),
    "rope_pairing": ("""                    double v = row[offset + 2 * j + 1];
                    row[offset + 2 * j]     = u * c - v * s;""", """                    double v = row[offset + j + d_a / 2];
                    row[offset + 2 * j]     = u * c - v * s;"""),
    "posrope_sign": ("row[offset + 2 * j]     = u * c - v * sn;", "row[offset + 2 * j]     = u * c + v * sn;"),
    "posrope_freq": ("double ang = p * pow(rope_base, -2.0 * (double)j / (double)d_a);",
                     "double ang = p * pow(rope_base, -1.0 * (double)j / (double)d_a);"),
    "rms_missing_mean": ("sqrt(ss / (double)D + eps)", "sqrt(ss + eps)"),
    "rms_scale_reversed": ("yr[d] = xr[d] / rms * g[d];", "yr[d] = xr[d] / rms * g[D - 1 - d];"),
    "attn_no_scale": ("s[j] = acc * scale;", "s[j] = acc;"),
    "attn_mask_off_by_one": ("int nk = Nv + L;", "int nk = Nv + L + (L < Nc ? 1 : 0);"),
    "attn_padded_rows_not_zero": ("if (i - Nv >= L) continue;", "if (i - Nv >= Nc) continue;"),
    "attn_no_max_sub": ("double p = exp(s[j] - m);", "double p = exp(s[j] - 0.5 * m);"),
    "ln_unbiased_var": ("var /= (double)C;", "var /= (double)(C - 1);"),
    "ln_missing_one_plus": ("* (1.0 + scale[b * C + c])", "* (scale[b * C + c])"),
    "residual_gate_index": ("gate[b * C + c] * branch", "gate[c] * branch"),
    "window_no_remainder": ("const int size = q + (k < r ? 1 : 0);", "const int size = q;"),
    "window_remainder_last": ("const int start = k * q + (k < r ? k : r);",
                              "const int start = k * q + (k > parts - 1 - r ? k - (parts - r) : 0);"),
    "window_axis_parts": ("const int kh = oracle_part_of(h, grid->H, parts[1]);",
                          "const int kh = oracle_part_of(h, grid->H, parts[2]);"),
    "window_cond_queries_windowed": ("if (i >= Nv || win[j] == win[i]) key[nk++] = j;",
                                     "if (win[j] == win[i < Nv ? i : 0]) key[nk++] = j;"),
    "window_padded_rows_not_zero": ("if (i >= Nv + L) continue;", "if (i >= Nv + Nc) continue;"),
    "bwd_no_delta": ("const double dS = p[j] * (dP - Di);", "const double dS = p[j] * dP;"),
    "bwd_dq_no_scale": ("dq[d] += scale * dS * k[d];", "dq[d] += dS * k[d];"),
    "bwd_dv_uses_dp": ("dv[d] += p[j] * dO[d];", "dv[d] += dP * dO[d];"),
    "bwd_dk_from_k": ("dk[d] += scale * dS * q[d];", "dk[d] += scale * dS * k[d];"),
    "bwd_lse_no_max": ("if (lse) lse[bh * (long)(Nv + Nc) + i] = m + log(den);",
                       "if (lse) lse[bh * (long)(Nv + Nc) + i] = log(den);"),
    "bwd_padded_rows_counted": ("if (i >= nk || nk == 0) continue;    /* padded query row */",
                                "if (nk == 0) continue;"),
    "dqrows_no_delta": ("const double w = scale * s[j] * (g - Dsum);",
                        "const double w = scale * s[j] * g;"),
    "dkdv_no_delta": ("const double dS = p * (dP - Dr[i]);", "const double dS = p * dP;"),
    "dkdv_padded_queries_counted": (
        "const int nval = Nv + L;    /* valid keys, and the query rows with an output */",
        "const int nval = Nv + Nc;"),
    "nrbwd_rotation_not_transposed": ("u[off + 2 * j] = a0 * c + a1 * s;        /* transpose of the rotation */",
                                      "u[off + 2 * j] = a0 * c - a1 * s;"),
    "nrbwd_no_dot_term": ("dxr[d] = g[d] * u[d] / rr - xr[d] * dot / ((double)D * rr * rr * rr);",
                          "dxr[d] = g[d] * u[d] / rr;"),
    "nrbwd_r_squared": ("dxr[d] = g[d] * u[d] / rr - xr[d] * dot / ((double)D * rr * rr * rr);",
                        "dxr[d] = g[d] * u[d] / rr - xr[d] * dot / ((double)D * rr * rr);"),
    "nrbwd_dg_no_norm": ("acc[d] += u[d] * xr[d] / rr;", "acc[d] += u[d] * xr[d];"),
    "q8_no_offset": ("const double p = exp2(x[j] - m + 6.0);",
                     "const double p = exp2(x[j] - m);"),
    "q8_no_kscale": ("x[j] = (double)dot * sq * skb * scale * log2e;",
                     "x[j] = (double)dot * sq * scale * log2e;"),
    "q8_cond_kscale_block": ("[(b * H + h) * (long)(seg ? tc : tv) + jj / 128];",
                             "[(b * H + h) * (long)(seg ? tc : tv) + j / 128];"),
    "q8_int8_step": ("const float s = amax / 127.0f;", "const float s = amax / 128.0f;"),
    "q8_v_scale": ("const float s = amax / 448.0f;", "const float s = amax / 256.0f;"),
    "q8_sum_rounded": ("                l += p;\n", "                l += oracle_e4m3_round(p);\n"),
    "q8_subnormal_step": ("        quantum = ldexp(1.0, -9);                               /* subnormal range */",
                          "        quantum = ldexp(1.0, -10);"),
    "modbwd_no_mean_g": ("dx[row + c] = rstd * (g - mg - xh[c] * mgx);",
                         "dx[row + c] = rstd * (g - xh[c] * mgx);"),
    "modbwd_no_xh_term": ("dx[row + c] = rstd * (g - mg - xh[c] * mgx);",
                          "dx[row + c] = rstd * (g - mg);"),
    "modbwd_rstd_squared": ("dx[row + c] = rstd * (g - mg - xh[c] * mgx);",
                            "dx[row + c] = rstd * rstd * (g - mg - xh[c] * mgx);"),
    "modbwd_no_one_plus": ("const double g = dr[c] * (1.0 + scale[(long)b * C + c]);\n"
                           "                dx[row + c]",
                           "const double g = dr[c] * scale[(long)b * C + c];\n"
                           "                dx[row + c]"),
    "modbwd_dscale_no_xh": ("dscale[(long)b * C + c] += dr[c] * xh[c];",
                            "dscale[(long)b * C + c] += dr[c];"),
    "resbwd_dbranch_no_gate": ("dbranch[row + c] = gate[(long)b * C + c] * dout[row + c];",
                               "dbranch[row + c] = dout[row + c];"),
    "resbwd_dgate_no_branch": ("dgate[(long)b * C + c] += dout[row + c] * branch[row + c];",
                               "dgate[(long)b * C + c] += dout[row + c];"),
    "wbwd_cond_queries_windowed": ("if (i >= Nv || win[j] == win[i]) key[nkeys++] = j;",
                                   "if (win[j] == win[i < Nv ? i : 0]) key[nkeys++] = j;"),
    "wbwd_window_ignored": ("if (i >= Nv || win[j] == win[i]) key[nkeys++] = j;",
                            "key[nkeys++] = j;"),
    "window_no_cond_keys": ("for (int j = 0; j < L; ++j) key[nk++] = Nv + j;",
                            "for (int j = 0; j < L && i >= Nv; ++j) key[nk++] = Nv + j;"),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_mutants_are_caught(mutant, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    old, new = MUTANTS[mutant]
    assert src.count(old) == 1, f"mutation anchor not found: {old}"
    (tmp_path / "oracle.c").write_text(src.replace(old, new))
    hdr = os.path.join(os.path.dirname(oracle.__file__), "oracle.h")
    (tmp_path / "oracle.h").write_text(open(hdr).read())
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", str(so),
                           str(tmp_path / "oracle.c"), "-lm"])
    saved = oracle._load()
    oracle._lib = oracle._configure(ctypes.CDLL(str(so)))
    failed = []
    try:
        for name, f in PINS.items():
            try:
                f()
            except AssertionError:
                failed.append(name)
    finally:
        oracle._lib = saved
    assert failed, f"mutant {mutant} passed every pin"


def test_residual_modulate_is_the_composition():
    """The fused oracle entry is literally the two defined steps in a row."""
    r = RNG(30)
    x = r.standard_normal((2, 5, 64))
    br = r.standard_normal((2, 5, 64))
    g, sh, sc = (r.standard_normal((2, 64)) * 0.1 for _ in range(3))
    xo, y = oracle.residual_modulate(x, br, g, sh, sc)
    _close(xo, x + g[:, None, :] * br, 1e-14)
    _close(y, brute.adaln_modulate(x + g[:, None, :] * br, sh, sc), 1e-12)
