"""GPU parity of 3D window attention (Seaweed-7B report, section 3.2) through
the C ABI: the row permutation, the permuting QK-norm + RoPE prologue, the
windowed joint attention and its backward, against the float64 oracle on
raster-order inputs.

Small grids compare every output element; the 480p grid compares sampled
query rows (every cond row, the first and last tokens and the tile
boundaries of every window, 512 random rows per (sample, head))."""
import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from mmdit_joint_attention_b200 import api
from mmdit_joint_attention_b200 import inputs as I
from helpers import device_inputs, from_dev, parity, to_dev

pytestmark = pytest.mark.gpu

W = I.WORKLOADS


def _ws(w: I.Workload, **kw) -> I.Workload:
    import dataclasses
    return dataclasses.replace(w, **kw)


def _order(grid, parts):
    """Raster index of the token at each window-major position."""
    return np.concatenate(brute.window_token_lists(grid, parts))


# ------------------------------------------------------------------ permutation

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("grid,parts", [((5, 8, 8), (1, 2, 2)), ((5, 8, 8), (4, 1, 1)),
                                        ((5, 6, 7), (2, 3, 2)), ((3, 4, 5), (3, 4, 5))])
def test_window_permute_is_the_permutation(dtype, grid, parts):
    B, N, C = 2, grid[0] * grid[1] * grid[2], 96
    x = torch.randn(B, N, C, device="cuda").to(dtype)
    y = api.window_permute(x, grid, parts)
    order = torch.from_numpy(_order(grid, parts)).cuda()
    assert torch.equal(y, x[:, order])
    back = api.window_permute(y, grid, parts, inverse=True)
    assert torch.equal(back, x)


# --------------------------------------------------------- permuting prologue

@pytest.mark.parametrize("name,parts", [("tiny", (1, 2, 2)), ("block", (1, 2, 2)),
                                        ("block", (4, 1, 1)), ("720p", (1, 2, 2))])
def test_qk_norm_rope_window(name, parts):
    w = W[name]
    inp = I.make_inputs(w, seed=3, parts=("qkv", "scales"))
    t = device_inputs(inp)
    qw, kw = api.qk_norm_rope_window(t["q_vis"], t["k_vis"], t["gq_vis"], t["gk_vis"], w.grid,
                                     parts, pos_scale=w.pos_scale)
    # the same arithmetic as the raster-order kernel, stored at permuted rows
    qr, kr = api.qk_norm_rope(t["q_vis"].clone(), t["k_vis"].clone(), t["gq_vis"], t["gk_vis"],
                              grid=w.grid, pos_scale=w.pos_scale)
    order = torch.from_numpy(_order(w.grid, parts)).cuda()
    assert torch.equal(qw, qr[:, order])
    assert torch.equal(kw, kr[:, order])
    if name in ("tiny", "block"):
        rq, rk = oracle.qk_norm_rope(inp["q_vis"].f64, inp["k_vis"].f64, inp["gq_vis"],
                                     inp["gk_vis"], grid=w.grid, pos_scale=w.pos_scale)
        o = _order(w.grid, parts)
        parity(from_dev(qw), rq[:, o], w.dtype, "q window-major")
        parity(from_dev(kw), rk[:, o], w.dtype, "k window-major")


# ------------------------------------------------------------- window attention

def _window_run(w: I.Workload, parts, seed=0):
    """Raster-order inputs -> window-major q/k/v on the device -> attention."""
    inp = I.make_inputs(w, seed=seed, parts=("qkv",))
    t = device_inputs(inp)
    q = api.window_permute(t["q_vis"], w.grid, parts)
    k = api.window_permute(t["k_vis"], w.grid, parts)
    v = api.window_permute(t["v_vis"], w.grid, parts)
    o_vis, o_ctx = api.joint_window_attention(q, k, v, t["q_ctx"], t["k_ctx"], t["v_ctx"],
                                              w.grid, parts,
                                              t["ctx_len"] if w.ctx_len is not None else None)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    return inp, from_dev(o_vis), from_dev(o_ctx)


SMALL = {
    "tiny_f32_122": (W["tiny"], (1, 2, 2)),
    "tiny_f32_211": (W["tiny"], (2, 1, 1)),
    "tiny_f32_single_tokens": (W["tiny"], (2, 4, 4)),
    "f32_ragged_232": (_ws(W["tiny"], B=2, H=3, grid=(2, 6, 9), Nc=33, ctx_len=(30, 0)), (2, 3, 2)),
    "block_122": (W["block"], (1, 2, 2)),
    "block_411": (W["block"], (4, 1, 1)),
    "ragged_122": (_ws(W["block"], B=2, H=3, grid=(3, 10, 10), Nc=77, ctx_len=(77, 5)), (1, 2, 2)),
    "ragged_311": (_ws(W["block"], B=2, H=2, grid=(5, 9, 11), Nc=130, ctx_len=(0, 129)), (3, 1, 1)),
    "uneven_235": (_ws(W["block"], H=2, grid=(7, 9, 11), Nc=64), (2, 3, 5)),
    "no_cond_122": (_ws(W["block"], H=2, grid=(2, 20, 20), Nc=0), (1, 2, 2)),
    "big_windows_411": (_ws(W["block"], H=2, grid=(8, 16, 32), Nc=256), (4, 1, 1)),
}


@pytest.mark.parametrize("case", sorted(SMALL))
def test_window_attention_full(case):
    w, parts = SMALL[case]
    inp, ov, oc = _window_run(w, parts)
    rv, rc = oracle.window_attention(inp["q_vis"].f64, inp["k_vis"].f64, inp["v_vis"].f64,
                                     inp["q_ctx"].f64, inp["k_ctx"].f64, inp["v_ctx"].f64,
                                     w.grid, parts, inp["ctx_len"])
    parity(ov, rv, w.dtype, f"{case} o_vis")
    parity(oc, rc, w.dtype, f"{case} o_ctx")
    for b, L in enumerate(w.ctx_lengths()):
        assert np.all(oc[b, L:] == 0.0), "padded cond rows must be zero"


def test_single_window_is_joint_attention_bitwise():
    """One window over the whole grid runs the same per-row arithmetic in the
    same key order as the joint attention, so the outputs match bit for bit."""
    w = _ws(W["block"], B=2, H=3, grid=(3, 10, 11), Nc=200, ctx_len=(200, 17))
    inp = I.make_inputs(w, seed=5, parts=("qkv",))
    t = device_inputs(inp)
    args = (t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"], t["v_ctx"])
    jv, jc = api.joint_attention(*args, t["ctx_len"])
    wv, wc = api.joint_window_attention(*args, w.grid, (1, 1, 1), t["ctx_len"])
    torch.cuda.synchronize()
    assert torch.equal(jv, wv) and torch.equal(jc, wc)


def _window_rows(w: I.Workload, parts, b: int, h: int) -> np.ndarray:
    """parity_rows plus, for every window, its first and last tokens and the
    tokens on both sides of each 128-row query tile boundary inside it."""
    rows = set(I.parity_rows(w, b, h).tolist())
    for toks in brute.window_token_lists(w.grid, parts):
        for r in (0, len(toks) - 1, 127, 128, 255, 256):
            if r < len(toks):
                rows.add(int(toks[r]))
        last = (len(toks) - 1) // 128 * 128
        for r in (last - 1, last):
            if 0 <= r < len(toks):
                rows.add(int(toks[r]))
    return np.asarray(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("name,parts", [("480p", (1, 2, 2)), ("480p", (4, 1, 1)),
                                        ("ragged", (4, 1, 1))])
def test_window_attention_sampled_full_size(name, parts):
    w = W[name]
    inp, ov, oc = _window_run(w, parts)
    full = np.concatenate([ov, oc], axis=1)
    trip = []
    for b in range(w.B):
        for h in range(w.H):
            rows = _window_rows(w, parts, b, h)
            trip.append(np.stack([np.full_like(rows, b), np.full_like(rows, h), rows], axis=1))
    trip = np.concatenate(trip)
    ref = oracle.window_attention_rows(inp["q_vis"].f64, inp["k_vis"].f64, inp["v_vis"].f64,
                                       inp["q_ctx"].f64, inp["k_ctx"].f64, inp["v_ctx"].f64,
                                       inp["ctx_len"], w.grid, parts, trip)
    got = full[trip[:, 0], trip[:, 2], trip[:, 1]]
    vis = trip[:, 2] < w.Nv
    parity(got[vis], ref[vis], w.dtype, f"{name} {parts} o_vis rows")
    parity(got[~vis], ref[~vis], w.dtype, f"{name} {parts} o_ctx rows")


def test_window_chain_from_raster_inputs():
    """The intended use: permuting prologue for q/k, permute for v, windowed
    attention back to raster order, against the oracle's whole definition."""
    w = W["block"]
    parts = (1, 2, 2)
    inp = I.make_inputs(w, seed=7, parts=("qkv", "scales"))
    t = device_inputs(inp)
    q, k = api.qk_norm_rope_window(t["q_vis"], t["k_vis"], t["gq_vis"], t["gk_vis"], w.grid,
                                   parts)
    v = api.window_permute(t["v_vis"], w.grid, parts)
    api.qk_norm_rope(t["q_ctx"], t["k_ctx"], t["gq_ctx"], t["gk_ctx"], grid=None)
    ov, oc = api.joint_window_attention(q, k, v, t["q_ctx"], t["k_ctx"], t["v_ctx"], w.grid,
                                        parts)
    torch.cuda.synchronize()
    rq, rk = oracle.qk_norm_rope(inp["q_vis"].f64, inp["k_vis"].f64, inp["gq_vis"],
                                 inp["gk_vis"], grid=w.grid)
    cq, ck = oracle.qk_norm_rope(inp["q_ctx"].f64, inp["k_ctx"].f64, inp["gq_ctx"],
                                 inp["gk_ctx"], grid=None)
    # the attention inputs are the bf16-stored prologue outputs
    rq, rk, cq, ck = (I.round_f64_to_bf16(a) for a in (rq, rk, cq, ck))
    rv, rc = oracle.window_attention(rq, rk, inp["v_vis"].f64, cq, ck, inp["v_ctx"].f64,
                                     w.grid, parts)
    parity(from_dev(ov), rv, w.dtype, "chain o_vis")
    parity(from_dev(oc), rc, w.dtype, "chain o_ctx")


def test_window_api_rejects_bad_arguments():
    w = W["block"]
    t = device_inputs(I.make_inputs(w, seed=0, parts=("qkv", "scales")))
    args = (t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"], t["v_ctx"])
    with pytest.raises(api._lib.MmditError):
        api.joint_window_attention(*args, w.grid, (6, 1, 1))      # more parts than frames
    with pytest.raises(api._lib.MmditError):
        api.joint_window_attention(*args, (5, 8, 9), (1, 2, 2))   # grid != Nv
    with pytest.raises(api._lib.MmditError):                       # permuting in place
        api.qk_norm_rope_window(t["q_vis"], t["k_vis"], t["gq_vis"], t["gk_vis"], w.grid,
                                (1, 2, 2), q_out=t["q_vis"])


# ------------------------------------------------------------- window backward

def _window_bwd_run(w: I.Workload, parts, seed=0, one_pass=False):
    """Window forward with lse, then the window backward (two-kernel or
    one-pass form); gradients returned to raster order, lse as written
    (window-major visual rows)."""
    inp = I.make_inputs(w, seed=seed, parts=("qkv",))
    gin = I.make_grad_outputs(w, seed=seed)
    t = device_inputs(inp)
    cl = t["ctx_len"] if w.ctx_len is not None else None
    q, k, v = (api.window_permute(t[n], w.grid, parts) for n in ("q_vis", "k_vis", "v_vis"))
    ov, oc, lse = api.joint_window_attention_fwd(q, k, v, t["q_ctx"], t["k_ctx"], t["v_ctx"],
                                                 w.grid, parts, cl)
    ws = api.bwd_workspace(w.B, w.Nv, w.Nc, w.H) if one_pass else None
    if ws is not None:
        ws.fill_(0xFF)
    g = api.joint_window_attention_bwd(q, k, v, t["q_ctx"], t["k_ctx"], t["v_ctx"], ov, oc,
                                       to_dev(gin["do_vis"]), to_dev(gin["do_ctx"]), lse, w.grid,
                                       parts, cl, workspace=ws)
    for n in ("dq_vis", "dk_vis", "dv_vis"):
        g[n] = api.window_permute(g[n], w.grid, parts, inverse=True)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    return inp, gin, {n: from_dev(x) for n, x in g.items()}, from_dev(lse)


BWD = {
    "tiny_f32_122": (W["tiny"], (1, 2, 2)),
    "f32_ragged_232": (_ws(W["tiny"], B=2, H=3, grid=(2, 6, 9), Nc=33, ctx_len=(30, 0)), (2, 3, 2)),
    "block_122": (W["block"], (1, 2, 2)),
    "block_411": (W["block"], (4, 1, 1)),
    "ragged_311": (_ws(W["block"], B=2, H=2, grid=(5, 9, 11), Nc=130, ctx_len=(0, 129)), (3, 1, 1)),
    "uneven_235": (_ws(W["block"], H=2, grid=(7, 9, 11), Nc=64), (2, 3, 5)),
    "no_cond_122": (_ws(W["block"], H=2, grid=(2, 20, 20), Nc=0), (1, 2, 2)),
    "medium_2k_122": (_ws(W["block"], H=2, grid=(2, 32, 32), Nc=256), (1, 2, 2)),
}


@pytest.mark.parametrize("one_pass", [False, True])
@pytest.mark.parametrize("case", sorted(BWD))
def test_window_backward_full(case, one_pass):
    w, parts = BWD[case]
    inp, gin, g, lse = _window_bwd_run(w, parts, one_pass=one_pass)
    ref = oracle.window_attention_bwd(inp["q_vis"].f64, inp["k_vis"].f64, inp["v_vis"].f64,
                                      inp["q_ctx"].f64, inp["k_ctx"].f64, inp["v_ctx"].f64,
                                      gin["do_vis"].f64, gin["do_ctx"].f64, w.grid, parts,
                                      inp["ctx_len"])
    for n in ("dq_vis", "dk_vis", "dv_vis", "dq_ctx", "dk_ctx", "dv_ctx"):
        parity(g[n], ref[n], w.dtype, f"{case} {n}")
    # lse: the oracle's raster rows, reordered to the window-major order of q_vis
    order = _order(w.grid, parts)
    want = np.concatenate([ref["lse"][:, :, order], ref["lse"][:, :, w.Nv:]], axis=2)
    assert np.array_equal(np.isinf(lse), np.isinf(want)), f"{case}: +inf rows differ"
    fin = ~np.isinf(want)
    if fin.any():
        assert np.abs(lse[fin] - want[fin]).max() <= 1e-3, f"{case}: lse"
    for b, L in enumerate(w.ctx_lengths()):
        for n in ("dq_ctx", "dk_ctx", "dv_ctx"):
            assert np.all(g[n][b, L:] == 0.0), f"{case} {n}: padded rows must be zero"


def test_single_window_backward_is_the_joint_backward_bitwise():
    """With one window the window backward runs the joint backward's per-row
    arithmetic in the same order: bit for bit the same gradients."""
    w = _ws(W["block"], B=2, H=3, grid=(3, 10, 11), Nc=200, ctx_len=(200, 17))
    inp = I.make_inputs(w, seed=6, parts=("qkv",))
    gin = I.make_grad_outputs(w, seed=6)
    t = device_inputs(inp)
    args = (t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"], t["v_ctx"])
    do_v, do_c = to_dev(gin["do_vis"]), to_dev(gin["do_ctx"])
    jv, jc, jl = api.joint_attention_fwd(*args, t["ctx_len"])
    jg = api.joint_attention_bwd(*args, jv, jc, do_v, do_c, jl, t["ctx_len"])
    wv, wc, wl = api.joint_window_attention_fwd(*args, w.grid, (1, 1, 1), t["ctx_len"])
    wg = api.joint_window_attention_bwd(*args, wv, wc, do_v, do_c, wl, w.grid, (1, 1, 1),
                                        t["ctx_len"])
    torch.cuda.synchronize()
    assert torch.equal(jl, wl)
    for n in jg:
        assert torch.equal(jg[n], wg[n]), n
