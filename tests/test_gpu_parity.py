"""GPU parity: every kernel of the path against the float64 oracle on the same
seeded inputs, through the C ABI (the ctypes binding in mmdit_joint_attention_b200).

Small cases compare every output element; the full 480p / 720p / ragged
workloads compare the elementwise kernels in full and attention on sampled
query rows (every cond row, both visual tails, tile and padding boundaries,
512 random rows per (sample, head)), each against the full key set."""
import numpy as np
import pytest
import torch

import oracle
from mmdit_joint_attention_b200 import api
from mmdit_joint_attention_b200 import inputs as I
from helpers import device_inputs, from_dev, parity, to_dev

pytestmark = pytest.mark.gpu

W = I.WORKLOADS


def _ws(w: I.Workload, **kw) -> I.Workload:
    import dataclasses
    return dataclasses.replace(w, **kw)


# ---------------------------------------------------------------- QK norm + RoPE

@pytest.mark.parametrize("name", ["tiny", "block", "480p", "720p", "ragged"])
def test_qk_norm_rope(name):
    w = W[name]
    inp = I.make_inputs(w, parts=("qkv", "scales"))
    for s, grid in (("vis", w.grid), ("ctx", None)):
        q, k = to_dev(inp["q_" + s]), to_dev(inp["k_" + s])
        gq, gk = to_dev(inp["gq_" + s]), to_dev(inp["gk_" + s])
        qo, ko = torch.empty_like(q), torch.empty_like(k)
        api.qk_norm_rope(q, k, gq, gk, grid=grid, pos_scale=w.pos_scale, q_out=qo, k_out=ko)
        api.qk_norm_rope(q, k, gq, gk, grid=grid, pos_scale=w.pos_scale)  # in place
        torch.cuda.synchronize()
        rq, rk = oracle.qk_norm_rope(inp["q_" + s].f64, inp["k_" + s].f64, inp["gq_" + s],
                                     inp["gk_" + s], grid=grid, pos_scale=w.pos_scale)
        parity(from_dev(qo), rq, w.dtype, f"{name} q_{s}")
        parity(from_dev(ko), rk, w.dtype, f"{name} k_{s}")
        assert torch.equal(qo, q) and torch.equal(ko, k), "in-place result differs"


def test_qk_norm_rope_odd_grid_and_base():
    """A grid whose extents are not powers of two, another base and scaling."""
    w = _ws(W["block"], grid=(3, 7, 11), Nc=5, H=3)
    inp = I.make_inputs(w, parts=("qkv", "scales"))
    q, k = to_dev(inp["q_vis"]), to_dev(inp["k_vis"])
    api.qk_norm_rope(q, k, to_dev(inp["gq_vis"]), to_dev(inp["gk_vis"]), grid=w.grid,
                     pos_scale=(0.5, 2.0, 1.25), rope_base=500.0, eps=1e-3)
    rq, rk = oracle.qk_norm_rope(inp["q_vis"].f64, inp["k_vis"].f64, inp["gq_vis"],
                                 inp["gk_vis"], grid=w.grid, pos_scale=(0.5, 2.0, 1.25),
                                 base=500.0, eps=1e-3)
    parity(from_dev(q), rq, "bf16", "q")
    parity(from_dev(k), rk, "bf16", "k")


# ---------------------------------------------------------------- modulate / residual

@pytest.mark.parametrize("name", ["tiny", "block", "480p", "720p", "ragged"])
def test_modulate_and_residual(name):
    w = W[name]
    inp = I.make_inputs(w, parts=("qkv", "adaln"))
    # both streams in one launch: bit-equal to one launch per stream
    yv, yc = api.adaln_modulate_pair(
        to_dev(inp["x_vis"]), to_dev(inp["shift_vis"]), to_dev(inp["scale_vis"]),
        to_dev(inp["x_ctx"]), to_dev(inp["shift_ctx"]), to_dev(inp["scale_ctx"]))
    pair = {"vis": yv, "ctx": yc}
    for s in ("vis", "ctx"):
        n = w.Nv if s == "vis" else w.Nc
        x = to_dev(inp["x_" + s])
        y = api.adaln_modulate(x, to_dev(inp["shift_" + s]), to_dev(inp["scale_" + s]))
        br = to_dev(inp["v_" + s]).view(w.B, n, w.C)
        out = api.gated_residual(x, br, to_dev(inp["gate_" + s]), out=torch.empty_like(x))
        torch.cuda.synchronize()
        ry = oracle.adaln_modulate(inp["x_" + s].f64, inp["shift_" + s], inp["scale_" + s])
        rr = oracle.gated_residual(inp["x_" + s].f64, inp["v_" + s].f64.reshape(w.B, n, w.C),
                                   inp["gate_" + s])
        parity(from_dev(y), ry, w.dtype, f"{name} y_{s}")
        parity(from_dev(out), rr, w.dtype, f"{name} residual_{s}")
        assert torch.equal(pair[s], y), f"{name} y_{s}: the pair launch differs"


def test_modulate_pair_one_stream_empty_and_in_place():
    """The pair launch with an empty conditioning stream equals the single
    launch; y may overwrite its own x."""
    w = _ws(W["block"], B=2, ctx_len=None)
    inp = I.make_inputs(w, parts=("adaln",))
    xv = to_dev(inp["x_vis"])
    sv, cv = to_dev(inp["shift_vis"]), to_dev(inp["scale_vis"])
    empty = torch.empty((w.B, 0, w.C), dtype=xv.dtype, device=xv.device)
    yv, _ = api.adaln_modulate_pair(xv, sv, cv, empty, sv, cv)
    assert torch.equal(yv, api.adaln_modulate(xv, sv, cv))
    xc = to_dev(inp["x_ctx"])
    yc_ref = api.adaln_modulate(xc, to_dev(inp["shift_ctx"]), to_dev(inp["scale_ctx"]))
    xv2, xc2 = xv.clone(), xc.clone()
    api.adaln_modulate_pair(xv2, sv, cv, xc2, to_dev(inp["shift_ctx"]), to_dev(inp["scale_ctx"]),
                            out_vis=xv2, out_ctx=xc2)
    torch.cuda.synchronize()
    assert torch.equal(xv2, yv) and torch.equal(xc2, yc_ref)


def test_modulate_large_mean_rows():
    """Rows with a large common offset (two-pass variance) and C not a
    multiple of 256 (partial last chunk per lane)."""
    C, B, N = 1000, 2, 37
    r = np.random.Generator(np.random.PCG64(5))
    x32 = (r.standard_normal((B, N, C)) * 0.5 + 40.0).astype(np.float32)
    xb = I.Tensor(I.f32_to_bf16_bits(x32), "bf16")
    shift = (r.standard_normal((B, C)) * 0.1).astype(np.float32)
    scale = (r.standard_normal((B, C)) * 0.1).astype(np.float32)
    y = api.adaln_modulate(to_dev(xb), to_dev(shift), to_dev(scale))
    parity(from_dev(y), oracle.adaln_modulate(xb.f64, shift, scale), "bf16", "y")


# ---------------------------------------------------------------- joint attention

def _attention_case(w: I.Workload, seed=0):
    inp = I.make_inputs(w, seed=seed, parts=("qkv",))
    t = device_inputs(inp)
    o_vis, o_ctx = api.joint_attention(t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"],
                                       t["k_ctx"], t["v_ctx"],
                                       t["ctx_len"] if w.ctx_len is not None else None)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    return inp, from_dev(o_vis), from_dev(o_ctx)


SMALL = {
    "tiny_f32": W["tiny"],
    "block": W["block"],
    "ragged_small": _ws(W["block"], B=2, H=3, grid=(3, 10, 10), Nc=77, ctx_len=(77, 5)),
    "self_only_odd_tiles": _ws(W["block"], H=2, grid=(1, 1, 257), Nc=0),
    "cond_all_masked": _ws(W["block"], H=2, grid=(2, 10, 10), Nc=130, ctx_len=(0,)),
    "batch3_mixed": _ws(W["block"], B=3, H=2, grid=(1, 13, 20), Nc=200, ctx_len=(0, 1, 200)),
    "long_2k": _ws(W["block"], H=2, grid=(4, 16, 32), Nc=64),
    "f32_ragged": _ws(W["tiny"], B=2, H=3, grid=(2, 5, 9), Nc=33, ctx_len=(30, 0)),
}


@pytest.mark.parametrize("case", sorted(SMALL))
def test_attention_full(case):
    w = SMALL[case]
    inp, ov, oc = _attention_case(w)
    rv, rc = oracle.joint_attention(inp["q_vis"].f64, inp["k_vis"].f64, inp["v_vis"].f64,
                                    inp["q_ctx"].f64, inp["k_ctx"].f64, inp["v_ctx"].f64,
                                    inp["ctx_len"])
    parity(ov, rv, w.dtype, f"{case} o_vis")
    parity(oc, rc, w.dtype, f"{case} o_ctx")
    for b, L in enumerate(w.ctx_lengths()):
        assert np.all(oc[b, L:] == 0.0), "padded cond rows must be zero"


def test_attention_cond_only():
    """No visual tokens: plain attention over the conditioning stream."""
    B, Nc, H = 1, 150, 2
    r = np.random.Generator(np.random.PCG64(9))
    mk = lambda n: I.Tensor(I.f32_to_bf16_bits(r.standard_normal((B, n, H, 128)).astype(np.float32)), "bf16")  # noqa: E731
    qc, kc, vc = mk(Nc), mk(Nc), mk(Nc)
    e = torch.empty((B, 0, H, 128), dtype=torch.bfloat16, device="cuda")
    ov, oc = api.joint_attention(e, e, e, to_dev(qc), to_dev(kc), to_dev(vc))
    empty = np.zeros((B, 0, H, 128))
    _, rc = oracle.joint_attention(empty, empty, empty, qc.f64, kc.f64, vc.f64)
    parity(from_dev(oc), rc, "bf16", "o_ctx")


def test_attention_large_scores():
    """Scores spanning hundreds of units exercise the lazy maximum update."""
    w = _ws(W["block"], H=2, grid=(2, 8, 20), Nc=64)
    inp = I.make_inputs(w, seed=3, parts=("qkv",))
    ramp = np.linspace(0.2, 12.0, w.Nv, dtype=np.float32)[None, :, None, None]
    for key in ("q_vis", "k_vis"):
        a = I.bf16_bits_to_f32(inp[key].storage) * ramp
        inp[key] = I.Tensor(I.f32_to_bf16_bits(a), "bf16")
    t = device_inputs(inp)
    ov, oc = api.joint_attention(t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"],
                                 t["v_ctx"])
    rv, rc = oracle.joint_attention(inp["q_vis"].f64, inp["k_vis"].f64, inp["v_vis"].f64,
                                    inp["q_ctx"].f64, inp["k_ctx"].f64, inp["v_ctx"].f64)
    parity(from_dev(ov), rv, "bf16", "o_vis")
    parity(from_dev(oc), rc, "bf16", "o_ctx")


@pytest.mark.parametrize("name", ["480p", "720p", "ragged"])
def test_attention_sampled_full_size(name):
    w = W[name]
    inp, ov, oc = _attention_case(w)
    full = np.concatenate([ov, oc], axis=1)          # [B, Nv+Nc, H, D]
    trip = []
    for b in range(w.B):
        for h in range(w.H):
            rows = I.parity_rows(w, b, h)
            trip.append(np.stack([np.full_like(rows, b), np.full_like(rows, h), rows], axis=1))
    trip = np.concatenate(trip)
    ref = oracle.joint_attention_rows(inp["q_vis"].f64, inp["k_vis"].f64, inp["v_vis"].f64,
                                      inp["q_ctx"].f64, inp["k_ctx"].f64, inp["v_ctx"].f64,
                                      inp["ctx_len"], trip)
    got = full[trip[:, 0], trip[:, 2], trip[:, 1]]
    vis = trip[:, 2] < w.Nv
    parity(got[vis], ref[vis], w.dtype, f"{name} o_vis rows")
    parity(got[~vis], ref[~vis], w.dtype, f"{name} o_ctx rows")


# ---------------------------------------------------------------- whole path

@pytest.mark.parametrize("name", ["tiny", "block"])
def test_block_full_path(name):
    w = W[name]
    inp = I.make_inputs(w)
    t = device_inputs(inp)
    out = api.block_forward(t, grid=w.grid, pos_scale=w.pos_scale)
    torch.cuda.synchronize()
    ref = oracle.block(inp)
    for k in ("y_vis", "y_ctx", "o_vis", "o_ctx", "x_vis", "x_ctx"):
        parity(from_dev(out[k]), ref[k], w.dtype, f"{name} {k}")
    for k in ("q_vis", "k_vis", "q_ctx", "k_ctx"):
        parity(from_dev(t[k]), ref[k], w.dtype, f"{name} {k}")


def test_api_rejects_bad_arguments():
    x = torch.zeros((1, 4, 3072), dtype=torch.bfloat16, device="cuda")
    bad = torch.zeros((1, 3070), dtype=torch.float32, device="cuda")
    with pytest.raises(Exception):
        api.adaln_modulate(x[:, :, :3070].contiguous(), bad, bad)
    q = torch.zeros((1, 32, 2, 128), dtype=torch.bfloat16, device="cuda")
    g = torch.ones(128, dtype=torch.float32, device="cuda")
    with pytest.raises(api._lib.MmditError) as e:
        api.qk_norm_rope(q, q.clone(), g, g, grid=(2, 4, 5))
    assert e.value.status == -2


# ---------------------------------------------------------------- fused residual + modulate

@pytest.mark.parametrize("name", ["tiny", "block", "480p"])
def test_residual_modulate_fused(name):
    """x' = x + gate * branch and y = LN(x') (1 + scale) + shift of the next
    branch in one pass; the LayerNorm reads x' as stored (rounded to the
    storage type), like the two separate kernels run back to back."""
    w = W[name]
    inp = I.make_inputs(w, parts=("qkv", "adaln"))
    rnd = I.round_f64_to_bf16 if w.dtype == "bf16" else I.round_f64_to_f32
    n = w.Nv
    x = to_dev(inp["x_vis"])
    br = to_dev(inp["v_vis"]).view(w.B, n, w.C)
    gate, shift, scale = (to_dev(inp[k]) for k in ("gate_vis", "shift_ctx", "scale_ctx"))
    xo, y = api.residual_modulate(x, br, gate, shift, scale, x_out=torch.empty_like(x))
    # the unfused pair on the same inputs
    xo2 = api.gated_residual(x, br, gate, out=torch.empty_like(x))
    y2 = api.adaln_modulate(xo2, shift, scale)
    torch.cuda.synchronize()
    assert torch.equal(xo, xo2) and torch.equal(y, y2)
    rxo, ry = oracle.residual_modulate(inp["x_vis"].f64, inp["v_vis"].f64.reshape(w.B, n, w.C),
                                       inp["gate_vis"], inp["shift_ctx"], inp["scale_ctx"],
                                       round_to=rnd)
    parity(from_dev(xo), rxo, w.dtype, f"{name} x_out")
    parity(from_dev(y), ry, w.dtype, f"{name} y")
    # in place into x
    api.residual_modulate(x, br, gate, shift, scale, y=y)
    torch.cuda.synchronize()
    assert torch.equal(x, xo)


# ---------------------------------------------------------------- MM-RoPE text positions

@pytest.mark.parametrize("name,offset", [("tiny", 0.0), ("block", 52.0), ("ragged", 3.0),
                                         ("480p", 80.0)])
def test_qk_norm_rope_text(name, offset):
    """QK-RMSNorm + MM-RoPE text positions (token n at offset + n on all three
    axis chunks) on the conditioning stream."""
    w = W[name]
    inp = I.make_inputs(w, parts=("qkv", "scales"))
    q, k = to_dev(inp["q_ctx"]), to_dev(inp["k_ctx"])
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    api.qk_norm_rope_text(q, k, to_dev(inp["gq_ctx"]), to_dev(inp["gk_ctx"]), pos_offset=offset,
                          q_out=qo, k_out=ko)
    torch.cuda.synchronize()
    rq, rk = oracle.qk_norm_rope_text(inp["q_ctx"].f64, inp["k_ctx"].f64, inp["gq_ctx"],
                                      inp["gk_ctx"], offset=offset)
    parity(from_dev(qo), rq, w.dtype, f"{name} q_ctx")
    parity(from_dev(ko), rk, w.dtype, f"{name} k_ctx")


# ---------------------------------------------------------------- invariants on the GPU

def test_attention_padded_keys_have_no_influence():
    """Changing the padded cond keys / values leaves every output bit-identical."""
    w = SMALL["ragged_small"]
    inp = I.make_inputs(w, parts=("qkv",))
    t = device_inputs(inp)
    a = api.joint_attention(t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"],
                            t["v_ctx"], t["ctx_len"])
    for b, L in enumerate(w.ctx_lengths()):
        t["k_ctx"][b, L:] = 50.0
        t["v_ctx"][b, L:] = -7.0
    c = api.joint_attention(t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"],
                            t["v_ctx"], t["ctx_len"])
    torch.cuda.synchronize()
    assert torch.equal(a[0], c[0]) and torch.equal(a[1], c[1])


def test_attention_identical_keys_give_mean_v_and_unit_v_gives_one():
    w = _ws(W["block"], B=2, H=2, grid=(2, 9, 15), Nc=70, ctx_len=(70, 31))
    inp = I.make_inputs(w, parts=("qkv",))
    t = device_inputs(inp)
    t["k_vis"][:] = t["k_vis"][0, 0]
    t["k_ctx"][:] = t["k_vis"][0, 0]
    ov, oc = api.joint_attention(t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"],
                                 t["v_ctx"], t["ctx_len"])
    v = from_dev(t["v_vis"])
    vc = from_dev(t["v_ctx"])
    for b, L in enumerate(w.ctx_lengths()):
        mean = np.concatenate([v[b], vc[b, :L]], axis=0).mean(axis=0)      # [H, D]
        parity(from_dev(ov)[b], np.broadcast_to(mean, ov[b].shape), "bf16", "o_vis = mean(V)")
        parity(from_dev(oc)[b, :L], np.broadcast_to(mean, oc[b, :L].shape), "bf16",
               "o_ctx = mean(V)")
    ones_v, ones_c = torch.ones_like(t["v_vis"]), torch.ones_like(t["v_ctx"])
    ov, oc = api.joint_attention(t["q_vis"], t["k_vis"], ones_v, t["q_ctx"], t["k_ctx"], ones_c,
                                 t["ctx_len"])
    parity(from_dev(ov), np.ones(ov.shape), "bf16", "rows sum to one")


# ------------------------------------------- q normalised inside the attention kernel

def _qnorm_paths(w: I.Workload, seed=6):
    inp = I.make_inputs(w, seed=seed, parts=("qkv", "scales"))
    t = device_inputs(inp)
    cl = t["ctx_len"] if w.ctx_len is not None else None
    # unfused: q and k through the prologue kernel, then the attention
    qv, kv = api.qk_norm_rope(t["q_vis"].clone(), t["k_vis"].clone(), t["gq_vis"], t["gk_vis"],
                              grid=w.grid, pos_scale=w.pos_scale)
    qc, kc = api.qk_norm_rope(t["q_ctx"].clone(), t["k_ctx"].clone(), t["gq_ctx"], t["gk_ctx"])
    a_v, a_c = api.joint_attention(qv, kv, t["v_vis"], qc, kc, t["v_ctx"], cl)
    # fused: k alone through the prologue, raw q into the attention kernel
    kv2 = api.k_norm_rope(t["k_vis"].clone(), t["gk_vis"], grid=w.grid, pos_scale=w.pos_scale)
    kc2 = api.k_norm_rope(t["k_ctx"].clone(), t["gk_ctx"])
    f_v, f_c = api.joint_attention_qnorm(t["q_vis"], kv2, t["v_vis"], t["q_ctx"], kc2, t["v_ctx"],
                                         t["gq_vis"], t["gq_ctx"], grid=w.grid,
                                         pos_scale=w.pos_scale, ctx_len=cl)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    assert torch.equal(kv, kv2) and torch.equal(kc, kc2), "k alone must match the pair kernel"
    return inp, (a_v, a_c), (f_v, f_c)


@pytest.mark.parametrize("case", ["block", "ragged_small", "batch3_mixed", "long_2k"])
def test_attention_qnorm_full(case):
    w = SMALL[case]
    inp, (a_v, a_c), (f_v, f_c) = _qnorm_paths(w)
    rq, rk = oracle.qk_norm_rope(inp["q_vis"].f64, inp["k_vis"].f64, inp["gq_vis"],
                                 inp["gk_vis"], grid=w.grid, pos_scale=w.pos_scale)
    cq, ck = oracle.qk_norm_rope(inp["q_ctx"].f64, inp["k_ctx"].f64, inp["gq_ctx"],
                                 inp["gk_ctx"], grid=None)
    rq, rk, cq, ck = (I.round_f64_to_bf16(a) for a in (rq, rk, cq, ck))
    rv, rc = oracle.joint_attention(rq, rk, inp["v_vis"].f64, cq, ck, inp["v_ctx"].f64,
                                    inp["ctx_len"])
    parity(from_dev(f_v), rv, w.dtype, f"{case} fused o_vis")
    parity(from_dev(f_c), rc, w.dtype, f"{case} fused o_ctx")
    # the fused and the unfused path agree to within the same bound
    parity(from_dev(f_v), from_dev(a_v), w.dtype, f"{case} fused vs unfused o_vis")
    parity(from_dev(f_c), from_dev(a_c), w.dtype, f"{case} fused vs unfused o_ctx")


@pytest.mark.parametrize("name", ["480p", "720p"])
def test_attention_qnorm_sampled_full_size(name):
    w = W[name]
    inp, _, (f_v, f_c) = _qnorm_paths(w)
    full = np.concatenate([from_dev(f_v), from_dev(f_c)], axis=1)
    rq, rk = oracle.qk_norm_rope(inp["q_vis"].f64, inp["k_vis"].f64, inp["gq_vis"],
                                 inp["gk_vis"], grid=w.grid, pos_scale=w.pos_scale)
    cq, ck = oracle.qk_norm_rope(inp["q_ctx"].f64, inp["k_ctx"].f64, inp["gq_ctx"],
                                 inp["gk_ctx"], grid=None)
    rq, rk, cq, ck = (I.round_f64_to_bf16(a) for a in (rq, rk, cq, ck))
    trip = []
    for h in range(w.H):
        rows = I.parity_rows(w, 0, h, n_random=128)
        trip.append(np.stack([np.zeros_like(rows), np.full_like(rows, h), rows], axis=1))
    trip = np.concatenate(trip)
    ref = oracle.joint_attention_rows(rq, rk, inp["v_vis"].f64, cq, ck, inp["v_ctx"].f64,
                                      inp["ctx_len"], trip)
    got = full[trip[:, 0], trip[:, 2], trip[:, 1]]
    vis = trip[:, 2] < w.Nv
    parity(got[vis], ref[vis], w.dtype, f"{name} fused o_vis rows")
    parity(got[~vis], ref[~vis], w.dtype, f"{name} fused o_ctx rows")
