"""GPU parity of the joint-attention backward (and of the forward's row
log-sum-exp) through the C ABI, against the float64 oracle on the same seeded
inputs and upstream gradients.

Small and medium cases compare every gradient element; the full 480p and
ragged workloads compare dq and lse on sampled query rows (each against the
full key set), dk and dv on sampled key rows of a few heads (each against every
query row), and dk / dv of every key through sum rules that hold at any size.
Each case runs both forms of the bf16 backward: the two-kernel form (dQ, then
dK / dV) and the one-pass form (dQ reduced into an fp32 workspace)."""
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


def _run(w: I.Workload, seed=0, one_pass=False):
    inp = I.make_inputs(w, seed=seed, parts=("qkv",))
    gin = I.make_grad_outputs(w, seed=seed)
    t = device_inputs(inp)
    do_vis, do_ctx = to_dev(gin["do_vis"]), to_dev(gin["do_ctx"])
    cl = t["ctx_len"] if w.ctx_len is not None else None
    ov, oc, lse = api.joint_attention_fwd(t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"],
                                          t["k_ctx"], t["v_ctx"], cl)
    ws = api.bwd_workspace(w.B, w.Nv, w.Nc, w.H) if one_pass else None
    if ws is not None:
        ws.fill_(0xFF)   # NaN bit patterns: the backward must not read stale contents
    g = api.joint_attention_bwd(t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"],
                                t["v_ctx"], ov, oc, do_vis, do_ctx, lse, cl, workspace=ws)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    return inp, gin, {k: from_dev(v) for k, v in g.items()}, from_dev(lse), (ov, oc)


def _check_lse(got, ref, name):
    assert np.array_equal(np.isinf(got), np.isinf(ref)), f"{name}: +inf rows differ"
    fin = ~np.isinf(ref)
    if fin.any():
        err = np.max(np.abs(got[fin] - ref[fin]))
        assert err <= 1e-3, f"{name}: lse max err {err}"


SMALL = {
    "tiny_f32": W["tiny"],
    "f32_ragged": _ws(W["tiny"], B=2, H=3, grid=(2, 5, 9), Nc=33, ctx_len=(30, 0)),
    "block": W["block"],
    "ragged_small": _ws(W["block"], B=2, H=3, grid=(3, 10, 10), Nc=77, ctx_len=(77, 5)),
    "odd_tiles": _ws(W["block"], H=2, grid=(1, 1, 257), Nc=0),
    "cond_all_masked": _ws(W["block"], H=2, grid=(2, 10, 10), Nc=130, ctx_len=(0,)),
    "batch3_mixed": _ws(W["block"], B=3, H=2, grid=(1, 13, 20), Nc=200, ctx_len=(0, 1, 200)),
    "medium_2k": _ws(W["block"], H=2, grid=(2, 32, 32), Nc=256),
}


@pytest.mark.parametrize("one_pass", [False, True])
@pytest.mark.parametrize("case", sorted(SMALL))
def test_backward_full(case, one_pass):
    w = SMALL[case]
    inp, gin, g, lse, _ = _run(w, one_pass=one_pass)
    ref = oracle.joint_attention_bwd(inp["q_vis"].f64, inp["k_vis"].f64, inp["v_vis"].f64,
                                     inp["q_ctx"].f64, inp["k_ctx"].f64, inp["v_ctx"].f64,
                                     gin["do_vis"].f64, gin["do_ctx"].f64, inp["ctx_len"])
    _check_lse(lse, ref["lse"], case)
    for k in ("dq_vis", "dk_vis", "dv_vis", "dq_ctx", "dk_ctx", "dv_ctx"):
        parity(g[k], ref[k], w.dtype, f"{case} {k}")
    for b, L in enumerate(w.ctx_lengths()):
        for k in ("dq_ctx", "dk_ctx", "dv_ctx"):
            assert np.all(g[k][b, L:] == 0.0), f"{case} {k}: padded rows must be zero"


@pytest.mark.parametrize("one_pass", [False, True])
@pytest.mark.parametrize("name", ["480p", "ragged"])
def test_backward_sampled_full_size(name, one_pass):
    w = W[name]
    inp, gin, g, lse, _ = _run(w, one_pass=one_pass)
    trip = []
    for b in range(w.B):
        for h in range(w.H):
            rows = I.parity_rows(w, b, h, n_random=128)
            trip.append(np.stack([np.full_like(rows, b), np.full_like(rows, h), rows], axis=1))
    trip = np.concatenate(trip)
    dq, lref = oracle.joint_attention_dq_rows(
        inp["q_vis"].f64, inp["k_vis"].f64, inp["v_vis"].f64, inp["q_ctx"].f64,
        inp["k_ctx"].f64, inp["v_ctx"].f64, gin["do_vis"].f64, gin["do_ctx"].f64,
        inp["ctx_len"], trip)
    full = np.concatenate([g["dq_vis"], g["dq_ctx"]], axis=1)
    got = full[trip[:, 0], trip[:, 2], trip[:, 1]]
    vis = trip[:, 2] < w.Nv
    parity(got[vis], dq[vis], w.dtype, f"{name} dq_vis rows")
    parity(got[~vis], dq[~vis], w.dtype, f"{name} dq_ctx rows")
    _check_lse(lse[trip[:, 0], trip[:, 1], trip[:, 2]], lref, f"{name} lse rows")
    # dk and dv element by element on sampled key rows (the query-row sampler
    # applied to keys: every cond key, both visual tails, the tile and padding
    # boundaries, 128 random keys), 2 heads at 480p and 1 head per sample of
    # the ragged batch; each key against every query row
    heads = {"480p": [(0, 0), (0, 17)], "ragged": [(0, 5), (1, 11)]}[name]
    keys = []
    for b, h in heads:
        rows = I.parity_rows(w, b, h, n_random=128)
        keys.append(np.stack([np.full_like(rows, b), np.full_like(rows, h), rows], axis=1))
    keys = np.concatenate(keys)
    dk, dv = oracle.joint_attention_dkdv_rows(
        inp["q_vis"].f64, inp["k_vis"].f64, inp["v_vis"].f64, inp["q_ctx"].f64,
        inp["k_ctx"].f64, inp["v_ctx"].f64, gin["do_vis"].f64, gin["do_ctx"].f64,
        inp["ctx_len"], keys)
    vis = keys[:, 2] < w.Nv
    for grad, ref, n in ((g["dk_vis"], g["dk_ctx"], "dk"), (g["dv_vis"], g["dv_ctx"], "dv")):
        full = np.concatenate([grad, ref], axis=1)
        got = full[keys[:, 0], keys[:, 2], keys[:, 1]]
        want = dk if n == "dk" else dv
        parity(got[vis], want[vis], w.dtype, f"{name} {n}_vis keys")
        parity(got[~vis], want[~vis], w.dtype, f"{name} {n}_ctx keys")
    # Sum rules, per (sample, head, dim): softmax rows sum to one, so
    # sum_j dv_j = sum_i dO_i over rows with an output, and sum_j dS_ij = 0, so
    # sum_j dk_j = 0.  Two bf16 roundings of random sign (P before the dV
    # product, and each stored gradient; relative 2^-8 at most) leave a
    # deviation of about 0.35 % of the root-sum-square of the terms per entry,
    # so about 1.2 % at the largest of the 3072 entries of a sample.  The bound
    # allows 3 %; one missing 128-key tile at 480p moves a sum by about 6 %.
    for b, L in enumerate(w.ctx_lengths()):
        do_sum = gin["do_vis"].f64[b].sum(0) + gin["do_ctx"].f64[b, :L].sum(0)
        dv = np.concatenate([g["dv_vis"][b], g["dv_ctx"][b]], 0)
        dk = np.concatenate([g["dk_vis"][b], g["dk_ctx"][b]], 0)
        rss_v = np.sqrt((dv ** 2).sum(0))
        rss_k = np.sqrt((dk ** 2).sum(0))
        assert np.all(np.abs(dv.sum(0) - do_sum) <= 3e-2 * rss_v + 1e-6), "sum of dv"
        assert np.all(np.abs(dk.sum(0)) <= 3e-2 * rss_k + 1e-6), "sum of dk"
        assert np.all(g["dk_ctx"][b, L:] == 0) and np.all(g["dv_ctx"][b, L:] == 0)


@pytest.mark.parametrize("case", ["ragged_small", "batch3_mixed", "medium_2k"])
def test_one_pass_dk_dv_equal_two_kernel_form(case):
    """Both forms form the same bf16 P^T and dS^T and the same dV and dK
    products in the same order (dS^T read from shared memory instead of tensor
    memory), so dK and dV agree bit for bit; dQ is summed in another order and
    agrees within the bf16 rounding of the two results."""
    w = SMALL[case]
    _, _, g2, _, _ = _run(w, one_pass=False)
    _, _, g1, _, _ = _run(w, one_pass=True)
    for k in ("dk_vis", "dv_vis", "dk_ctx", "dv_ctx"):
        assert np.array_equal(g1[k], g2[k]), f"{case} {k} differs between the forms"
    for k in ("dq_vis", "dq_ctx"):
        a, b = g1[k].astype(np.float64), g2[k].astype(np.float64)
        scale = np.sqrt(np.mean(b ** 2)) + 1e-30
        assert np.max(np.abs(a - b)) <= 2 ** -6 * scale + 1e-30, f"{case} {k}"


def test_one_pass_workspace_too_small_runs_two_kernel_form():
    w = SMALL["ragged_small"]
    inp = I.make_inputs(w, seed=0, parts=("qkv",))
    gin = I.make_grad_outputs(w, seed=0)
    t = device_inputs(inp)
    do_vis, do_ctx = to_dev(gin["do_vis"]), to_dev(gin["do_ctx"])
    args = (t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"], t["v_ctx"])
    ov, oc, lse = api.joint_attention_fwd(*args, t["ctx_len"])
    small = torch.empty(api.bwd_workspace_bytes(w.B, w.Nv, w.Nc, w.H) - 256, dtype=torch.uint8,
                        device="cuda")
    g_small = api.joint_attention_bwd(*args, ov, oc, do_vis, do_ctx, lse, t["ctx_len"],
                                      workspace=small)
    g_two = api.joint_attention_bwd(*args, ov, oc, do_vis, do_ctx, lse, t["ctx_len"])
    torch.cuda.synchronize()
    for k in g_two:   # the two-kernel form is deterministic
        assert torch.equal(g_small[k], g_two[k]), k


def test_forward_with_lse_matches_forward():
    """The forward with the lse output writes the same o as the plain one."""
    w = _ws(W["block"], B=2, H=3, grid=(3, 10, 11), Nc=200, ctx_len=(200, 17))
    t = device_inputs(I.make_inputs(w, seed=4, parts=("qkv",)))
    args = (t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"], t["v_ctx"], t["ctx_len"])
    a_v, a_c = api.joint_attention(*args)
    b_v, b_c, _ = api.joint_attention_fwd(*args)
    torch.cuda.synchronize()
    assert torch.equal(a_v, b_v) and torch.equal(a_c, b_c)


def test_backward_rejects_bad_arguments():
    w = W["block"]
    t = device_inputs(I.make_inputs(w, seed=0, parts=("qkv",)))
    args = (t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"], t["v_ctx"])
    ov, oc, lse = api.joint_attention_fwd(*args)
    with pytest.raises(api._lib.MmditError):
        api.joint_attention_bwd(*args, ov, oc, ov, oc, lse, softmax_scale=-1.0)
    bad = torch.empty(t["q_vis"].numel() + 8, dtype=torch.bfloat16, device="cuda")[1:]
    with pytest.raises(api._lib.MmditError):        # dq_vis not 16-byte aligned
        api.joint_attention_bwd(*args, ov, oc, ov, oc, lse,
                                grads={"dq_vis": bad[:t["q_vis"].numel()].view(t["q_vis"].shape)})


# ------------------------------------------------------ QK-RMSNorm + RoPE backward

@pytest.mark.parametrize("name", ["tiny", "block", "480p", "720p", "ragged"])
def test_qk_norm_rope_bwd(name):
    """dx against the oracle in full (bf16 / fp32 criterion); dg, a sum over
    every row, within 1e-3 of its largest entry."""
    w = W[name]
    inp = I.make_inputs(w, seed=2, parts=("qkv", "scales"))
    gin = I.make_grad_outputs(w, seed=2)
    t = device_inputs(inp)
    for stream, grid, dO in (("vis", w.grid, gin["do_vis"]), ("ctx", None, gin["do_ctx"])):
        dy = to_dev(dO)
        dq, dk, dgq, dgk = api.qk_norm_rope_bwd(
            t["q_" + stream], t["k_" + stream], t["gq_" + stream], t["gk_" + stream], dy, dy,
            grid=grid, pos_scale=w.pos_scale)
        torch.cuda.synchronize()
        rq, rk, rgq, rgk = oracle.qk_norm_rope_bwd(
            inp["q_" + stream].f64, inp["k_" + stream].f64, inp["gq_" + stream],
            inp["gk_" + stream], dO.f64, dO.f64, grid=grid, pos_scale=w.pos_scale)
        parity(from_dev(dq), rq, w.dtype, f"{name} dq_{stream}")
        parity(from_dev(dk), rk, w.dtype, f"{name} dk_{stream}")
        for got, ref, n in ((dgq, rgq, "dgq"), (dgk, rgk, "dgk")):
            err = np.max(np.abs(from_dev(got) - ref)) if ref.size else 0.0
            assert err <= 1e-3 * max(np.abs(ref).max(), 1e-30), (name, stream, n, err)


@pytest.mark.parametrize("name", ["block", "480p", "ragged"])
def test_qk_norm_rope_text_bwd(name):
    """The backward with MM-RoPE text positions (cond token n at offset + n on
    every axis chunk): dx in full against the oracle, dg within 1e-3 of its
    largest entry."""
    w = W[name]
    inp = I.make_inputs(w, seed=3, parts=("qkv", "scales"))
    gin = I.make_grad_outputs(w, seed=3)
    t = device_inputs(inp)
    off = float(max(w.grid))
    dy = to_dev(gin["do_ctx"])
    dq, dk, dgq, dgk = api.qk_norm_rope_text_bwd(t["q_ctx"], t["k_ctx"], t["gq_ctx"],
                                                 t["gk_ctx"], dy, dy, pos_offset=off)
    torch.cuda.synchronize()
    rq, rk, rgq, rgk = oracle.qk_norm_rope_text_bwd(
        inp["q_ctx"].f64, inp["k_ctx"].f64, inp["gq_ctx"], inp["gk_ctx"], gin["do_ctx"].f64,
        gin["do_ctx"].f64, offset=off)
    parity(from_dev(dq), rq, w.dtype, f"{name} dq_ctx text")
    parity(from_dev(dk), rk, w.dtype, f"{name} dk_ctx text")
    for got, ref, n in ((dgq, rgq, "dgq"), (dgk, rgk, "dgk")):
        err = np.max(np.abs(from_dev(got) - ref))
        assert err <= 1e-3 * max(np.abs(ref).max(), 1e-30), (name, n, err)
