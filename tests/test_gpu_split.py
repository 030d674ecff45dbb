"""Split tail of the bf16 joint attention (mmdit_joint_attention_ws): the items
past the last whole wave of CTAs (every item, when a launch is smaller than a
wave) are split over their key tiles, and a second kernel merges the pieces.
Outputs and the row log-sum-exp must match the oracle as the unsplit kernel's
do.  The cases cover pieces left without a valid key by a short ctx_len, a
last query-tile pair with a single tile, and a launch whose first items stay
whole; a workspace too small for the plan must give the unsplit result."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from mmdit_joint_attention_b200 import api
from mmdit_joint_attention_b200 import inputs as I
from helpers import device_inputs, from_dev, parity

pytestmark = pytest.mark.gpu

W = I.WORKLOADS


def _ws(w, **kw):
    return dataclasses.replace(w, **kw)


# (workload, plan on 148 SMs: items, split items x pieces of key tiles)
CASES = {
    # 72 items < 148: every item in 2 pieces of 3 + 2 key tiles
    "all_split": _ws(W["block"]),
    # 12 items in 3 pieces of 2 tiles; ctx_len 0 leaves pieces 2 and 3 of
    # sample 0 without a valid key, ctx_len 130 leaves piece 3 of sample 1
    "empty_pieces": _ws(W["block"], B=2, H=2, grid=(1, 16, 16), Nc=512, ctx_len=(0, 130)),
    # 5 query tiles (the last pair has one), 2 pieces of 3 + 2 tiles
    "single_tile_pair": _ws(W["block"], H=3, grid=(1, 5, 61), Nc=200, ctx_len=(150,)),
    # 200 items: the first 148 whole, the last 52 in 2 pieces of 5 + 4 tiles
    "whole_then_split": _ws(W["block"], H=40, grid=(4, 16, 16), Nc=128),
}


def _run(w, workspace, seed=5):
    inp = I.make_inputs(w, seed=seed, parts=("qkv",))
    t = device_inputs(inp)
    cl = t["ctx_len"] if w.ctx_len is not None else None
    ov, oc, lse = api.joint_attention_fwd(t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"],
                                          t["k_ctx"], t["v_ctx"], cl, workspace=workspace)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    return inp, ov, oc, lse


@pytest.mark.parametrize("case", sorted(CASES))
def test_split_tail_matches_oracle(case):
    w = CASES[case]
    inp, ov, oc, lse = _run(w, api.attention_workspace())
    rv, rc = oracle.joint_attention(inp["q_vis"].f64, inp["k_vis"].f64, inp["v_vis"].f64,
                                    inp["q_ctx"].f64, inp["k_ctx"].f64, inp["v_ctx"].f64,
                                    inp["ctx_len"])
    parity(from_dev(ov), rv, "bf16", f"{case} o_vis")
    parity(from_dev(oc), rc, "bf16", f"{case} o_ctx")
    if case == "whole_then_split":
        return          # the lse oracle (a full backward) is slow at this size
    zeros = lambda a: np.zeros(a.shape)  # noqa: E731
    ref = oracle.joint_attention_bwd(inp["q_vis"].f64, inp["k_vis"].f64, inp["v_vis"].f64,
                                     inp["q_ctx"].f64, inp["k_ctx"].f64, inp["v_ctx"].f64,
                                     zeros(inp["q_vis"].f64), zeros(inp["q_ctx"].f64),
                                     inp["ctx_len"])["lse"]
    got = from_dev(lse)
    assert np.array_equal(np.isinf(got), np.isinf(ref)), f"{case}: +inf rows differ"
    fin = ~np.isinf(ref)
    assert np.max(np.abs(got[fin] - ref[fin])) <= 1e-3, case


def test_split_tail_close_to_unsplit_and_small_workspace_falls_back():
    """The split result differs from the unsplit one only by the order of the
    sums; a workspace smaller than the plan needs runs the unsplit kernel."""
    w = CASES["empty_pieces"]
    _, ov_s, oc_s, lse_s = _run(w, api.attention_workspace())
    _, ov_u, oc_u, lse_u = _run(w, None)
    _, ov_f, oc_f, lse_f = _run(w, torch.empty(4096, dtype=torch.uint8, device="cuda"))
    for a, b in ((ov_f, ov_u), (oc_f, oc_u)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(lse_f, lse_u)
    for a, b in ((ov_s, ov_u), (oc_s, oc_u)):
        d = (a.float() - b.float()).abs().max().item()
        assert d <= 1e-2 * b.float().abs().max().item(), d
    fin = torch.isfinite(lse_u)
    assert torch.equal(torch.isfinite(lse_s), fin)
    assert (lse_s[fin] - lse_u[fin]).abs().max().item() <= 1e-4


@pytest.mark.parametrize("case", ["all_split", "whole_then_split"])
def test_split_tail_with_qnorm(case):
    """The split tail with q normalised and rotated inside the kernel
    (mmdit_joint_attention_qnorm_ws): every piece normalises its own copy of
    the query tiles, and the merged rows match the oracle."""
    w = CASES[case]
    inp = I.make_inputs(w, seed=7, parts=("qkv", "scales"))
    t = device_inputs(inp)
    cl = t["ctx_len"] if w.ctx_len is not None else None
    kv = api.k_norm_rope(t["k_vis"].clone(), t["gk_vis"], grid=w.grid, pos_scale=w.pos_scale)
    kc = api.k_norm_rope(t["k_ctx"].clone(), t["gk_ctx"])
    fv, fc = api.joint_attention_qnorm(t["q_vis"], kv, t["v_vis"], t["q_ctx"], kc, t["v_ctx"],
                                       t["gq_vis"], t["gq_ctx"], grid=w.grid,
                                       pos_scale=w.pos_scale, ctx_len=cl,
                                       workspace=api.attention_workspace())
    torch.cuda.synchronize()
    assert api.device_status() == 0
    rq, rk = oracle.qk_norm_rope(inp["q_vis"].f64, inp["k_vis"].f64, inp["gq_vis"],
                                 inp["gk_vis"], grid=w.grid, pos_scale=w.pos_scale)
    cq, ck = oracle.qk_norm_rope(inp["q_ctx"].f64, inp["k_ctx"].f64, inp["gq_ctx"],
                                 inp["gk_ctx"], grid=None)
    rq, rk, cq, ck = (I.round_f64_to_bf16(a) for a in (rq, rk, cq, ck))
    rv, rc = oracle.joint_attention(rq, rk, inp["v_vis"].f64, cq, ck, inp["v_ctx"].f64,
                                    inp["ctx_len"])
    parity(from_dev(fv), rv, "bf16", f"{case} qnorm split o_vis")
    parity(from_dev(fc), rc, "bf16", f"{case} qnorm split o_ctx")
