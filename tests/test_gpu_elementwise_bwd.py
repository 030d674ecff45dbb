"""Backward of the adaLN modulate and of the gated residual against the
oracle's backward (pinned by finite differences, torch autograd and the
LayerNorm invariances).  dx and dbranch, stored in the workload's dtype, meet
the usual criterion; the [B, C] sums over the rows (fp32, added with atomics)
are checked against a relative 1e-4 of their largest magnitude."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from mmdit_joint_attention_b200 import api
from mmdit_joint_attention_b200 import inputs as I
from helpers import from_dev, parity, to_dev

pytestmark = pytest.mark.gpu

W = I.WORKLOADS
CASES = {
    "tiny_f32": W["tiny"],
    "block": W["block"],
    "batch2_ragged_rows": dataclasses.replace(W["block"], B=2, grid=(1, 7, 11), Nc=77),
    "480p_vis": W["480p"],
}


def _rows(t: I.Tensor, B: int, N: int, C: int) -> I.Tensor:
    return I.Tensor(t.storage.reshape(B, N, C), t.dtype)


def _sum_close(got, ref, name):
    err = float(np.max(np.abs(got - ref)))
    scale = max(float(np.max(np.abs(ref))), 1.0)
    assert err <= 1e-4 * scale, (name, err, scale)


def _inputs(w, seed):
    inp = I.make_inputs(w, seed=seed, parts=("adaln",))
    gin = I.make_grad_outputs(w, seed=seed)
    other = I.make_inputs(w, seed=seed + 1, parts=("adaln",))
    return inp, _rows(gin["do_vis"], w.B, w.Nv, w.C), other["x_vis"]


@pytest.mark.parametrize("case", sorted(CASES))
def test_modulate_bwd_matches_oracle(case):
    w = CASES[case]
    inp, dy, _ = _inputs(w, 41)
    x, sc = inp["x_vis"], inp["scale_vis"]
    # caller-held outputs full of NaN: every element must be written, and the
    # column sums zeroed before the rows add into them
    xd = to_dev(x)
    nan = lambda shape, dt: torch.full(shape, float("nan"), dtype=dt, device=xd.device)
    dx, dsh, dsc = api.adaln_modulate_bwd(
        xd, to_dev(sc), to_dev(dy), dx=nan(xd.shape, xd.dtype),
        dshift=nan((w.B, w.C), torch.float32), dscale=nan((w.B, w.C), torch.float32))
    torch.cuda.synchronize()
    ref = oracle.adaln_modulate_bwd(x.f64, sc, dy.f64)
    parity(from_dev(dx), ref["dx"], w.dtype, f"{case} dx")
    _sum_close(from_dev(dsh), ref["dshift"], f"{case} dshift")
    _sum_close(from_dev(dsc), ref["dscale"], f"{case} dscale")


@pytest.mark.parametrize("case", sorted(CASES))
def test_residual_bwd_matches_oracle(case):
    w = CASES[case]
    inp, dout, br = _inputs(w, 43)
    g = inp["gate_vis"]
    brd = to_dev(br)
    dbr, dg = api.gated_residual_bwd(
        brd, to_dev(g), to_dev(dout),
        dbranch=torch.full(brd.shape, float("nan"), dtype=brd.dtype, device=brd.device),
        dgate=torch.full((w.B, w.C), float("nan"), dtype=torch.float32, device=brd.device))
    torch.cuda.synchronize()
    ref = oracle.gated_residual_bwd(br.f64, g, dout.f64)
    parity(from_dev(dbr), ref["dbranch"], w.dtype, f"{case} dbranch")
    _sum_close(from_dev(dg), ref["dgate"], f"{case} dgate")


def test_residual_bwd_dx_copy_and_in_place_modulate():
    """The residual's optional dx is dout bit for bit; the modulate's dx may
    overwrite dy and then equals the out-of-place result."""
    from mmdit_joint_attention_b200 import _lib
    w = W["block"]
    inp, dout, br = _inputs(w, 47)
    d_dout, d_br, d_g = to_dev(dout), to_dev(br), to_dev(inp["gate_vis"])
    dx = torch.empty_like(d_dout)
    dbr = torch.empty_like(d_br)
    dg = torch.empty_like(d_g)
    st = _lib.lib().mmdit_gated_residual_bwd(d_br.data_ptr(), d_g.data_ptr(), d_dout.data_ptr(),
                                             dx.data_ptr(), dbr.data_ptr(), dg.data_ptr(),
                                             w.B, w.Nv, w.C, _lib.MMDIT_BF16, None)
    assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(dx.view(torch.int16), d_dout.view(torch.int16))
    x, sc = to_dev(inp["x_vis"]), to_dev(inp["scale_vis"])
    d_dy = to_dev(dout)
    ref_dx, _, _ = api.adaln_modulate_bwd(x, sc, d_dy)
    dsh, dsc = torch.empty_like(d_g), torch.empty_like(d_g)
    st = _lib.lib().mmdit_adaln_modulate_bwd(x.data_ptr(), sc.data_ptr(), d_dy.data_ptr(),
                                             d_dy.data_ptr(), dsh.data_ptr(), dsc.data_ptr(),
                                             w.B, w.Nv, w.C, 1e-6, _lib.MMDIT_BF16, None)
    assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(d_dy.view(torch.int16), ref_dx.view(torch.int16))
