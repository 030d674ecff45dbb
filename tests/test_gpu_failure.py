"""Failure detection on the GPU without a fault: every wait in the attention
kernels (forward, backward, 8-bit) is bounded; when one runs out the kernel
drains, frees its tensor memory, returns, and the status word reports
MMDIT_ERR_TIMEOUT.  The tests shorten the wait limit so that the waits of an
ordinary launch run out, then check the status, and that the context is
healthy afterwards."""
import pytest
import torch

import oracle
from mmdit_joint_attention_b200 import _lib, api
from mmdit_joint_attention_b200 import inputs as I
from helpers import device_inputs, from_dev, parity, q8_parity, q8_rel

pytestmark = pytest.mark.gpu


def _run(t, w):
    return api.joint_attention(t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"],
                               t["v_ctx"], t["ctx_len"] if w.ctx_len is not None else None)


def test_wait_timeout_is_reported_and_context_survives():
    w = I.WORKLOADS["block"]
    inp = I.make_inputs(w, parts=("qkv",))
    t = device_inputs(inp)
    L = _lib.lib()
    assert api.device_status() == 0
    try:
        L.mmdit_set_wait_timeout_ns(1)
        _run(t, w)
        status = api.device_status()
    finally:
        L.mmdit_set_wait_timeout_ns(0)
    assert status == _lib.STATUS_CODES["MMDIT_ERR_TIMEOUT"]
    assert api.device_status() == 0          # read-and-clear
    ov, oc = _run(t, w)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    rv, rc = oracle.joint_attention(inp["q_vis"].f64, inp["k_vis"].f64, inp["v_vis"].f64,
                                    inp["q_ctx"].f64, inp["k_ctx"].f64, inp["v_ctx"].f64)
    parity(from_dev(ov), rv, "bf16", "o_vis after a timed-out launch")
    parity(from_dev(oc), rc, "bf16", "o_ctx after a timed-out launch")


def test_backward_and_q8_wait_timeouts_are_reported():
    """The same for the backward kernels (both forms) and the 8-bit attention
    kernel: with the waits cut short each reports MMDIT_ERR_TIMEOUT, and the
    next call at the default limit is correct."""
    w = I.WORKLOADS["block"]
    inp = I.make_inputs(w, seed=3, parts=("qkv",))
    gin = I.make_grad_outputs(w, seed=3)
    t = device_inputs(inp)
    from helpers import to_dev
    do_vis, do_ctx = to_dev(gin["do_vis"]), to_dev(gin["do_ctx"])
    qkv = (t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"], t["v_ctx"])
    ov, oc, lse = api.joint_attention_fwd(*qkv)
    ws = api.bwd_workspace(w.B, w.Nv, w.Nc, w.H)
    torch.cuda.synchronize()
    L = _lib.lib()
    for call in ("bwd", "bwd_one_pass", "q8"):
        assert api.device_status() == 0
        try:
            L.mmdit_set_wait_timeout_ns(1)
            if call == "bwd":
                api.joint_attention_bwd(*qkv, ov, oc, do_vis, do_ctx, lse)
            elif call == "bwd_one_pass":
                api.joint_attention_bwd(*qkv, ov, oc, do_vis, do_ctx, lse, workspace=ws)
            else:
                api.joint_attention_8bit(*qkv)
            status = api.device_status()
        finally:
            L.mmdit_set_wait_timeout_ns(0)
        assert status == _lib.STATUS_CODES["MMDIT_ERR_TIMEOUT"], call
        assert api.device_status() == 0
    g = api.joint_attention_bwd(*qkv, ov, oc, do_vis, do_ctx, lse)
    g1 = api.joint_attention_bwd(*qkv, ov, oc, do_vis, do_ctx, lse, workspace=ws)
    q8v, q8c, _ = api.joint_attention_8bit(*qkv)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    ref = oracle.joint_attention_bwd(inp["q_vis"].f64, inp["k_vis"].f64, inp["v_vis"].f64,
                                     inp["q_ctx"].f64, inp["k_ctx"].f64, inp["v_ctx"].f64,
                                     gin["do_vis"].f64, gin["do_ctx"].f64)
    for k in ("dq_vis", "dk_vis", "dv_vis"):
        parity(from_dev(g[k]), ref[k], "bf16", f"{k} after a timed-out launch")
        parity(from_dev(g1[k]), ref[k], "bf16", f"one-pass {k} after a timed-out launch")
    a = [inp[k].f64 for k in ("q_vis", "k_vis", "v_vis", "q_ctx", "k_ctx", "v_ctx")]
    rel = q8_rel(a[0], a[1], a[3], a[4])
    rv, _, av, _ = oracle.attention_q8(*a, rel=rel)
    q8_parity(from_dev(q8v), rv, av, rel, "8-bit o_vis after a timed-out launch")
