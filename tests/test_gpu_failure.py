"""Failure detection on the GPU without a fault: every wait in the attention
kernel is bounded; when one runs out the kernel drains, frees its tensor
memory, returns, and the status word reports MMDIT_ERR_TIMEOUT.  The test
shortens the wait limit so that the waits of an ordinary launch run out, then
checks the status, and that the context is healthy afterwards."""
import pytest
import torch

import oracle
from mmdit_joint_attention_b200 import _lib, api
from mmdit_joint_attention_b200 import inputs as I
from helpers import device_inputs, from_dev, parity

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
