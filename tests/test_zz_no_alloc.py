"""mmdit_joint_attention_bwd_noalloc, the backward entry point for callers that
cannot allocate device memory (it uses a workspace built into the library
instead of one passed in), gives the gradients of mmdit_joint_attention_bwd.

Called through the C ABI twice in a row, because every call shares the
library's workspace and must not depend on what the previous call left in it.
Collected last (file name), so that a run that stops at the first failure has
run every other test before this one."""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

from mmdit_joint_attention_b200 import _lib, api
from mmdit_joint_attention_b200 import inputs as I
from helpers import device_inputs, to_dev

pytestmark = pytest.mark.gpu

KEYS = ("dq_vis", "dk_vis", "dv_vis", "dq_ctx", "dk_ctx", "dv_ctx")


def _noalloc():
    f = _lib.lib().mmdit_joint_attention_bwd_noalloc
    f.argtypes = [ctypes.c_void_p] * 18 + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_int,
                                                                ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def test_noalloc_backward_matches_the_workspace_entry_point():
    w = dataclasses.replace(I.WORKLOADS["block"], B=2, ctx_len=(200, 37))
    inp = I.make_inputs(w, seed=11, parts=("qkv",))
    gin = I.make_grad_outputs(w, seed=11)
    t = device_inputs(inp)
    do_vis, do_ctx = to_dev(gin["do_vis"]), to_dev(gin["do_ctx"])
    qkv = (t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"], t["v_ctx"])
    ov, oc, lse = api.joint_attention_fwd(*qkv, t["ctx_len"])
    ref = api.joint_attention_bwd(*qkv, ov, oc, do_vis, do_ctx, lse, t["ctx_len"])
    torch.cuda.synchronize()
    f = _noalloc()
    p = lambda x: ctypes.c_void_p(x.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = {k: torch.full_like(ref[k], float("nan")) for k in KEYS}
        st = f(*(p(x) for x in qkv), p(t["ctx_len"]), p(ov), p(oc), p(do_vis), p(do_ctx), p(lse),
               *(p(out[k]) for k in KEYS), w.B, w.Nv, w.Nc, w.H, w.D, 1.0 / np.sqrt(w.D),
               _lib.MMDIT_BF16, stream)
        assert st == 0, _lib.STATUS.get(st, st)
        torch.cuda.synchronize()
        assert api.device_status() == 0
        # the same kernels on the same inputs: bit for bit, so that a stale
        # value left in the built-in workspace cannot hide inside a tolerance
        for k in KEYS:
            assert torch.equal(out[k], ref[k]), f"call {call} {k} differs"
