"""The pair kernel (attention_pair.cu: CTA pairs sharing one MMA-issuing
thread, cta_group::2 products) against the one-SM kernel.

joint_attention without lse runs the pair kernel; joint_attention_fwd (with
lse) runs the one-SM kernel.  Both compute every tile's scores, softmax and
sums in the same order, so their outputs must agree bit for bit; the oracle
parity of the pair kernel itself is covered by every test that calls
joint_attention (tests/test_gpu_parity.py and others)."""
import dataclasses

import pytest
import torch

from mmdit_joint_attention_b200 import api
from mmdit_joint_attention_b200 import inputs as I
from helpers import device_inputs

pytestmark = pytest.mark.gpu

W = I.WORKLOADS
CASES = {
    "block": W["block"],
    "ragged": W["ragged"],
    "480p": W["480p"],
    "one_query_tile": dataclasses.replace(W["block"], H=2, grid=(1, 1, 100), Nc=20),
    "five_tiles_no_cond": dataclasses.replace(W["block"], H=3, grid=(1, 5, 120), Nc=0),
    "cond_all_masked_b3": dataclasses.replace(W["block"], B=3, H=2, grid=(1, 13, 20), Nc=200,
                                              ctx_len=(0, 1, 200)),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_pair_kernel_equals_one_sm_kernel(case):
    w = CASES[case]
    inp = I.make_inputs(w, seed=11, parts=("qkv",))
    t = device_inputs(inp)
    cl = t["ctx_len"] if w.ctx_len is not None else None
    args = (t["q_vis"], t["k_vis"], t["v_vis"], t["q_ctx"], t["k_ctx"], t["v_ctx"])
    ov, oc = api.joint_attention(*args, cl)
    rv, rc, _ = api.joint_attention_fwd(*args, cl)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    assert torch.equal(ov, rv), case
    assert torch.equal(oc, rc), case
