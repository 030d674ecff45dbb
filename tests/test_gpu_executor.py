"""mmdit_block_forward_host, the host-buffer executor: several steps from and
to host buffers, pipelined over the library's own streams and a workspace of
one or more slots.  Each step's outputs must equal, bit for bit, the same
six calls run on device buffers (api.block_forward), and match the
oracle's whole-path result within the stated tolerances."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from mmdit_joint_attention_b200 import api
from mmdit_joint_attention_b200 import inputs as I
from helpers import device_inputs, parity, to_dev

pytestmark = pytest.mark.gpu

IN = ("q_vis", "k_vis", "v_vis", "q_ctx", "k_ctx", "v_ctx", "x_vis", "x_ctx", "shift_vis",
      "scale_vis", "gate_vis", "shift_ctx", "scale_ctx", "gate_ctx")
SCALES = ("gq_vis", "gk_vis", "gq_ctx", "gk_ctx")


def _host(v, pin: bool) -> torch.Tensor:
    if isinstance(v, I.Tensor):
        a = np.ascontiguousarray(v.storage)
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if v.dtype == "bf16" \
            else torch.from_numpy(a)
    else:
        t = torch.from_numpy(np.ascontiguousarray(v))
    t = t.clone()
    return t.pin_memory() if pin else t


def _steps(w, seeds):
    """Inputs of one step per seed; every step shares the first one's RMSNorm
    scales (model weights, fixed for the executor's lifetime)."""
    inps = [I.make_inputs(w, seed=s) for s in seeds]
    for inp in inps[1:]:
        for k in SCALES:
            inp[k] = inps[0][k]
    return inps


def _executor(w, inp0, slots):
    g = [to_dev(inp0[k]) for k in SCALES]
    return api.BlockHostExecutor(w.B, w.Nv, w.Nc, w.H, w.grid, *g, pos_scale=w.pos_scale,
                                 dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32,
                                 slots=slots), g


def _host_step(inp, pin=True, outputs=("y", "o", "x_out")):
    st = {k: _host(inp[k], pin) for k in IN}
    if inp["ctx_len"] is not None:
        st["ctx_len"] = _host(inp["ctx_len"].astype(np.int32), pin)
    for s in ("vis", "ctx"):
        for o in outputs:
            src = "x_" + s if o in ("y", "x_out") else "q_" + s
            st[f"{o}_{s}"] = torch.empty_like(st[src])
            if pin:
                st[f"{o}_{s}"] = st[f"{o}_{s}"].pin_memory()
    return st


def _device_reference(w, inp):
    t = device_inputs(inp)
    out = api.block_forward(t, grid=w.grid, pos_scale=w.pos_scale)
    torch.cuda.synchronize()
    return {k: v.cpu() for k, v in out.items()}


def _bits(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@pytest.mark.parametrize("slots", [1, 2, 3])
def test_executor_equals_device_path_bit_for_bit(slots):
    w = dataclasses.replace(I.WORKLOADS["block"], B=2, ctx_len=(200, 37))
    inps = _steps(w, seeds=[21, 22, 23, 24, 25])
    ex, _ = _executor(w, inps[0], slots)
    steps = [_host_step(inp) for inp in inps]
    ex.run(steps)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    for i, inp in enumerate(inps):
        ref = _device_reference(w, inp)
        for s in ("vis", "ctx"):
            for got, want in ((f"y_{s}", f"y_{s}"), (f"o_{s}", f"o_{s}"), (f"x_out_{s}", f"x_{s}")):
                g = steps[i][got].reshape(ref[want].shape)
                assert torch.equal(_bits(g), _bits(ref[want])), (slots, i, got)


@pytest.mark.parametrize("name", ["tiny", "block"])
def test_executor_matches_oracle(name):
    w = I.WORKLOADS[name]
    inps = _steps(w, seeds=[3, 4])
    ex, _ = _executor(w, inps[0], slots=2)
    steps = [_host_step(inp) for inp in inps]
    ex.run(steps)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    for i, inp in enumerate(inps):
        ref = oracle.block(inp)
        for s in ("vis", "ctx"):
            for got, want in ((f"y_{s}", f"y_{s}"), (f"o_{s}", f"o_{s}"), (f"x_out_{s}", f"x_{s}")):
                g = steps[i][got].float().numpy().astype(np.float64).reshape(ref[want].shape)
                parity(g, ref[want], w.dtype, f"{name} step {i} {got}")


def test_executor_pageable_memory_and_skipped_outputs():
    """Pageable host buffers give the same results (without the overlap); y and
    o left out are not copied back; one shared output set for all steps holds
    the last step's values, since the output copies run in step order."""
    w = dataclasses.replace(I.WORKLOADS["block"], ctx_len=(99,))
    inps = _steps(w, seeds=[7, 8, 9])
    ex, _ = _executor(w, inps[0], slots=3)
    shared = _host_step(inps[0], pin=False, outputs=("x_out",))
    steps = []
    for inp in inps:
        st = _host_step(inp, pin=False, outputs=())
        st["x_out_vis"], st["x_out_ctx"] = shared["x_out_vis"], shared["x_out_ctx"]
        steps.append(st)
    ex.run(steps)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    ref = _device_reference(w, inps[-1])
    for s in ("vis", "ctx"):
        assert torch.equal(_bits(shared[f"x_out_{s}"].reshape(ref[f"x_{s}"].shape)),
                           _bits(ref[f"x_{s}"])), s


def test_executor_orders_against_the_callers_stream():
    """Work queued on the caller's stream before the call finishes before the
    executor reads its inputs, and work queued after waits for its outputs."""
    w = I.WORKLOADS["block"]
    inps = _steps(w, seeds=[31])
    ex, _ = _executor(w, inps[0], slots=1)
    st = _host_step(inps[0])
    s = torch.cuda.Stream()
    ws_probe = torch.empty(ex.workspace.numel(), dtype=torch.uint8, device="cuda")
    with torch.cuda.stream(s):
        # a long copy into the workspace ahead of the call: the executor's input
        # copies must not start before it ends, or they would be overwritten
        for _ in range(4):
            ex.workspace.copy_(ws_probe)
        ex.run([st], stream=s)
    s.synchronize()
    ref = _device_reference(w, inps[0])
    for k in ("y_vis", "o_vis", "x_out_vis"):
        want = ref[k.replace("x_out", "x")]
        assert torch.equal(_bits(st[k].reshape(want.shape)), _bits(want)), k
