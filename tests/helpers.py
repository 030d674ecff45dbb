"""Shared test helpers: device transfer of synthetic inputs and the parity
criterion.

Parity criterion (the tolerances stated for this path):
  * fp32 outputs: max |gpu - exact| <= 1e-4, exact = float64 oracle result;
  * bf16 outputs: the reference is the float64 oracle result rounded (RNE) to
    bf16, the storage type of the output buffer, i.e. the best answer a bf16
    buffer can hold; then max |gpu - ref| <= 1e-2 * max |ref| and
    mean |gpu - ref| <= 1e-3 per output tensor.
"""
import numpy as np
import torch

from mmdit_joint_attention_b200 import inputs as I


def to_dev(t) -> torch.Tensor:
    if isinstance(t, I.Tensor):
        if t.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(t.storage).view(np.int16)).view(
                torch.bfloat16).cuda()
        return torch.from_numpy(np.ascontiguousarray(t.storage)).cuda()
    a = np.ascontiguousarray(t)
    if a.dtype == np.float64:
        a = a.astype(np.float32)
    return torch.from_numpy(a).cuda()


def from_dev(x: torch.Tensor) -> np.ndarray:
    return x.detach().float().cpu().numpy().astype(np.float64)


def device_inputs(inp: dict) -> dict:
    out = {}
    for k, v in inp.items():
        if k == "workload":
            continue
        out[k] = to_dev(v)
    return out


def parity(got: np.ndarray, ref: np.ndarray, dtype: str, name: str = "") -> dict:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite output"
    if got.size == 0:
        return {"max_err": 0.0}
    if dtype == "f32":
        err = np.abs(got - ref)
        rep = {"max_err": float(err.max()), "mean_err": float(err.mean()),
               "max_ref": float(np.abs(ref).max())}
        assert rep["max_err"] <= 1e-4, (name, rep)
        return rep
    refr = I.round_f64_to_bf16(ref)
    err = np.abs(got - refr)
    scale = float(np.abs(refr).max())
    rep = {"max_err": float(err.max()), "mean_err": float(err.mean()), "max_ref": scale,
           "max_err_vs_exact": float(np.abs(got - ref).max())}
    assert rep["max_err"] <= 1e-2 * max(scale, 1e-30), (name, rep)
    assert rep["mean_err"] <= 1e-3, (name, rep)
    return rep
