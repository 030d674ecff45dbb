"""Seeded input generator: determinism, shapes and storage rounding."""
import numpy as np
import torch

from mmdit_joint_attention_b200 import inputs as I


def test_bf16_rounding_matches_torch_rne():
    a = np.random.Generator(np.random.PCG64(0)).standard_normal(100_000).astype(np.float32)
    a[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0]      # ties to even both ways
    ours = I.f32_to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(I.bf16_bits_to_f32(ours), torch.from_numpy(a).to(torch.bfloat16).float().numpy())


def test_round_f64_to_bf16():
    x = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -40, -3.0, 0.0, 1e-3])
    want = np.array([1.0, 1.0 + 2 ** -6, 1.0 + 2 ** -7, -3.0, 0.0,
                     float(torch.tensor(1e-3, dtype=torch.float64).to(torch.bfloat16).double())])
    assert np.array_equal(I.round_f64_to_bf16(x), want)


def test_workload_sizes():
    W = I.WORKLOADS
    assert W["tiny"].Nv == 32 and W["tiny"].C == 256
    assert W["block"].Nv == 320
    assert W["480p"].Nv == 32760 and W["480p"].C == 3072
    assert W["720p"].Nv == 75600
    assert W["ragged"].Nv == 20280 and W["ragged"].ctx_lengths() == (77, 300)
    assert abs(W["480p"].attention_flops() - 13.60e12) < 0.01e12
    assert abs(W["720p"].attention_flops() - 71.18e12) < 0.01e12
    assert abs(W["ragged"].attention_flops() - 10.30e12) < 0.01e12
    assert W["medium"].Nv == 8190 and W["medium"].Nv * W["medium"].C * 2 * 3 > 126e6


def test_make_inputs_deterministic_and_shaped():
    w = I.WORKLOADS["block"]
    a = I.make_inputs(w, seed=0)
    b = I.make_inputs(w, seed=0)
    c = I.make_inputs(w, seed=0, parts=("adaln",))
    assert a["q_vis"].shape == (1, 320, 24, 128) and a["q_vis"].storage.dtype == np.uint16
    assert a["x_ctx"].shape == (1, 256, 3072)
    assert np.array_equal(a["k_ctx"].storage, b["k_ctx"].storage)
    assert np.array_equal(a["x_vis"].storage, c["x_vis"].storage)
    assert a["gq_vis"].dtype == np.float32 and 0.5 <= a["gq_vis"].min() and a["gq_vis"].max() <= 1.5
    t = I.make_inputs(I.WORKLOADS["tiny"])
    assert t["q_vis"].storage.dtype == np.float32


def test_parity_rows_cover_boundaries():
    w = I.WORKLOADS["ragged"]
    rows = I.parity_rows(w, 1, 3)
    Nv = w.Nv
    assert set(range(Nv, Nv + w.Nc)) <= set(rows.tolist())
    for r in (0, 127, 128, Nv - 1, (Nv // 128) * 128, Nv + 299, Nv + 300):
        assert r in rows
    assert rows.min() >= 0 and rows.max() < Nv + w.Nc


def test_grad_outputs_deterministic_and_independent():
    w = I.WORKLOADS["block"]
    a = I.make_grad_outputs(w, seed=4)
    b = I.make_grad_outputs(w, seed=4)
    assert np.array_equal(a["do_vis"].storage, b["do_vis"].storage)
    assert a["do_vis"].shape == (w.B, w.Nv, w.H, w.D) and a["do_ctx"].shape == (w.B, w.Nc, w.H, w.D)
    q = I.make_inputs(w, seed=4, parts=("qkv",))["q_vis"]
    assert not np.array_equal(a["do_vis"].storage, q.storage)   # its own random stream
