"""Seeded synthetic inputs for the MMDiT joint-attention block.

This module is shared by the float64 oracle tests, the GPU parity tests and
the benchmark.  It holds none of the block's arithmetic: it only draws random
numbers (NumPy PCG64), rounds them to the storage type, and describes the
workload shapes.  Both sides of every parity check consume exactly the arrays
produced here.

Workload shapes follow the video-latent geometry of the Wan technical report
(section 4.1.1: a 4x8x8 VAE to 16 channels; section 4.2.1: a (1,2,2) patchify,
so a latent of T x H/8 x W/8 becomes T x H/16 x W/16 tokens) and the Vimoo 1.0
backbone (section 2.2: hidden width 3072, head dimension 128 split 16/56/56 over
T/H/W, RoPE on the visual stream only).  24 heads = 3072 / 128.

Value recipe (seed 0 unless stated):
  * q, k, v, x, branch ~ N(0, 1), drawn in fp32, rounded RNE to the dtype;
  * RMSNorm scales g ~ U(0.5, 1.5), one [D] vector per (stream, q/k), kept fp32;
  * adaLN shift / scale / gate ~ N(0, 0.1), one [B, C] array per stream, fp32.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Tuple

import numpy as np

HEAD_DIM = 128
ROPE_SPLIT = (16, 56, 56)
ROPE_BASE = 10000.0


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: sizes of both streams and the visual grid."""

    name: str
    dtype: str                 # "f32" or "bf16": storage and I/O type of q/k/v/x/o
    B: int
    H: int                     # heads
    grid: Tuple[int, int, int]  # (T, Hp, Wp) visual token grid
    Nc: int                    # padded conditioning length
    ctx_len: Optional[Tuple[int, ...]] = None  # valid cond tokens per sample (None: all Nc)
    pos_scale: Tuple[float, float, float] = (1.0, 1.0, 1.0)
    D: int = HEAD_DIM

    @property
    def Nv(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def C(self) -> int:
        return self.H * self.D

    def ctx_lengths(self) -> Tuple[int, ...]:
        return tuple(self.ctx_len) if self.ctx_len is not None else (self.Nc,) * self.B

    def attention_flops(self) -> float:
        """4 * Nq * Nk * D per (sample, head) over valid tokens.

        The factor 4 is the Wan report's non-causal forward attention cost
        (section 4.3.1, beta = 4): 2 for Q K^T and 2 for P V.  Padded cond query
        rows are not counted (their output is defined to be zero)."""
        total = 0.0
        for L in self.ctx_lengths():
            n = self.Nv + L
            total += 4.0 * n * n * self.D * self.H
        return total

    def with_batch(self, B: int, ctx_len=None) -> "Workload":
        return dataclasses.replace(self, B=B, ctx_len=ctx_len)


# The five workloads: tiny fp32 parity case; one 17-frame 128x128 block;
# 81-frame 480p; 81-frame 720p with per-axis position scaling; a batch of two
# 49-frame 480p samples with ragged conditioning lengths.  "medium" is a
# quarter of the 480p grid (81 frames of 240x416: 21x15x26 = 8190 visual
# tokens), the smallest case whose q, k and v (50 MB each) still exceed the
# L2 together: the size for profiler captures that replay a launch many times.
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", "f32", B=1, H=2, grid=(2, 4, 4), Nc=8),
    "block": Workload("block", "bf16", B=1, H=24, grid=(5, 8, 8), Nc=256),
    "480p": Workload("480p", "bf16", B=1, H=24, grid=(21, 30, 52), Nc=512),
    "720p": Workload("720p", "bf16", B=1, H=24, grid=(21, 45, 80), Nc=512,
                     pos_scale=(1.0, 1.0 / 1.5, 1.0 / 1.5)),
    "ragged": Workload("ragged", "bf16", B=2, H=24, grid=(13, 30, 52), Nc=320,
                       ctx_len=(77, 300)),
    "medium": Workload("medium", "bf16", B=1, H=24, grid=(21, 15, 26), Nc=512),
}


# ---------------------------------------------------------------------------
# storage-type rounding (IEEE round-to-nearest-even)
# ---------------------------------------------------------------------------

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bfloat16 (RNE) and return the 16-bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bfloat16 bit patterns as float64."""
    u = bits.astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    u = bits.astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


def round_f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values directly to the nearest bfloat16 (ties to even),
    returned as float64.  Used to express an exact result in the storage type
    of a bf16 output buffer (no double rounding through fp32)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.round(m * 256.0) / 256.0, e)   # 8 significant bits


def round_f64_to_f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# tensors
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Tensor:
    """A synthetic tensor: its storage (uint16 bf16 bits or float32) and its
    exact value as float64 (what the oracle consumes)."""

    storage: np.ndarray
    dtype: str

    @property
    def f64(self) -> np.ndarray:
        if self.dtype == "bf16":
            return bf16_bits_to_f64(self.storage)
        return self.storage.astype(np.float64)

    @property
    def shape(self):
        return self.storage.shape


def _draw_normal(rng: np.random.Generator, shape, dtype: str, std: float = 1.0) -> Tensor:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    if dtype == "bf16":
        return Tensor(f32_to_bf16_bits(a), "bf16")
    return Tensor(a, "f32")


def make_grad_outputs(w: Workload, seed: int = 0) -> Dict[str, Tensor]:
    """Upstream gradients do_vis [B,Nv,H,D] and do_ctx [B,Nc,H,D] of the
    attention outputs for a backward pass: N(0,1) in the workload's dtype,
    from their own PCG64 stream (seed + 1000)."""
    rng = np.random.Generator(np.random.PCG64(seed + 1000))
    return {"do_vis": _draw_normal(rng, (w.B, w.Nv, w.H, w.D), w.dtype),
            "do_ctx": _draw_normal(rng, (w.B, w.Nc, w.H, w.D), w.dtype)}


def make_inputs(w: Workload, seed: int = 0, parts=("qkv", "scales", "adaln")) -> Dict[str, object]:
    """Draw every input of one block pass for workload ``w``.

    Keys: q_vis k_vis v_vis [B,Nv,H,D]; q_ctx k_ctx v_ctx [B,Nc,H,D];
    gq_vis gk_vis gq_ctx gk_ctx [D] fp32; ctx_len int32 [B];
    x_vis [B,Nv,C], x_ctx [B,Nc,C]; shift/scale/gate _vis/_ctx [B,C] fp32.
    The draw order is fixed so that a given (workload, seed) always yields the
    same arrays; ``parts`` selects groups but does not change any group's values
    (each group has its own child generator)."""
    ss = np.random.SeedSequence(seed)
    g_qkv, g_scales, g_adaln = (np.random.Generator(np.random.PCG64(s)) for s in ss.spawn(3))
    B, Nv, Nc, H, D, C = w.B, w.Nv, w.Nc, w.H, w.D, w.C
    out: Dict[str, object] = {"workload": w,
                              "ctx_len": np.asarray(w.ctx_lengths(), dtype=np.int32)}
    if "qkv" in parts:
        for name in ("q", "k", "v"):
            out[name + "_vis"] = _draw_normal(g_qkv, (B, Nv, H, D), w.dtype)
            out[name + "_ctx"] = _draw_normal(g_qkv, (B, Nc, H, D), w.dtype)
    if "scales" in parts:
        for name in ("gq_vis", "gk_vis", "gq_ctx", "gk_ctx"):
            out[name] = g_scales.uniform(0.5, 1.5, size=D).astype(np.float32)
    if "adaln" in parts:
        out["x_vis"] = _draw_normal(g_adaln, (B, Nv, C), w.dtype)
        out["x_ctx"] = _draw_normal(g_adaln, (B, Nc, C), w.dtype)
        for s in ("vis", "ctx"):
            for name in ("shift", "scale", "gate"):
                a = g_adaln.standard_normal(size=(B, C), dtype=np.float32) * np.float32(0.1)
                out[f"{name}_{s}"] = a
    return out


def parity_rows(w: Workload, b: int, h: int, n_random: int = 512, seed: int = 1) -> np.ndarray:
    """Joint query-row indices (0..Nv+Nc-1) sampled for attention parity at
    sizes where the float64 oracle cannot compute every row.

    Every cond row; the first and last 128 visual rows; rows on both sides of
    each visual 128-row tile boundary near the visual tail and of the
    cond padding boundary; and ``n_random`` PCG64-drawn rows per (b, h)."""
    Nv, Nc = w.Nv, w.Nc
    L = w.ctx_lengths()[b]
    rows = set(range(Nv, Nv + Nc))
    rows.update(range(0, min(128, Nv)))
    rows.update(range(max(0, Nv - 128), Nv))
    last_full = (Nv // 128) * 128
    for r in (last_full - 1, last_full, last_full + 1, 127, 128, 129):
        if 0 <= r < Nv:
            rows.add(r)
    for r in (Nv + L - 1, Nv + L):
        if Nv <= r < Nv + Nc:
            rows.add(r)
    rng = np.random.Generator(np.random.PCG64([seed, b, h]))
    rows.update(int(r) for r in rng.integers(0, Nv + Nc, size=n_random))
    return np.asarray(sorted(rows), dtype=np.int64)
