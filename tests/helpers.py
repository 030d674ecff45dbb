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


# ---------------------------------------------------------------- 8-bit method vs exact
#
# The 8-bit joint attention (Int8 S = Q K^T, E4M3 O = P V) is not meant to
# equal the exact attention; its distance from it is set by three rounding
# steps, each bounded by the number format:
#   * the int8 codes of q and k move the score of key j (log2 units) by
#     delta_j, computed here exactly from the codes and scales;
#   * E4M3 keeps 3 mantissa bits: in the normal range the relative error of a
#     rounded value is at most 2^-4, a uniform error of standard deviation
#     2^-4 / sqrt(3) or less; below 2^-6 (subnormal) the absolute error is at
#     most 2^-10, standard deviation 2^-10 / sqrt(3) or less.  P' is rounded
#     (in units of P' itself), and so is v / scale_v (in units of scale_v).
# To first order the output error of element (i, d) is then a sum over keys of
# independent terms, with variance
#   sigma^2 = sum_j [ (w_j ln2 delta_j (v_jd - o_d))^2
#                     + (v_jd sigma_P'j / l)^2 + (w_j sigma_vjd)^2 ]
# (w the exact softmax weights, o the exact output, l the sum of P').  The
# check: |o8 - o| <= 6 sigma + 2^-8 |o| (the last term: the bf16 output) for
# every element, and the mean of |o8 - o| / sigma at most 0.8, what a Gaussian
# error of exactly the modelled size would give (the format bounds make sigma
# an overestimate: the method itself measures about 0.6, and an output scaled
# by 1.05 about 1.0).
Q8_SIGMAS = 6.0
Q8_MEAN_SIGMA = 0.8
_R = 2.0 ** -4 / np.sqrt(3.0)
_A = 2.0 ** -10 / np.sqrt(3.0)


def q8_rel(qv, kv, qc, kc, scale=None) -> float:
    """Relative bound on how far the 8-bit kernel's P' (before its E4M3
    rounding) can sit from the oracle's float64 P', for the oracle's
    rounding-ambiguity bound.  The kernel forms x = S c - m + 6 (log2 units,
    c = s_q s_k scale log2 e from three float32 roundings) as one float32 FMA of
    1.5 * 2^23 + S (exact) by c with the addend rounded from
    6 - m - 1.5 * 2^23 c, then P' = ex2.approx(x).  Against the exact x that
    leaves, in log2 units, at most 2^-24 (1.5 * 2^23 c + m + 6) from the addend,
    3 * 2^-24 (m + 12) from c over the keys in E4M3's normal range
    (|S c| <= m + 12) and 2^-24 * 16 from the FMA's result; ex2.approx adds a
    relative 2^-21.  c and m are bounded from the inputs: every quantisation
    scale is at most the tensor's max |x| / 127, and |S| <= 127^2 * 128.
    The bound is doubled."""
    D = np.shape(qv)[-1]
    if scale is None:
        scale = D ** -0.5
    amax = lambda *xs: max(float(np.abs(x).max()) if np.size(x) else 0.0 for x in xs)
    c = amax(qv, qc) / 127.0 * amax(kv, kc) / 127.0 * scale * np.log2(np.e)
    m = 127.0 * 127.0 * 128.0 * c + 1.0
    dx = 2.0 ** -24 * (1.5 * 2.0 ** 23 * c + m + 6.0 + 3.0 * (m + 12.0) + 16.0)
    return 2.0 * (np.log(2.0) * dx + 2.0 ** -21)


def q8_parity(got: np.ndarray, ref: np.ndarray, amb: np.ndarray, rel: float, name: str = ""):
    """The 8-bit kernel against the oracle's 8-bit method: the bf16 tolerance
    of parity(), plus the oracle's bound amb on rounding the P' that lie within
    rel of an E4M3 midpoint the other way, plus 2 rel of |o| (the row sum
    takes the kernel's P' unrounded)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite output"
    if got.size == 0:
        return {"max_err": 0.0}
    refr = I.round_f64_to_bf16(ref)
    err = np.abs(got - refr)
    scale = float(np.abs(refr).max())
    allowed = 1e-2 * max(scale, 1e-30) + amb + 2.0 * rel * np.abs(ref)
    rep = {"max_err": float(err.max()), "max_ref": scale, "max_amb": float(amb.max()),
           "elements_past_bf16_tol": int((err > 1e-2 * max(scale, 1e-30)).sum())}
    assert np.all(err <= allowed), (name, rep)
    return rep


def q8_exact_rows(qv, kv, vv, qc, kc, vc, ctx_len, trip, scale=None, chunk=128):
    """Exact attention rows and the 8-bit method's error sigma at the query
    rows ``trip`` [(b, h, i)]: returns (o [R, D], sigma [R, D]), float64."""
    import oracle
    qv, kv, vv, qc, kc, vc = (np.asarray(a, np.float64) for a in (qv, kv, vv, qc, kc, vc))
    B, Nv, H, D = qv.shape
    Nc = qc.shape[1]
    scale = D ** -0.5 if scale is None else scale
    cl = np.full(B, Nc, np.int32) if ctx_len is None else np.asarray(ctx_len, np.int32)
    trip = np.asarray(trip, np.int64)
    o = np.zeros((len(trip), D))
    sig = np.zeros((len(trip), D))
    c2 = scale / np.log(2.0)                       # scores in log2 units
    _, _, sv = oracle.quant_v_e4m3(vv, vc, cl)     # [B, H, D]
    for (b, h) in sorted({(int(t[0]), int(t[1])) for t in trip}):
        L = int(cl[b])
        sel = np.nonzero((trip[:, 0] == b) & (trip[:, 1] == h))[0]
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
        qvc, sqv = oracle.quant_int8(qv[sl], 1)
        qcc, sqc = oracle.quant_int8(qc[sl], 1)
        kvc, skv = oracle.quant_int8(kv[sl], 128)
        kcc, skc = oracle.quant_int8(kc[sl], 128)
        K = np.concatenate([kv[b, :, h], kc[b, :L, h]])
        V = np.concatenate([vv[b, :, h], vc[b, :L, h]])
        Kq = np.concatenate([kvc[0, :, 0] * np.repeat(skv[0, 0], 128)[:Nv, None],
                             kcc[0, :L, 0] * np.repeat(skc[0, 0], 128)[:L, None]])
        s = sv[b, h].astype(np.float64)
        with np.errstate(divide="ignore", invalid="ignore"):
            vn = np.where(s > 0, np.abs(V) / np.where(s > 0, s, 1.0), 0.0)
        sig_v = np.where(vn >= 2.0 ** -6, _R * np.abs(V), _A * s)        # [Nk, D]
        V2, SV2 = V * V, sig_v * sig_v
        for c0 in range(0, len(sel), chunk):
            rows = sel[c0:c0 + chunk]
            ii = trip[rows, 2]
            ok = ii < Nv + L
            ii = np.where(ok, ii, 0)
            Q = np.where((ii < Nv)[:, None], qv[b, np.minimum(ii, Nv - 1), h],
                         qc[b, np.clip(ii - Nv, 0, max(Nc - 1, 0)), h] if Nc else 0.0)
            Qq = np.where((ii < Nv)[:, None],
                          qvc[0, np.minimum(ii, Nv - 1), 0] * sqv[0, 0, np.minimum(ii, Nv - 1)][:, None],
                          (qcc[0, np.clip(ii - Nv, 0, max(Nc - 1, 0)), 0] *
                           sqc[0, 0, np.clip(ii - Nv, 0, max(Nc - 1, 0))][:, None]) if Nc else 0.0)
            S = (Q @ K.T) * c2
            Sq = (Qq @ Kq.T) * c2
            p = np.exp2(S - S.max(axis=1, keepdims=True))
            w = p / p.sum(axis=1, keepdims=True)
            orow = w @ V
            pq = np.exp2(Sq - np.ceil(Sq.max(axis=1, keepdims=True)) + 6.0)
            lq = pq.sum(axis=1, keepdims=True)
            sig_p = np.where(pq >= 2.0 ** -6, _R * pq, _A) / lq
            a = (w * np.log(2.0) * (Sq - S)) ** 2
            var = (a @ V2 - 2.0 * orow * (a @ V) + orow ** 2 * a.sum(axis=1, keepdims=True)
                   + (sig_p ** 2) @ V2 + (w ** 2) @ SV2)
            o[rows] = np.where(ok[:, None], orow, 0.0)
            sig[rows] = np.where(ok[:, None], np.sqrt(np.maximum(var, 0.0)), 0.0)
    return o, sig


def q8_close_to_exact(got, o, sig, name=""):
    """The 8-bit output ``got`` [R, D] against the exact rows ``o`` with the
    error model's ``sig`` (q8_exact_rows); returns a report."""
    got = np.asarray(got, np.float64)
    err = np.abs(got - o)
    tol = Q8_SIGMAS * sig + 2.0 ** -8 * np.abs(o)
    live = sig > 0
    ratio = err[live] / sig[live]
    rep = {"max_err": float(err.max()), "max_ref": float(np.abs(o).max()),
           "max_err_over_sigma": float(ratio.max()) if ratio.size else 0.0,
           "mean_err_over_sigma": float(ratio.mean()) if ratio.size else 0.0}
    assert np.all(np.isfinite(got)), f"{name}: non-finite output"
    assert np.all(err <= tol + 1e-300), (name, rep)    # rows without output: exactly 0
    assert rep["mean_err_over_sigma"] <= Q8_MEAN_SIGMA, (name, rep)
    return rep
