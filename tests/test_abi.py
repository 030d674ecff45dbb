"""The C-ABI library loads on a CPU host, exports every symbol the header
declares, and rejects bad arguments on the host before touching a GPU."""
import ctypes

import pytest

from mmdit_joint_attention_b200 import _lib


@pytest.fixture(scope="module")
def L():
    from mmdit_joint_attention_b200 import build
    build.build()
    return _lib.lib()


def test_exports_every_declared_symbol(L):
    names = _lib.declared_functions()
    assert set(names) >= {"mmdit_qk_norm_rope", "mmdit_joint_attention", "mmdit_adaln_modulate",
                          "mmdit_gated_residual", "mmdit_residual_modulate",
                          "mmdit_status_string", "mmdit_device_status", "mmdit_last_error"}
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code in _lib.STATUS:
        assert L.mmdit_status_string(code)
    assert L.mmdit_status_string(-99) == b"unknown status"


P = ctypes.c_void_p(16)   # aligned, never dereferenced: validation fails first
U = ctypes.c_void_p(18)   # misaligned


def test_qk_norm_rope_validation(L):
    f = L.mmdit_qk_norm_rope
    g = _lib.Grid(2, 4, 4, (ctypes.c_float * 3)(1, 1, 1), 10000.0, (ctypes.c_int * 3)(16, 56, 56))
    assert f(P, P, P, P, P, P, 1, 32, 2, 64, ctypes.byref(g), 1e-6, 1, None) == -4  # D != 128
    assert f(P, P, P, P, P, P, 1, 32, 2, 128, ctypes.byref(g), 1e-6, 7, None) == -1  # dtype
    assert f(None, P, P, P, P, P, 1, 32, 2, 128, ctypes.byref(g), 1e-6, 1, None) == -1
    assert f(U, P, P, P, P, P, 1, 32, 2, 128, ctypes.byref(g), 1e-6, 1, None) == -3
    assert f(P, P, P, P, P, P, 1, 31, 2, 128, ctypes.byref(g), 1e-6, 1, None) == -2  # N != THW
    g.split[1] = 58
    assert f(P, P, P, P, P, P, 1, 32, 2, 128, ctypes.byref(g), 1e-6, 1, None) == -2  # sum != D
    g.split[0], g.split[1] = 12, 60
    assert f(P, P, P, P, P, P, 1, 32, 2, 128, ctypes.byref(g), 1e-6, 1, None) == -4  # bf16 chunk
    assert f(P, P, P, P, P, P, 1, 32, 2, 128, None, -1.0, 1, None) == -1  # eps
    assert f(None, None, None, None, None, None, 0, 32, 2, 128, None, 1e-6, 1, None) == 0  # empty


def test_attention_validation(L):
    f = L.mmdit_joint_attention
    assert f(P, P, P, P, P, P, None, P, P, 1, 8, 8, 2, 64, 0.1, 1, None) == -4
    assert f(P, P, P, P, P, P, None, P, P, 1, 8, 8, 2, 128, 0.0, 1, None) == -1
    assert f(P, P, P, P, P, P, None, P, P, 1, 8, 8, 2, 128, float("nan"), 1, None) == -1
    assert f(P, P, P, None, P, P, None, P, P, 1, 8, 8, 2, 128, 0.1, 1, None) == -1
    assert f(P, P, P, P, P, P, None, U, P, 1, 8, 8, 2, 128, 0.1, 1, None) == -3
    assert f(P, P, P, P, P, P, ctypes.c_void_p(18), P, P, 1, 8, 8, 2, 128, 0.1, 1, None) == -3
    assert f(P, P, P, P, P, P, None, P, P, 1, -1, 8, 2, 128, 0.1, 1, None) == -1
    assert f(None, None, None, None, None, None, None, None, None, 0, 8, 8, 2, 128, 0.1, 1, None) == 0


def test_modulate_residual_validation(L):
    m = L.mmdit_adaln_modulate
    r = L.mmdit_gated_residual
    assert m(P, P, P, P, 1, 4, 3070, 1e-6, 1, None) == -4
    assert m(P, P, P, P, 1, 4, 8192, 1e-6, 1, None) == -4      # above the register budget
    assert m(P, None, P, P, 1, 4, 3072, 1e-6, 1, None) == -1
    assert m(P, P, U, P, 1, 4, 3072, 1e-6, 1, None) == -3
    assert r(P, P, P, P, 1, 4, 3068, 1, None) == -4
    assert r(P, P, None, P, 1, 4, 3072, 1, None) == -1
    assert r(P, P, P, U, 1, 4, 3072, 1, None) == -3
    assert r(P, P, P, P, 1, 0, 3072, 1, None) == 0
    # both streams in one launch: x, shift, scale, y, N for each stream, then B, C
    mp = L.mmdit_adaln_modulate_pair
    assert mp(P, P, P, P, 4, P, P, P, P, 2, 1, 3070, 1e-6, 1, None) == -4    # C % 8
    assert mp(P, P, P, P, 4, P, P, P, P, 2, 1, 8192, 1e-6, 1, None) == -4    # register budget
    assert mp(P, P, P, P, -1, P, P, P, P, 2, 1, 3072, 1e-6, 1, None) == -1   # N_vis < 0
    assert mp(P, P, P, P, 4, P, P, P, P, -2, 1, 3072, 1e-6, 1, None) == -1   # N_ctx < 0
    assert mp(P, P, P, P, 4, P, P, P, P, 2, 1, 3072, -1.0, 1, None) == -1    # eps
    assert mp(P, P, P, P, 4, P, P, P, P, 2, 1, 3072, 1e-6, 7, None) == -1    # dtype
    assert mp(P, P, P, P, 4, P, None, P, P, 2, 1, 3072, 1e-6, 1, None) == -1  # ctx shift
    assert mp(P, P, P, U, 4, P, P, P, P, 2, 1, 3072, 1e-6, 1, None) == -3    # y_vis unaligned
    assert mp(P, P, P, P, 4, U, P, P, P, 2, 1, 3072, 1e-6, 1, None) == -3    # x_ctx unaligned
    assert mp(None, None, None, None, 0, None, None, None, None, 0, 1, 3072, 1e-6, 1,
              None) == 0                                                      # both empty
    assert mp(P, P, P, P, 4, P, P, P, P, 2, 0, 3072, 1e-6, 1, None) == 0     # B = 0


def test_residual_modulate_validation(L):
    f = L.mmdit_residual_modulate
    Q = ctypes.c_void_p(32)
    assert f(P, P, P, P, P, P, Q, 1, 4, 4096, 1e-6, 1, None) == -4     # above 3072 for bf16
    assert f(P, P, P, P, P, P, Q, 1, 4, 3070, 1e-6, 1, None) == -4
    assert f(P, P, P, P, P, P, P, 1, 4, 3072, 1e-6, 1, None) == -1     # y aliases x
    assert f(P, None, P, P, P, P, Q, 1, 4, 3072, 1e-6, 1, None) == -1
    assert f(P, P, P, U, P, P, Q, 1, 4, 3072, 1e-6, 1, None) == -3
    assert f(P, P, P, P, P, P, Q, 1, 0, 3072, 1e-6, 1, None) == 0


def test_qk_norm_rope_text_validation(L):
    f = L.mmdit_qk_norm_rope_text
    r = _lib.TextRope(3.0, 10000.0, (ctypes.c_int * 3)(16, 56, 56))
    assert f(P, P, P, P, P, P, 1, 8, 2, 128, None, 1e-6, 1, None) == -1          # no rope
    assert f(P, P, P, P, P, P, 1, 8, 2, 64, ctypes.byref(r), 1e-6, 1, None) == -4
    r.split[1] = 58
    assert f(P, P, P, P, P, P, 1, 8, 2, 128, ctypes.byref(r), 1e-6, 1, None) == -2
    r.split[0], r.split[1] = 12, 60
    assert f(P, P, P, P, P, P, 1, 8, 2, 128, ctypes.byref(r), 1e-6, 1, None) == -4
    r.split[0], r.split[1] = 16, 56
    r.pos_offset = float("inf")
    assert f(P, P, P, P, P, P, 1, 8, 2, 128, ctypes.byref(r), 1e-6, 1, None) == -1
    assert f(U, P, P, P, P, P, 1, 8, 2, 128, ctypes.byref(r), 1e-6, 1, None) == -3


def test_window_validation(L):
    g = _lib.Grid(5, 8, 8, (ctypes.c_float * 3)(1, 1, 1), 10000.0, (ctypes.c_int * 3)(16, 56, 56))
    w = _lib.Window((ctypes.c_int * 3)(1, 2, 2))
    R = ctypes.byref
    f = L.mmdit_joint_window_attention
    Q = ctypes.c_void_p(1 << 20)
    assert f(P, P, P, P, P, P, None, Q, Q, 1, 320, 8, 2, 128, None, R(w), 0.1, 1, None) == -1
    assert f(P, P, P, P, P, P, None, Q, Q, 1, 321, 8, 2, 128, R(g), R(w), 0.1, 1, None) == -2
    for bad in ((0, 1, 1), (6, 1, 1), (1, 9, 1), (1, 1, -1)):
        wb = _lib.Window((ctypes.c_int * 3)(*bad))
        assert f(P, P, P, P, P, P, None, Q, Q, 1, 320, 8, 2, 128, R(g), R(wb), 0.1, 1, None) == -2
    many = _lib.Window((ctypes.c_int * 3)(5, 8, 2))   # 80 windows > 64
    assert f(P, P, P, P, P, P, None, Q, Q, 1, 320, 8, 2, 128, R(g), R(many), 0.1, 1, None) == -4
    assert f(P, P, P, P, P, P, None, Q, Q, 1, 320, 8, 2, 64, R(g), R(w), 0.1, 1, None) == -4
    assert f(P, P, P, P, P, P, None, U, Q, 1, 320, 8, 2, 128, R(g), R(w), 0.1, 1, None) == -3

    # forward with lse: lse required, 4-byte aligned
    ff = L.mmdit_joint_window_attention_fwd
    assert ff(P, P, P, P, P, P, None, Q, Q, None, 1, 320, 8, 2, 128, R(g), R(w), 0.1, 1,
              None) == -1
    assert ff(P, P, P, P, P, P, None, Q, Q, ctypes.c_void_p(4098), 1, 320, 8, 2, 128, R(g),
              R(w), 0.1, 1, None) == -3
    assert ff(P, P, P, P, P, P, None, Q, Q, P, 1, 321, 8, 2, 128, R(g), R(w), 0.1, 1, None) == -2
    assert ff(P, P, P, P, P, P, None, Q, Q, P, 1, 320, 8, 2, 128, None, R(w), 0.1, 1, None) == -1
    # backward: the window checks first, then those of the joint backward
    fb = L.mmdit_joint_window_attention_bwd
    args = [P] * 6 + [None] + [P] * 12

    def bwd(*rest):
        return fb(*args, *rest)
    assert bwd(1, 320, 8, 2, 128, None, R(w), 0.1, 1, None) == -1
    assert bwd(1, 321, 8, 2, 128, R(g), R(w), 0.1, 1, None) == -2
    assert bwd(1, 320, 8, 2, 128, R(g), R(many), 0.1, 1, None) == -4
    assert bwd(1, 320, 8, 2, 64, R(g), R(w), 0.1, 1, None) == -4
    assert bwd(1, 320, 8, 2, 128, R(g), R(w), -0.1, 1, None) == -1
    bad = [P] * 6 + [None] + [P] * 4 + [None] + [P] * 7                      # lse NULL
    assert fb(*bad, 1, 320, 8, 2, 128, R(g), R(w), 0.1, 1, None) == -1

    p = L.mmdit_window_permute
    assert p(P, Q, 1, 320, 250, R(g), R(w), 0, 1, None) == -4     # 500-byte rows
    assert p(P, Q, 1, 321, 256, R(g), R(w), 0, 1, None) == -2
    assert p(P, P, 1, 320, 256, R(g), R(w), 0, 1, None) == -1     # y overlaps x
    assert p(U, Q, 1, 320, 256, R(g), R(w), 0, 1, None) == -3
    assert p(P, Q, 1, 320, 256, None, R(w), 0, 1, None) == -1
    assert p(None, None, 0, 320, 256, R(g), R(w), 0, 1, None) == 0   # empty batch

    q = L.mmdit_qk_norm_rope_window
    Q2 = ctypes.c_void_p(1 << 24)
    assert q(P, P, P, Q2, P, P, 1, 320, 2, 128, R(g), R(w), 1e-6, 1, None) == -1   # q_out == q_in
    assert q(P, Q, Q2, ctypes.c_void_p((1 << 24) + 16), P, P, 1, 320, 2, 128, R(g), R(w), 1e-6, 1,
             None) == -1                                                              # outputs overlap
    assert q(P, P, Q, Q2, P, P, 1, 320, 2, 128, None, R(w), 1e-6, 1, None) == -1
    assert q(P, P, Q, Q2, P, P, 1, 320, 2, 128, R(g), None, 1e-6, 1, None) == -1
    assert q(P, P, Q, Q2, P, P, 1, 321, 2, 128, R(g), R(w), 1e-6, 1, None) == -2


def test_backward_validation(L):
    f = L.mmdit_joint_attention_bwd
    Q = ctypes.c_void_p(1 << 20)
    ptrs = [P] * 6 + [None] + [P] * 4 + [Q, Q] + [P] * 6       # q..v, ctx_len, o, do, lse, delta, grads
    bad = list(ptrs)
    bad[11] = None                                             # lse missing
    assert f(*bad, 1, 8, 8, 2, 128, 0.1, 1, None) == -1
    bad = list(ptrs)
    bad[12] = ctypes.c_void_p((1 << 20) + 2)                   # delta misaligned
    assert f(*bad, 1, 8, 8, 2, 128, 0.1, 1, None) == -3
    bad = list(ptrs)
    bad[13] = U                                                # dq_vis misaligned
    assert f(*bad, 1, 8, 8, 2, 128, 0.1, 1, None) == -3
    assert f(*ptrs, 1, 8, 8, 2, 64, 0.1, 1, None) == -4         # D != 128
    assert f(*ptrs, 1, 8, 8, 2, 128, 0.0, 1, None) == -1        # scale
    assert f(*([None] * 19), 0, 8, 8, 2, 128, 0.1, 1, None) == 0  # empty
    g = L.mmdit_joint_attention_fwd
    assert g(P, P, P, P, P, P, None, P, P, None, 1, 8, 8, 2, 128, 0.1, 1, None) == -1  # no lse
    assert g(P, P, P, P, P, P, None, P, P, ctypes.c_void_p(18), 1, 8, 8, 2, 128, 0.1, 1,
             None) == -3


def test_noalloc_backward_rejects_sizes_beyond_its_workspace(L):
    f = L.mmdit_joint_attention_bwd_noalloc
    f.restype = ctypes.c_int
    rows = (1 << 22) // 24 + 1            # B = 1, H = 24: one row too many
    args = [P] * 6 + [None] + [P] * 5 + [P] * 6
    assert f(*args, 1, rows, 0, 24, 128, ctypes.c_float(0.1), 1, None) == -4
    assert f(*([None] * 18), 0, 8, 8, 2, 128, ctypes.c_float(0.1), 1, None) == 0


def test_qk_norm_rope_bwd_validation(L):
    f = L.mmdit_qk_norm_rope_bwd
    g = _lib.Grid(2, 4, 4, (ctypes.c_float * 3)(1, 1, 1), 10000.0, (ctypes.c_int * 3)(16, 56, 56))
    R = ctypes.byref
    assert f(P, P, P, P, P, P, P, P, P, P, 1, 32, 2, 64, R(g), 1e-6, 1, None) == -4   # D
    assert f(P, P, P, P, P, P, P, P, None, P, 1, 32, 2, 128, R(g), 1e-6, 1, None) == -1
    assert f(P, P, P, P, P, P, U, P, P, P, 1, 32, 2, 128, R(g), 1e-6, 1, None) == -3
    assert f(P, P, P, P, P, P, P, P, P, P, 1, 31, 2, 128, R(g), 1e-6, 1, None) == -2  # N != THW
    assert f(P, P, P, P, P, P, P, P, P, P, 1, 32, 2, 128, R(g), -1.0, 1, None) == -1  # eps


def _block_cfg(B=1, Nv=32, Nc=8, H=2, dt=1):
    c = _lib.BlockConfig()
    c.B, c.Nv, c.Nc, c.H, c.D = B, Nv, Nc, H, 128
    c.grid = _lib.Grid(2, 4, 4, (ctypes.c_float * 3)(1, 1, 1), 10000.0,
                       (ctypes.c_int * 3)(16, 56, 56))
    c.gq_vis = c.gk_vis = c.gq_ctx = c.gk_ctx = 16
    c.norm_eps = c.ln_eps = 1e-6
    c.softmax_scale = 128 ** -0.5
    c.dt = dt
    return c


def test_block_slot_bytes_layout(L):
    """A slot holds q, k, v, x, y, o of both streams, the three [B, C] fp32
    vectors of both streams, ctx_len and the attention's split-tail workspace,
    each region rounded up to 256 bytes."""
    r256 = lambda n: (n + 255) // 256 * 256
    for B, Nv, Nc, H, dt, esz in ((1, 32, 8, 2, 1, 2), (3, 32, 0, 4, 1, 2), (2, 32, 5, 1, 0, 4)):
        C = H * 128
        want = sum(6 * r256(B * n * C * esz) + 3 * r256(B * C * 4) for n in (Nv, Nc)) + r256(4 * B)
        want += r256(_lib.ATTENTION_WORKSPACE_BYTES)
        assert L.mmdit_block_slot_bytes(ctypes.byref(_block_cfg(B, Nv, Nc, H, dt))) == want


def test_block_config_validation(L):
    f = L.mmdit_block_slot_bytes
    assert f(None) == -1
    c = _block_cfg(); c.D = 64
    assert f(ctypes.byref(c)) == -4
    c = _block_cfg(); c.dt = 5
    assert f(ctypes.byref(c)) == -1
    c = _block_cfg(Nv=31)
    assert f(ctypes.byref(c)) == -2                       # Nv != T*H*W
    c = _block_cfg(); c.grid.split[1] = 58
    assert f(ctypes.byref(c)) == -2                       # split sum != D
    c = _block_cfg(); c.softmax_scale = 0.0
    assert f(ctypes.byref(c)) == -1
    c = _block_cfg(); c.ln_eps = float("nan")
    assert f(ctypes.byref(c)) == -1
    c = _block_cfg(H=40)
    assert f(ctypes.byref(c)) == -4                       # C = 5120 > 4096 bf16 per LN row
    c = _block_cfg(); c.gk_ctx = None
    assert f(ctypes.byref(c)) == -1
    c = _block_cfg(Nc=0); c.gq_ctx = c.gk_ctx = None
    assert f(ctypes.byref(c)) > 0                         # no cond stream: no cond scales
    c = _block_cfg(); c.gq_vis = 18
    assert f(ctypes.byref(c)) == -3


def test_block_forward_host_validation(L):
    """Every rejection happens before any CUDA call, so this runs without a GPU."""
    f = L.mmdit_block_forward_host
    c = _block_cfg()
    slot = L.mmdit_block_slot_bytes(ctypes.byref(c))
    steps = (_lib.BlockStep * 2)()
    for s in steps:
        for name in _lib.BLOCK_STEP_FIELDS:
            setattr(s, name, 64)
    ws = ctypes.c_void_p(256)
    assert f(ctypes.byref(c), steps, 0, None, 0, None) == 0            # nothing to do
    assert f(ctypes.byref(c), steps, -1, ws, slot, None) == -1
    assert f(ctypes.byref(c), None, 2, ws, slot, None) == -1
    assert f(ctypes.byref(c), steps, 2, None, slot, None) == -1
    assert f(ctypes.byref(c), steps, 2, ctypes.c_void_p(272), slot, None) == -3  # 256-byte rule
    assert f(ctypes.byref(c), steps, 2, ws, slot - 1, None) == -1      # less than one slot
    steps[1].x_out_vis = None
    assert f(ctypes.byref(c), steps, 2, ws, slot, None) == -1          # required output
    steps[1].x_out_vis = 64
    steps[0].gate_ctx = None
    assert f(ctypes.byref(c), steps, 2, ws, slot, None) == -1          # cond input missing
    c.D = 64
    assert f(ctypes.byref(c), steps, 2, ws, slot, None) == -4


def test_attention_workspace_constant_matches_header():
    import re
    text = open(_lib.HEADER).read()
    pieces = int(re.search(r"#define MMDIT_ATTENTION_SPLIT_MAX_PIECES (\d+)", text).group(1))
    assert re.search(r"#define MMDIT_ATTENTION_WORKSPACE_BYTES \(MMDIT_ATTENTION_SPLIT_MAX_PIECES "
                     r"\* 256LL \* 130 \* 4\)", text)
    assert _lib.ATTENTION_WORKSPACE_BYTES == pieces * 256 * 130 * 4


def test_attention_ws_validation(L):
    f = L.mmdit_joint_attention_ws
    args = lambda ws, n: (P, P, P, P, P, P, None, P, P, None, ws, n, 1, 8, 8, 2, 128, 0.1, 1, None)
    assert f(*args(ctypes.c_void_p(272), 1 << 20)) == -3          # workspace not 256-aligned
    assert f(*args(ctypes.c_void_p(256), -1)) == -1
    a = list(args(None, 0)); a[16] = 64                              # D != 128
    assert f(*a) == -4
    a = list(args(None, 0)); a[13] = -1                              # Nv < 0
    assert f(*a) == -1
    a = list(args(None, 0)); a[12] = 0                               # B = 0: nothing to do
    assert f(*a) == 0


def test_attention_qnorm_ws_validation(L):
    f = L.mmdit_joint_attention_qnorm_ws
    # q, k, v of both streams, ctx_len, o of both streams, q scales, grid, eps,
    # workspace, bytes, B, Nv, Nc, H, D, softmax_scale, dtype, stream
    args = lambda ws, n: (P, P, P, P, P, P, None, P, P, P, P, None, 1e-6, ws, n, 1, 8, 8, 2, 128,
                          0.1, 1, None)
    assert f(*args(ctypes.c_void_p(272), 1 << 20)) == -3          # workspace not 256-aligned
    assert f(*args(ctypes.c_void_p(256), -1)) == -1
    a = list(args(None, 0)); a[19] = 64                              # D != 128
    assert f(*a) == -4
    a = list(args(None, 0)); a[21] = 0                               # fp32: bf16 only
    assert f(*a) == -4
    a = list(args(None, 0)); a[15] = 0                               # B = 0: nothing to do
    assert f(*a) == 0


def test_backward_ws_validation(L):
    f = L.mmdit_joint_attention_bwd_ws
    Q = ctypes.c_void_p(1 << 20)
    # q..v, ctx_len, o, do, lse, delta, workspace, bytes, the six gradients
    args = lambda ws, n: ([P] * 6 + [None] + [P] * 4 + [Q, Q, ws, n] + [P] * 6 +
                          [1, 8, 8, 2, 128, 0.1, 1, None])
    assert f(*args(ctypes.c_void_p(272), 1 << 20)) == -3          # workspace not 256-aligned
    assert f(*args(ctypes.c_void_p(256), -1)) == -1
    a = args(None, 0); a[11] = None                                 # lse missing
    assert f(*a) == -1
    a = args(None, 0); a[25] = 64                                   # D != 128
    assert f(*a) == -4
    a = args(None, 0); a[21] = 0                                    # B = 0: nothing to do
    assert f(*a) == 0
    w = L.mmdit_joint_window_attention_bwd_ws
    g, win = _lib.Grid(), _lib.Window()
    g.T, g.H, g.W = 1, 2, 4                                          # Nv = 8
    win.parts[0], win.parts[1], win.parts[2] = 1, 1, 2
    wargs = args(ctypes.c_void_p(272), 1 << 20)
    wargs = wargs[:26] + [ctypes.byref(g), ctypes.byref(win)] + wargs[26:]
    assert w(*wargs) == -3                                          # workspace not 256-aligned
    wargs[26] = None
    assert w(*wargs) == -1                                          # no grid


def test_bwd_workspace_bytes_rule():
    """The one-pass backward's accumulator: fp32 [B, Nv + Nc, H, 128]."""
    from mmdit_joint_attention_b200 import api
    assert api.bwd_workspace_bytes(1, 32760, 512, 24) == 1 * 33272 * 24 * 128 * 4
    assert api.bwd_workspace_bytes(2, 0, 5, 3) == 2 * 5 * 3 * 512


def _plan_rule(B, Nv, Nc, H, nsm, ws):
    """The split-tail rule restated: the items past the last whole wave
    (total mod nsm) are split into as many pieces as fill the SMs, at least 2
    key tiles a piece and 160 pieces in all; pieces then get equal tile counts."""
    tiles = -(-Nv // 128) + -(-Nc // 128)
    total = B * H * ((tiles + 1) // 2)
    t = total % nsm
    parts = min(nsm // t, tiles // 2, 160 // t) if t else 0
    if parts < 2:
        return [0, 0, 0, total]
    per = -(-tiles // parts)
    parts = -(-tiles // per)
    if t * parts * 256 * 130 * 4 > ws:
        return [0, 0, 0, total]
    return [t, parts, per, total - t + t * parts]


def test_split_plan(L):
    plan = (ctypes.c_longlong * 4)()
    f = L.mmdit_joint_attention_split_plan
    ws = _lib.ATTENTION_WORKSPACE_BYTES
    # 480p (32,760 + 512 tokens, 24 heads): 3,120 items = 21 waves of 148 + 12,
    # the 12 split into 12 pieces of 22 key tiles
    assert f(1, 32760, 512, 24, 148, ws, plan) == 0
    assert list(plan) == [12, 12, 22, 3108 + 144]
    assert f(1, 32760, 512, 24, 148, 0, plan) == 0 and list(plan) == [0, 0, 0, 3120]
    for B, Nv, Nc, H, nsm in [(b, nv, nc, h, n) for b in (1, 2, 3) for h in (1, 2, 24, 40)
                              for nv in (0, 1, 128, 305, 1024, 32760) for nc in (0, 77, 512)
                              for n in (1, 7, 148)]:
        assert f(B, Nv, Nc, H, nsm, ws, plan) == 0
        got = list(plan)
        assert got == _plan_rule(B, Nv, Nc, H, nsm, ws), (B, Nv, Nc, H, nsm, got)
        t, parts, per, ctas = got
        if parts:
            tiles = -(-Nv // 128) + -(-Nc // 128)
            assert parts * per >= tiles > (parts - 1) * per     # every tile in one piece
            assert t * parts <= min(nsm, 160)
    assert f(-1, 8, 8, 2, 148, ws, plan) == -1
    assert f(1, 8, 8, 2, 0, ws, plan) == -1
    assert f(1, 8, 8, 2, 148, ws, None) == -1


def test_elementwise_bwd_validation(L):
    fm, fr = L.mmdit_adaln_modulate_bwd, L.mmdit_gated_residual_bwd
    # modulate: x, scale, dy, dx, dshift, dscale, B, N, C, eps, dt, stream
    assert fm(P, P, P, ctypes.c_void_p(4096), P, P, 1, 4, 60, 1e-6, 1, None) == -4   # C % 8
    assert fm(P, P, P, ctypes.c_void_p(4096), P, P, 1, 4, 4104, 1e-6, 1, None) == -4  # C > 4096
    assert fm(P, P, P, ctypes.c_void_p(4096), P, P, 1, 4, 64, -1.0, 1, None) == -1   # eps
    assert fm(P, P, P, ctypes.c_void_p(4096), P, P, 1, 4, 64, 1e-6, 9, None) == -1   # dtype
    assert fm(P, None, P, ctypes.c_void_p(4096), P, P, 1, 4, 64, 1e-6, 1, None) == -1
    assert fm(P, P, P, ctypes.c_void_p(4097), P, P, 1, 4, 64, 1e-6, 1, None) == -3
    assert fm(P, P, P, P, ctypes.c_void_p(4096), P, 1, 4, 64, 1e-6, 1, None) == -1   # dx aliases x
    assert fm(None, None, None, None, None, None, 0, 4, 64, 1e-6, 1, None) == 0      # B = 0
    dy0, dy16 = ctypes.c_void_p(8192), ctypes.c_void_p(8192 + 16)
    assert fm(P, P, dy0, dy16, P, P, 1, 4, 64, 1e-6, 1, None) == -1   # dx shifted against dy
    # residual: branch, gate, dout, dx, dbranch, dgate, B, N, C, dt, stream
    assert fr(P, P, P, None, ctypes.c_void_p(4096), P, 1, 4, 60, 1, None) == -4
    assert fr(P, None, P, None, ctypes.c_void_p(4096), P, 1, 4, 64, 1, None) == -1
    assert fr(P, P, P, None, None, P, 1, 4, 64, 1, None) == -1
    assert fr(P, P, P, ctypes.c_void_p(18), ctypes.c_void_p(4096), P, 1, 4, 64, 1, None) == -3
    assert fr(P, P, P, None, P, P, 1, 4, 64, 1, None) == -1                          # dbranch aliases branch
    assert fr(None, None, None, None, None, None, 0, 4, 64, 1, None) == 0
    do0, a0, a16 = ctypes.c_void_p(8192), ctypes.c_void_p(16384), ctypes.c_void_p(16384 + 16)
    assert fr(P, P, do0, a0, a16, P, 1, 4, 64, 1, None) == -1   # dx overlaps dbranch
    assert fr(P, P, do0, a0, a0, P, 1, 4, 64, 1, None) == -1    # dx is dbranch
    assert fr(P, P, do0, None, ctypes.c_void_p(8192 + 16), P, 1, 4, 64, 1, None) == -1
    assert fr(P, P, do0, ctypes.c_void_p(8192 + 32), a0, P, 1, 4, 64, 1, None) == -1
