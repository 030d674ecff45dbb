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
