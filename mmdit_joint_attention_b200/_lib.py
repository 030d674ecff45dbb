"""ctypes binding of libmmdit.so (declared in include/mmdit.h).

Argument marshalling only: every step runs in the library's CUDA kernels.
Loading fails loudly (ImportError) when the library has not been built; there
is no fallback implementation."""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmmdit.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "mmdit.h")

MMDIT_F32 = 0
MMDIT_BF16 = 1

STATUS = {0: "MMDIT_OK", -1: "MMDIT_ERR_ARG", -2: "MMDIT_ERR_SHAPE", -3: "MMDIT_ERR_ALIGN",
          -4: "MMDIT_ERR_UNSUPPORTED", -5: "MMDIT_ERR_CUDA", -6: "MMDIT_ERR_TIMEOUT"}


STATUS_CODES = {v: k for k, v in STATUS.items()}

# MMDIT_ATTENTION_WORKSPACE_BYTES: 160 split pieces x 256 rows x (128 + 2) fp32
ATTENTION_WORKSPACE_BYTES = 160 * 256 * 130 * 4


class Grid(ctypes.Structure):
    """mmdit_grid: visual token grid (T, H, W) and RoPE parameters."""
    _fields_ = [("T", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("pos_scale", ctypes.c_float * 3), ("rope_base", ctypes.c_float),
                ("split", ctypes.c_int * 3)]


class TextRope(ctypes.Structure):
    """mmdit_text_rope: MM-RoPE text positions pos_offset + n on every axis."""
    _fields_ = [("pos_offset", ctypes.c_float), ("rope_base", ctypes.c_float),
                ("split", ctypes.c_int * 3)]


class Window(ctypes.Structure):
    """mmdit_window: number of 3D windows along T, H, W."""
    _fields_ = [("parts", ctypes.c_int * 3)]


class BlockConfig(ctypes.Structure):
    """mmdit_block_config: sizes and constants of the host-buffer executor."""
    _fields_ = [("B", ctypes.c_int), ("Nv", ctypes.c_int), ("Nc", ctypes.c_int),
                ("H", ctypes.c_int), ("D", ctypes.c_int), ("grid", Grid),
                ("gq_vis", ctypes.c_void_p), ("gk_vis", ctypes.c_void_p),
                ("gq_ctx", ctypes.c_void_p), ("gk_ctx", ctypes.c_void_p),
                ("norm_eps", ctypes.c_float), ("ln_eps", ctypes.c_float),
                ("softmax_scale", ctypes.c_float), ("dt", ctypes.c_int)]


BLOCK_STEP_FIELDS = ("q_vis", "k_vis", "v_vis", "q_ctx", "k_ctx", "v_ctx", "x_vis", "x_ctx",
                     "shift_vis", "scale_vis", "gate_vis", "shift_ctx", "scale_ctx", "gate_ctx",
                     "ctx_len", "y_vis", "y_ctx", "o_vis", "o_ctx", "x_out_vis", "x_out_ctx")


class BlockStep(ctypes.Structure):
    """mmdit_block_step: host buffers of one step (every field a pointer)."""
    _fields_ = [(name, ctypes.c_void_p) for name in BLOCK_STEP_FIELDS]


class MmditError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        detail = lib().mmdit_status_string(status).decode()
        if status == -5:
            detail += ": " + lib().mmdit_last_error().decode()
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({detail})")


_LIB = None
_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float


def declared_functions():
    """Names of the functions include/mmdit.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^MMDIT_API\s+(?:int|void|long long|const char\*)\s+(mmdit_\w+)\s*\(",
                                 text, re.M)))


def lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m mmdit_joint_attention_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        L.mmdit_qk_norm_rope.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                         ctypes.POINTER(Grid), _f, _i, _vp]
        L.mmdit_qk_norm_rope_text.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                              ctypes.POINTER(TextRope), _f, _i, _vp]
        L.mmdit_k_norm_rope.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, ctypes.POINTER(Grid), _f,
                                        _i, _vp]
        L.mmdit_joint_attention_qnorm.argtypes = ([_vp] * 11 + [ctypes.POINTER(Grid), _f] +
                                                  [_i] * 5 + [_f, _i, _vp])
        L.mmdit_joint_attention_qnorm_ws.argtypes = ([_vp] * 11 + [ctypes.POINTER(Grid), _f, _vp,
                                                      ctypes.c_longlong] + [_i] * 5 +
                                                     [_f, _i, _vp])
        L.mmdit_quantize_int8.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]
        L.mmdit_quantize_v_e4m3.argtypes = [_vp] * 6 + [_i] * 5 + [_vp]
        L.mmdit_joint_attention_q8.argtypes = [_vp] * 14 + [_i] * 5 + [_f, _vp]
        L.mmdit_qk_norm_rope_bwd.argtypes = [_vp] * 10 + [_i] * 4 + [ctypes.POINTER(Grid), _f,
                                                                   _i, _vp]
        L.mmdit_qk_norm_rope_text_bwd.argtypes = [_vp] * 10 + [_i] * 4 + [
            ctypes.POINTER(TextRope), _f, _i, _vp]
        L.mmdit_qk_norm_rope_window.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                                ctypes.POINTER(Grid), ctypes.POINTER(Window),
                                                _f, _i, _vp]
        L.mmdit_window_permute.argtypes = [_vp, _vp, _i, _i, _i, ctypes.POINTER(Grid),
                                           ctypes.POINTER(Window), _i, _i, _vp]
        L.mmdit_joint_attention.argtypes = [_vp] * 9 + [_i] * 5 + [_f, _i, _vp]
        L.mmdit_joint_attention_fwd.argtypes = [_vp] * 10 + [_i] * 5 + [_f, _i, _vp]
        L.mmdit_joint_attention_ws.argtypes = ([_vp] * 11 + [ctypes.c_longlong] + [_i] * 5 +
                                               [_f, _i, _vp])
        L.mmdit_joint_attention_split_plan.argtypes = [_i] * 5 + [ctypes.c_longlong, _vp]
        L.mmdit_joint_attention_bwd.argtypes = [_vp] * 19 + [_i] * 5 + [_f, _i, _vp]
        L.mmdit_joint_attention_bwd_ws.argtypes = ([_vp] * 14 + [ctypes.c_longlong] + [_vp] * 6 +
                                                   [_i] * 5 + [_f, _i, _vp])
        L.mmdit_joint_window_attention.argtypes = ([_vp] * 9 + [_i] * 5 +
                                                   [ctypes.POINTER(Grid), ctypes.POINTER(Window),
                                                    _f, _i, _vp])
        L.mmdit_joint_window_attention_fwd.argtypes = ([_vp] * 10 + [_i] * 5 +
                                                       [ctypes.POINTER(Grid),
                                                        ctypes.POINTER(Window), _f, _i, _vp])
        L.mmdit_joint_window_attention_bwd.argtypes = ([_vp] * 19 + [_i] * 5 +
                                                       [ctypes.POINTER(Grid),
                                                        ctypes.POINTER(Window), _f, _i, _vp])
        L.mmdit_joint_window_attention_bwd_ws.argtypes = ([_vp] * 14 + [ctypes.c_longlong] +
                                                          [_vp] * 6 + [_i] * 5 +
                                                          [ctypes.POINTER(Grid),
                                                           ctypes.POINTER(Window), _f, _i, _vp])
        L.mmdit_adaln_modulate.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _f, _i, _vp]
        L.mmdit_adaln_modulate_pair.argtypes = ([_vp] * 4 + [_i] + [_vp] * 4 + [_i] * 3 +
                                                [_f, _i, _vp])
        L.mmdit_gated_residual.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]
        L.mmdit_residual_modulate.argtypes = [_vp] * 7 + [_i, _i, _i, _f, _i, _vp]
        L.mmdit_adaln_modulate_bwd.argtypes = [_vp] * 6 + [_i, _i, _i, _f, _i, _vp]
        L.mmdit_gated_residual_bwd.argtypes = [_vp] * 6 + [_i, _i, _i, _i, _vp]
        L.mmdit_device_status.argtypes = [_vp]
        L.mmdit_block_slot_bytes.argtypes = [ctypes.POINTER(BlockConfig)]
        L.mmdit_block_slot_bytes.restype = ctypes.c_longlong
        L.mmdit_block_forward_host.argtypes = [ctypes.POINTER(BlockConfig),
                                               ctypes.POINTER(BlockStep), _i, _vp,
                                               ctypes.c_longlong, _vp]
        L.mmdit_set_wait_timeout_ns.argtypes = [ctypes.c_ulonglong]
        L.mmdit_set_wait_timeout_ns.restype = None
        L.mmdit_last_error.argtypes = []
        L.mmdit_last_error.restype = ctypes.c_char_p
        L.mmdit_status_string.argtypes = [_i]
        L.mmdit_status_string.restype = ctypes.c_char_p
        for name in ("mmdit_qk_norm_rope", "mmdit_qk_norm_rope_text", "mmdit_qk_norm_rope_window",
                     "mmdit_qk_norm_rope_bwd", "mmdit_qk_norm_rope_text_bwd", "mmdit_k_norm_rope",
                     "mmdit_joint_attention_qnorm", "mmdit_joint_attention_qnorm_ws",
                     "mmdit_quantize_int8", "mmdit_quantize_v_e4m3", "mmdit_joint_attention_q8",
                     "mmdit_window_permute", "mmdit_joint_attention",
                     "mmdit_joint_attention_fwd", "mmdit_joint_attention_bwd",
                     "mmdit_joint_attention_bwd_ws", "mmdit_joint_window_attention_bwd_ws",
                     "mmdit_joint_attention_ws", "mmdit_joint_attention_split_plan",
                     "mmdit_joint_window_attention", "mmdit_joint_window_attention_fwd",
                     "mmdit_joint_window_attention_bwd", "mmdit_adaln_modulate",
                     "mmdit_adaln_modulate_pair", "mmdit_gated_residual", "mmdit_residual_modulate", "mmdit_device_status",
                     "mmdit_adaln_modulate_bwd", "mmdit_gated_residual_bwd",
                     "mmdit_block_forward_host"):
            getattr(L, name).restype = ctypes.c_int
        _LIB = L
    return _LIB


def check(fn: str, status: int) -> None:
    if status != 0:
        raise MmditError(fn, status)
