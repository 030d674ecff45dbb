"""B200-native joint-attention core of a dual-stream MMDiT block.

The compute path is libmmdit.so (hand-written sm_100a CUDA behind a C ABI,
declared in include/mmdit.h); ``api`` binds it for torch CUDA tensors.
``inputs`` holds the seeded synthetic workload generator.  Importing the
package does not load the library; the first use of an ``api`` function does,
and fails loudly if it has not been built."""
import importlib

_API = ("qk_norm_rope", "qk_norm_rope_text", "joint_attention", "adaln_modulate", "gated_residual",
        "residual_modulate", "block_forward", "device_status")
__all__ = list(_API)


def __getattr__(name):
    if name in _API:
        return getattr(importlib.import_module(".api", __name__), name)
    raise AttributeError(name)
