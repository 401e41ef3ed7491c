"""AVQ-attention forward path for NVIDIA B200 (sm_100a).

Two calls, both hand-written CUDA behind a C ABI (``include/avq.h``):
``precompute`` (fused full-tree vector quantisation of the keys with
per-codeword counts and value sums) and ``attention`` (parent attention,
per-tile importance, top-P refinement with children, output).

The binding loads ``_lib/libavq_b200.so`` on first use and raises if it is
missing; ``synthetic`` holds the seeded input generator.
"""
from __future__ import annotations

_BINDING_NAMES = {
    "precompute", "attention", "workspace", "AVQError", "make_shape", "lib", "library_path",
    "avq_precompute", "avq_attention", "avq_precompute_workspace_bytes",
    "avq_attention_workspace_bytes", "avq_device_status", "avq_status_string", "avq_version",
    "avq_kernel_launches", "avq_attention_noalloc",
    "EXPORTS",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
