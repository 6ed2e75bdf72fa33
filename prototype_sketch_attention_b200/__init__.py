"""B200-native Sketch Attention (sm_100a).

Sketch Attention compresses a user's raw history into a fixed k x d sketch.
Learnable prototypes score every token, each token spreads unit mass over the
prototypes, and each sketch row is the mass-weighted mean of the tokens' values
(blog "100,000 videos in your pocket", section "1. Sketch Attention compresses the
history"; evolve.pub review of arXiv 2609.08443, "Summary").

The computation lives in libsa_sketch.so (C ABI: include/sa_sketch.h). The
``binding`` module wraps it with ctypes. Its names load lazily, so
``prototype_sketch_attention_b200.inputs`` can be imported before the library is
built.
"""
from __future__ import annotations

_BINDING_NAMES = {
    "sa_sketch_workspace_size", "sa_sketch_forward", "sa_sketch_backward",
    "sa_sketch_get_device_status", "sa_status_string", "sa_sketch_debug_wait_timeout",
    "forward", "backward", "workspace", "device_status", "SketchAttentionError",
    "SA_F32", "SA_BF16", "SA_OK",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
