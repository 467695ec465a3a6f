"""B200-native decode-step hot path of confidence-aware KV-cache eviction (CONF-KV).

The compute lives in libconfkv.so (CUDA, sm_100a) behind the C ABI declared in
include/confkv.h; ``binding`` is its ctypes marshalling layer, ``synth`` the
seeded synthetic workload generator, ``build`` the in-tree nvcc build.
Importing this package does not load the library; the first call into
``binding`` does, and raises if the library is missing.
"""
from .binding import (ALL_LAYERS, COMPACT_HOLEFILL, COMPACT_STABLE, GATE_LITERAL, GATE_PROSE,
                      MODE_CONF, MODE_FIXED, ConfKV, ConfKVError, load_library, logical_segment)

__all__ = ["ALL_LAYERS", "COMPACT_HOLEFILL", "COMPACT_STABLE", "GATE_LITERAL", "GATE_PROSE",
           "MODE_CONF", "MODE_FIXED", "ConfKV", "ConfKVError", "load_library", "logical_segment"]
