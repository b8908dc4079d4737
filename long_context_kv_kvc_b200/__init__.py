"""B200-native attention-saliency KV-cache compaction.

The compute path is libkvc.so (hand-written CUDA for sm_100a behind the C ABI in
include/kvc.h); ``long_context_kv_kvc_b200.kvc`` is its ctypes binding and raises on import
if the library is not built.  ``long_context_kv_kvc_b200.synth`` draws the seeded synthetic
workloads.
"""
__all__ = ["kvc", "synth", "build"]
