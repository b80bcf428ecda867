"""B200-native fused ShortConv K/V step (causal depthwise token conv ->
per-head RMSNorm -> paged KV-cache write, with a carried conv state).

The compute path is the C-ABI library ``libsconvkv.so`` (hand-written
sm_100a CUDA kernels); ``short_conv_kv_b200.binding`` is its thin ctypes
front end.  ``workloads`` holds the seeded synthetic input generators.
"""
__all__ = ["binding", "workloads"]
