"""B200-native MoE layer hot path: routing, dispatch, expert FFN, combine, popularity.

The compute lives in ``libmoe.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/moe.h``).  ``routing_dispatch_expert_fp32_b200.moe`` is the
thin ctypes binding over it; ``workloads`` builds seeded synthetic inputs.
"""
