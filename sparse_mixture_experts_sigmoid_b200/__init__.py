"""B200-native forward pass of a top-k routed mixture-of-experts SwiGLU FFN layer.

The compute lives in ``libmoe.so`` (hand-written CUDA for sm_100a behind a C
ABI, declared in ``include/moe.h``).  This package is its thin Python binding
(``binding``), the workload shapes (``workloads``), the seeded synthetic input
generator (``synth``) and the roofline arithmetic used by the benchmark
(``roofline``).  The library is loaded on first use; if it is missing the
binding raises instead of computing anything another way.
"""
from .workloads import WORKLOADS, Workload, HEADLINE  # noqa: F401
