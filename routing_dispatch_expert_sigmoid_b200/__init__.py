"""One Mixture-of-Experts layer on one B200: router, top-k gating with capacity,
histogram and prefix sum, dispatch, grouped SwiGLU expert FFN and combine.

The compute lives in libmoe.so (hand-written sm_100a CUDA behind a C ABI,
declared in include/moe.h); `ops` is its thin Python binding.  The binding
loads the library on first use and raises if it is missing: there is no CPU
fallback.
"""
from .workloads import WORKLOADS, Workload, make_inputs  # noqa: F401
