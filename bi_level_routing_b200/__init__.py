"""Bi-Level Routing Attention (BRA) forward pass for NVIDIA B200 (sm_100a).

The compute lives in ``libbra.so`` (hand-written CUDA behind a C ABI, declared in
``include/bra.h``); this package only marshals torch tensors into it. The library is loaded
on first use and a missing library raises: there is no CPU fallback.
"""
from .api import (BraError, attend, attend_backward, attend_heads, check_device_error, forward,  # noqa: F401
                  forward_auto_pad, forward_heads, forward_host, forward_lepe, kernels_per_call, lepe, route,
                  route_heads, route_scratch_bytes, selected_attend_kernel, set_attend_kernel, set_max_ctas)
from .workloads import HEADLINE, WORKLOADS, Workload, make_inputs  # noqa: F401
