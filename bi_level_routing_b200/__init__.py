"""Bi-Level Routing Attention (BRA) forward pass for NVIDIA B200 (sm_100a).

The compute lives in ``libbra.so`` (hand-written CUDA behind a C ABI, declared in
``include/bra.h``); this package only marshals torch tensors into it. The binding is
loaded on first use and raises if the library is missing: there is no CPU fallback.
"""
from .workloads import HEADLINE, WORKLOADS, Workload, make_inputs  # noqa: F401
