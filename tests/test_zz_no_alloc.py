"""bra_route_noalloc: routing with no device allocation, checked against bra_route.

Callers that cannot allocate device memory mid-run use bra_route_noalloc instead of
bra_route: a process that hands all of HBM to its own allocator at start-up, or a
latency-critical loop that must not take allocator locks or risk an out-of-memory error.
Its scratch is a fixed array inside the library, shared by every call, so this test makes
two calls in a row on different shapes and checks that each returns exactly bra_route's
indices (the same kernels run, so the routing must be bit-identical). Shapes that route on chip
(one-token regions, and up to 256 regions of several tokens) need no scratch at all; the others
use the fixed array. It sits in a file of its own, collected last.
"""
import ctypes

import pytest
import torch

import bi_level_routing_b200 as bra
from bi_level_routing_b200 import api
from bi_level_routing_b200.workloads import WORKLOADS, Workload
from parity import make

pytestmark = pytest.mark.gpu


def _lib():
    L = api.lib()
    vp, I = ctypes.c_void_p, ctypes.c_int
    L.bra_route_noalloc.argtypes = [vp, vp, vp, I, I, I, I, I, I, I, vp]
    L.bra_route_noalloc.restype = I
    return L


def _route_noalloc(L, q, k, idx, n_win, topk):
    B, H, W, C = q.shape
    return L.bra_route_noalloc(q.data_ptr(), k.data_ptr(), idx.data_ptr(), B, H, W, C, n_win, topk,
                               api.DTYPES[q.dtype], torch.cuda.current_stream().cuda_stream)


# Shapes the on-chip routing kernel does not take (more than 256 regions) use the fixed scratch;
# the named workloads route on chip and need none. Both kinds, two calls in a row.
WIDE = Workload("r400_rs4", 2, 40, 40, 64, 2, 20, 6, "bf16", "region_offset", 31)
WIDE_F32 = Workload("r324_rs4_f32", 3, 36, 36, 32, 1, 18, 5, "f32", "region_offset", 32)


def test_no_alloc_route_matches_bra_route_on_two_calls_in_a_row():
    L = _lib()
    # full-size stage3 needs the most scratch of the named workloads (2 * 64 * 49 * 256 * 4 = 6.4 MB)
    for w in (WIDE, WORKLOADS["stage1"].with_(B=16), WIDE_F32, WORKLOADS["highres"].with_(B=2), WORKLOADS["stage3"],
              WORKLOADS["highres"]):
        _, (q, k, _) = make(w)
        ref = bra.route(q, k, w.n_win, w.topk)
        idx = torch.full_like(ref, -7)
        assert _route_noalloc(L, q, k, idx, w.n_win, w.topk) == 0, L.bra_last_error_message()
        torch.cuda.synchronize()
        assert torch.equal(idx, ref), f"{w.name}: bra_route_noalloc differs from bra_route"
    # the largest of these that fits the fixed scratch: 2 * 24 * 400 * 64 * 4 bytes = 4.9 MB
    w = WIDE.with_(B=24)
    assert 2 * w.B * w.R * w.C * 4 <= 8 << 20
    _, (q, k, _) = make(w)
    ref = bra.route(q, k, w.n_win, w.topk)
    idx = torch.full_like(ref, -7)
    assert _route_noalloc(L, q, k, idx, w.n_win, w.topk) == 0, L.bra_last_error_message()
    torch.cuda.synchronize()
    assert torch.equal(idx, ref), "full-scratch call differs from bra_route"


def test_no_alloc_route_rejects_sizes_beyond_its_scratch():
    L = _lib()
    # more than 256 four-token regions, so the means go through scratch:
    # 2 * 16 * 400 * 256 * 4 bytes = 13.1 MB > 8 MiB
    w = WIDE.with_(B=16, C=256, heads=8)
    assert w.H // w.n_win * (w.W // w.n_win) > 1 and w.R > 256
    fake = 0x10000  # rejected before any use
    status = L.bra_route_noalloc(fake, fake, fake, w.B, w.H, w.W, w.C, w.n_win, w.topk, 1, None)
    assert status == 2  # BRA_ERR_UNSUPPORTED
    assert b"bytes of scratch" in L.bra_last_error_message()


def test_one_token_regions_route_from_the_tokens_without_scratch():
    """For one-token regions the means are the tokens, so both entry points route from q and k
    directly and need no scratch: the full stage4 batch, whose fp32 means would not fit the fixed
    scratch, routes too. The indices must equal bra_route's bit for bit, bf16 (tensor-core
    kernel) and fp32 (CUDA-core kernel)."""
    L = _lib()
    for w in (WORKLOADS["stage4"], WORKLOADS["stage4"].with_(B=3, dtype="f32")):
        assert w.H == w.n_win and w.W == w.n_win
        _, (q, k, _) = make(w)
        ref = bra.route(q, k, w.n_win, w.topk)
        idx = torch.full_like(ref, -7)
        assert _route_noalloc(L, q, k, idx, w.n_win, w.topk) == 0, L.bra_last_error_message()
        torch.cuda.synchronize()
        assert torch.equal(idx, ref), f"{w.name} {w.dtype}: bra_route_noalloc differs from bra_route"
