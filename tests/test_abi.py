"""The C ABI on the host: the library loads, exports what include/bra.h declares, and
rejects bad arguments before touching a GPU. No kernel is launched here."""
import ctypes

import pytest

from bi_level_routing_b200 import api
from bi_level_routing_b200.workloads import WORKLOADS

OK, INVALID, UNSUPPORTED = 0, 1, 2


@pytest.fixture(scope="module")
def L():
    from bi_level_routing_b200 import build
    build.build()
    return api.lib()


def test_exports_every_declared_symbol(L):
    names = api.declared_symbols()
    assert len(names) >= 11, names
    for name in names:
        assert hasattr(L, name), f"libbra.so does not export {name}"


def test_status_strings(L):
    for code, name in api.STATUS.items():
        assert L.bra_status_string(code).decode() == name


FAKE = 0x10000  # a 16-byte aligned non-NULL value; these calls must fail before using it


def _route(L, q=FAKE, k=FAKE, idx=FAKE, B=1, H=28, W=28, C=64, n_win=7, topk=4, dtype=1):
    return L.bra_route(q, k, idx, B, H, W, C, n_win, topk, dtype, None)


def _attend(L, q=FAKE, k=FAKE, v=FAKE, idx=FAKE, out=FAKE, B=1, H=28, W=28, C=64, heads=2, n_win=7, topk=4,
            dtype=1):
    return L.bra_attend(q, k, v, idx, out, B, H, W, C, heads, n_win, topk, dtype, None)


def _forward(L, q=FAKE, k=FAKE, v=FAKE, idx=FAKE, out=FAKE, B=1, H=28, W=28, C=64, heads=2, n_win=7, topk=4,
             dtype=1):
    return L.bra_forward(q, k, v, idx, out, B, H, W, C, heads, n_win, topk, dtype, None)


@pytest.mark.parametrize("kw", [
    dict(H=30),            # H % n_win != 0
    dict(W=27),            # W % n_win != 0
    dict(topk=50),         # topk > R
    dict(topk=0), dict(n_win=0), dict(C=0), dict(H=-7), dict(B=-1),
    dict(dtype=7),         # unknown dtype
    dict(C=60),            # C * 2 bytes not a multiple of 16
    dict(q=0), dict(k=0), dict(idx=0),
    dict(q=FAKE + 8),      # not 16-byte aligned
    dict(idx=FAKE + 2),    # not 4-byte aligned
])
def test_route_rejects(L, kw):
    assert _route(L, **kw) == INVALID


@pytest.mark.parametrize("kw", [
    dict(heads=3),         # C % heads != 0
    dict(heads=0), dict(v=0), dict(out=0), dict(v=FAKE + 4), dict(out=FAKE + 8),
    dict(dtype=0, C=62, heads=2),  # fp32: C * 4 bytes not a multiple of 16
    dict(topk=50),
])
def test_attend_and_forward_reject(L, kw):
    assert _attend(L, **kw) == INVALID
    assert _forward(L, **kw) == INVALID


def test_empty_batch_is_a_no_op(L):
    assert _route(L, B=0, q=0, k=0, idx=0) == OK
    assert _attend(L, B=0, q=0, k=0, v=0, idx=0, out=0) == OK
    assert _forward(L, B=0, q=0, k=0, v=0, idx=0, out=0) == OK
    assert L.bra_kernels_per_call(b"bra_forward", 0, 28, 28, 64, 2, 7, 4, 1) == 0


def test_unsupported_sizes(L):
    assert _route(L, H=33, W=33, n_win=33, topk=1) == UNSUPPORTED  # R = 1089 > 1024
    assert L.bra_selected_attend_kernel(1, 8, 8, 1024, 4, 2, 1, 1) == -1  # head_dim 256 > 128


def test_kernel_selection_per_workload(L):
    assert L.bra_set_attend_kernel(0) == OK
    want = {"tiny_f32": "simt", "stage1": "gather_umma", "stage2": "gather_mma", "stage3": "region_mma",
            "stage4": "dense_mma", "highres": "gather_umma"}
    import torch
    for name, kernel in want.items():
        w = WORKLOADS[name]
        dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
        assert api.selected_attend_kernel(w.B, w.H, w.W, w.C, w.heads, w.n_win, w.topk, dt) == kernel, name


def test_forcing_a_kernel(L):
    try:
        assert L.bra_set_attend_kernel(9) == INVALID
        assert L.bra_set_attend_kernel(4) == OK
        assert L.bra_selected_attend_kernel(64, 56, 56, 64, 2, 7, 1, 1) == 4
        assert L.bra_selected_attend_kernel(64, 28, 28, 128, 4, 7, 4, 1) == -1  # 16-token regions
        assert L.bra_set_attend_kernel(1) == OK
        assert L.bra_selected_attend_kernel(64, 56, 56, 64, 2, 7, 1, 1) == 1
        assert L.bra_set_attend_kernel(3) == OK
        assert L.bra_selected_attend_kernel(64, 56, 56, 64, 2, 7, 1, 1) == -1  # 3136 tokens > 256
        assert L.bra_selected_attend_kernel(64, 14, 14, 256, 8, 7, 16, 1) == 3
        assert L.bra_set_attend_kernel(2) == OK
        assert L.bra_selected_attend_kernel(1, 28, 28, 64, 2, 7, 4, 0) == -1  # fp32 has no tensor-core kernel
        assert L.bra_set_attend_kernel(6) == INVALID
        assert L.bra_set_attend_kernel(5) == OK
        assert L.bra_selected_attend_kernel(64, 14, 14, 256, 8, 7, 16, 1) == 5  # 4-token regions
        assert L.bra_selected_attend_kernel(64, 14, 14, 64, 2, 7, 16, 1) == -1  # C % 128 != 0
        assert L.bra_selected_attend_kernel(64, 28, 28, 128, 4, 7, 4, 1) == -1  # 16-token regions
        assert L.bra_selected_attend_kernel(4, 28, 28, 128, 4, 14, 4, 1) == -1  # 784 tokens > 256
    finally:
        L.bra_set_attend_kernel(0)


def test_scratch_and_launch_accounting(L):
    assert L.bra_route_scratch_bytes(64, 56, 56, 64, 7) == 2 * 64 * 49 * 64 * 4
    stage1 = (64, 56, 56, 64, 2, 7, 1, 1)
    highres = (8, 128, 128, 64, 2, 16, 4, 1)
    assert L.bra_kernels_per_call(b"bra_route", *stage1) == 2  # means, then affinity + top-k
    assert L.bra_kernels_per_call(b"bra_route", *highres) == 2
    assert L.bra_kernels_per_call(b"bra_attend", *stage1) == 1
    assert L.bra_kernels_per_call(b"bra_forward", *stage1) == 3
    assert L.bra_kernels_per_call(b"bra_forward", *highres) == 3
    assert L.bra_kernels_per_call(b"bra_forward", 1, 30, 28, 64, 2, 7, 4, 1) == 0  # rejected
    stage4 = (64, 7, 7, 512, 16, 7, 49, 1)  # one-token regions: routing reads q and k directly
    assert L.bra_kernels_per_call(b"bra_route", *stage4) == 1
    assert L.bra_kernels_per_call(b"bra_forward", *stage4) == 1  # routing inside the dense kernel
    assert L.bra_kernels_per_call(b"bra_forward_host", *stage4) == 1
    f32_stage4 = stage4[:-1] + (0,)  # fp32: the CUDA-core kernels, routing then attention
    assert L.bra_kernels_per_call(b"bra_forward", *f32_stage4) == 2
    try:  # with another attention kernel forced, the forward pass is routing then attention
        L.bra_set_attend_kernel(1)
        assert L.bra_kernels_per_call(b"bra_forward", *stage4) == 2
    finally:
        L.bra_set_attend_kernel(0)
    # the fused kernel's limits: a cluster of at most 8 CTAs (C <= 1024 with two 64-channel blocks
    # per CTA, an odd block count one per CTA up to 8 blocks), at most 64 one-token regions
    assert L.bra_kernels_per_call(b"bra_forward", 2, 5, 5, 1024, 32, 5, 25, 1) == 1
    assert L.bra_kernels_per_call(b"bra_forward", 2, 7, 7, 448, 14, 7, 7, 1) == 1   # 7 blocks, cluster of 7
    assert L.bra_kernels_per_call(b"bra_forward", 2, 7, 7, 576, 18, 7, 7, 1) == 2   # 9 blocks: unfused
    assert L.bra_kernels_per_call(b"bra_forward", 2, 9, 9, 64, 2, 9, 9, 1) == 2     # R = 81: unfused
    assert L.bra_route_scratch_bytes(64, 7, 7, 512, 7) == 0
    assert L.bra_kernels_per_call(b"nonsense", *stage1) == 0


# ------------------------------------------------------------------ the added entry points: rejected before any launch

def _heads(L, q=FAKE, k=FAKE, idx=FAKE, B=1, H=28, W=28, C=64, heads=2, n_win=7, topk=4, dtype=1):
    return L.bra_route_heads(q, k, idx, B, H, W, C, heads, n_win, topk, dtype, None)


@pytest.mark.parametrize("kw", [dict(heads=3), dict(topk=50), dict(heads=0), dict(q=0), dict(idx=FAKE + 2),
                                dict(H=30), dict(dtype=5)])
def test_route_heads_rejects(L, kw):
    assert _heads(L, **kw) == INVALID


def test_route_heads_unsupported(L):
    # one-token bf16 regions with 4-channel heads: a head's slice is not a 16-byte vector
    assert _heads(L, H=7, W=7, C=8, heads=2, topk=3) == UNSUPPORTED
    assert _heads(L, H=34, W=34, n_win=17, topk=3) == UNSUPPORTED  # R = 289 > 256


def test_attend_heads_and_forward_heads_reject(L):
    args = (FAKE, FAKE, FAKE, FAKE, FAKE, 1, 28, 28, 64, 2, 7, 4, 1, None)
    for fn in (L.bra_attend_heads, L.bra_forward_heads):
        assert fn(0, *args[1:]) == INVALID
        assert fn(*args[:4], FAKE + 8, *args[5:]) == INVALID
        assert fn(*args[:8], 3, *args[9:]) == INVALID  # C % heads


def test_forward_auto_pad_rejects(L):
    base = [FAKE, FAKE, FAKE, FAKE, FAKE, 1, 27, 30, 64, 2, 7, 4, 1, None]
    for pos, val in ((10, 0), (6, 0), (7, -3), (11, 50), (8, 60), (0, 0), (4, FAKE + 8)):
        a = list(base)
        a[pos] = val
        assert L.bra_forward_auto_pad(*a) == INVALID, (pos, val)


def test_lepe_rejects(L):
    assert L.bra_lepe(FAKE, FAKE, FAKE, FAKE, 1, 8, 8, 64, 1, None) == INVALID  # x == y
    assert L.bra_lepe(FAKE, FAKE, FAKE, FAKE + 4096, 1, 8, 8, 12, 1, None) == INVALID  # bf16 C % 8
    assert L.bra_lepe(FAKE, 0, FAKE, FAKE + 4096, 1, 8, 8, 64, 1, None) == INVALID
    assert L.bra_lepe(FAKE, FAKE, FAKE, FAKE + 4096, -1, 8, 8, 64, 1, None) == INVALID
    assert L.bra_lepe(FAKE, FAKE, FAKE, FAKE + 4096, 0, 8, 8, 64, 1, None) == OK  # empty batch
    # out == attn is rejected before the forward pass runs
    assert L.bra_forward_lepe(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 28, 28, 64, 2, 7, 4, 1, None) == INVALID


def test_backward_rejects(L):
    good = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 28, 28, 64, 2, 7, 4, 1, None]
    a = list(good)
    a[5] = 0  # dq
    assert L.bra_attend_backward(*a) == INVALID
    a = list(good)
    a[6] = FAKE + 4  # dk not 16-byte aligned
    assert L.bra_attend_backward(*a) == INVALID
    a = list(good)
    a[11], a[12], a[15] = 8, 4, 0  # fp32, C = 8, heads = 4: head_dim 2
    assert L.bra_attend_backward(*a) == UNSUPPORTED
