"""The forward pass of one-token regions in one kernel (routing inside the dense attention
kernel, one thread-block cluster per image) against the two-kernel path and the oracle.

Its index must be the same bits as bra_route's (the same partial products, added in the same
order) and its output the same bits as bra_attend's with the dense kernel; both are also
checked against the oracle under the usual rules."""
import numpy as np
import pytest
import torch

import bi_level_routing_b200 as bra
import oracle
from bi_level_routing_b200.workloads import WORKLOADS, Workload
from parity import check_output, check_routing, host_values, make

pytestmark = pytest.mark.gpu

FUSED = [
    # name, B, H=W=n_win, C, heads, topk: CTAs per image = C / 128 (two blocks each) or C / 64
    ("c64_one_cta", 3, 7, 64, 2, 5),            # one block: a cluster of one CTA
    ("c128_pair", 3, 7, 128, 4, 49),            # two blocks in one CTA, full sort
    ("c192_three", 2, 7, 192, 6, 7),            # odd block count: one block per CTA, cluster of 3
    ("c512_r64_topk64", 2, 8, 512, 16, 64),     # R = 64: four row tiles, eight key tiles
    ("c512_r9_topk1", 4, 3, 512, 16, 1),        # R = 9: one row tile, two key tiles, argmax rounds
    ("c1024_cluster8", 2, 5, 1024, 32, 25),     # sixteen blocks: the widest cluster (8 CTAs)
    ("c256_r36_topk6", 5, 6, 256, 8, 6),
]


def _workload(spec, values="iid", seed=4321):
    name, B, n, C, heads, topk = spec
    return Workload(name, B, n, n, C, heads, n, topk, "bf16", values, seed)


def _two_kernel_path(q, k, v, w):
    idx = bra.route(q, k, w.n_win, w.topk)
    try:
        bra.set_attend_kernel("dense_mma")
        out = bra.attend(q, k, v, idx, w.heads, w.n_win)
    finally:
        bra.set_attend_kernel("auto")
    return out, idx


def _check(w, q, k, v, inp):
    assert bra.kernels_per_call("bra_forward", w.B, w.H, w.W, w.C, w.heads, w.n_win, w.topk,
                                torch.bfloat16) == 1, "the shape does not take the fused kernel"
    out, idx = bra.forward(q, k, v, w.n_win, w.topk, w.heads)
    out2, idx2 = _two_kernel_path(q, k, v, w)
    torch.cuda.synchronize()
    assert bra.check_device_error() == 0
    assert torch.equal(idx, idx2), "fused routing differs from bra_route"
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16)), "fused attention differs from bra_attend"
    gidx = idx.cpu().numpy()
    check_routing(gidx, inp["q"], inp["k"], w.n_win, w.topk)
    ref = oracle.attend(inp["q"], inp["k"], inp["v"], gidx, w.heads, w.n_win)
    check_output(host_values(out), ref, "bf16", f"{w.name} fused forward")


@pytest.mark.parametrize("spec", FUSED, ids=[s[0] for s in FUSED])
def test_fused_forward_small(spec):
    w = _workload(spec)
    inp, (q, k, v) = make(w)
    _check(w, q, k, v, inp)


def test_fused_forward_stage4_full_size():
    w = WORKLOADS["stage4"]
    inp, (q, k, v) = make(w)
    _check(w, q, k, v, inp)


def test_fused_forward_ties_and_nan():
    """Equal tokens give equal affinities (ties go to the lower region) and a NaN token ranks
    last, in both paths alike."""
    w = _workload(("ties", 2, 7, 256, 8, 10))
    inp, (q, k, v) = make(w)
    k[0, 0, 3] = k[0, 0, 1]      # regions 1 and 3 of image 0: equal keys
    k[0, 2, 2] = k[0, 1, 5]      # regions 16 and 12
    k[1, 4, 4] = float("nan")    # region 32 of image 1: NaN affinities
    out, idx = bra.forward(q, k, v, w.n_win, w.topk, w.heads)
    out2, idx2 = _two_kernel_path(q, k, v, w)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    gidx = idx.cpu().numpy()
    for r in range(w.R):
        row = list(gidx[0, r])
        if 1 in row and 3 in row:
            assert row.index(1) < row.index(3)
        assert 32 not in gidx[1, r] or w.topk == w.R


def test_fused_forward_host_chunks():
    """bra_forward_host runs the fused kernel per chunk of images: the same bits as on device."""
    w = _workload(("host", 5, 7, 512, 16, 49))
    inp, (q, k, v) = make(w)
    out, idx = bra.forward(q, k, v, w.n_win, w.topk, w.heads)
    hout, hidx = bra.forward_host(q.cpu().pin_memory(), k.cpu().pin_memory(), v.cpu().pin_memory(), w.n_win,
                                  w.topk, w.heads)
    torch.cuda.synchronize()
    assert torch.equal(hidx, idx.cpu())
    assert torch.equal(hout.view(torch.int16), out.cpu().view(torch.int16))
