"""The rows after the forward pass, through the C ABI against the CPU oracle, every element:
per-head routing and attention, the LePE epilogue, the backward pass and auto_pad."""
import numpy as np
import pytest
import torch

import bi_level_routing_b200 as bra
import oracle
from bi_level_routing_b200.workloads import WORKLOADS, Workload, make_inputs
from parity import check_grad, check_output, check_routing, check_routing_heads, host_values, make

pytestmark = pytest.mark.gpu


def _w(name, B, H, W, C, heads, n, topk, dt, values="region_offset", seed=4242):
    return Workload(name, B, H, W, C, heads, n, topk, dt, values, seed)


# ------------------------------------------------------------------ per-head routing

HEADS_SHAPES = [WORKLOADS["stage1"], WORKLOADS["stage2"], WORKLOADS["stage3"],
                WORKLOADS["stage4"].with_(B=8), WORKLOADS["highres"].with_(B=2), WORKLOADS["tiny_f32"],
                _w("rs15_f32", 2, 12, 20, 32, 4, 4, 3, "f32"), _w("rs4_hd64", 2, 16, 16, 128, 2, 8, 6, "bf16")]


@pytest.mark.parametrize("w", HEADS_SHAPES, ids=[w.name for w in HEADS_SHAPES])
def test_forward_heads(w):
    inp, (q, k, v) = make(w)
    out, idx = bra.forward_heads(q, k, v, w.n_win, w.topk, w.heads)
    torch.cuda.synchronize()
    assert bra.check_device_error() == 0
    gidx = idx.cpu().numpy()
    _, near = check_routing_heads(gidx, inp["q"], inp["k"], w.n_win, w.topk, w.heads)
    assert near <= max(2, gidx.size // gidx.shape[-1] // 1000)
    ref = oracle.attend_heads(inp["q"], inp["k"], inp["v"], gidx, w.n_win)
    check_output(host_values(out), ref, w.dtype, f"{w.name} per-head forward")
    # route_heads + attend_heads give the same as the fused call
    idx2 = bra.route_heads(q, k, w.n_win, w.topk, w.heads)
    out2 = bra.attend_heads(q, k, v, idx2, w.n_win)
    assert torch.equal(idx2, idx) and torch.equal(out2, out)


# shapes the tensor-core gather kernel takes in its per-head mode (bf16, hd 32, rs % 16 == 0):
# one and two 64-channel blocks per item, a last item group with a block past C, 48-token regions
HEADS_GATHER = [WORKLOADS["stage1"].with_(B=6), WORKLOADS["stage2"].with_(B=6),
                WORKLOADS["highres"].with_(B=1),
                _w("rs32_c192", 3, 16, 32, 192, 6, 4, 5, "bf16"), _w("rs48_c64", 2, 24, 32, 64, 2, 4, 3, "bf16")]


@pytest.mark.parametrize("w", HEADS_GATHER, ids=[w.name for w in HEADS_GATHER])
def test_heads_both_kernels(w):
    """Per-head attention on the tensor cores and on CUDA cores: each against the oracle over the
    same per-head index; any other forced kernel refuses per-head indices."""
    inp, (q, k, v) = make(w)
    idx = bra.route_heads(q, k, w.n_win, w.topk, w.heads)
    torch.cuda.synchronize()
    ref = oracle.attend_heads(inp["q"], inp["k"], inp["v"], idx.cpu().numpy(), w.n_win)
    try:
        for kname in ("gather_mma", "simt"):
            bra.set_attend_kernel(kname)
            out = bra.attend_heads(q, k, v, idx, w.n_win)
            out2, idx2 = bra.forward_heads(q, k, v, w.n_win, w.topk, w.heads)
            torch.cuda.synchronize()
            assert bra.check_device_error() == 0
            assert torch.equal(idx2, idx) and torch.equal(out2, out), kname
            check_output(host_values(out), ref, w.dtype, f"{w.name} per-head / {kname}")
        bra.set_attend_kernel("region_mma")
        with pytest.raises(RuntimeError):
            bra.attend_heads(q, k, v, idx, w.n_win)
    finally:
        bra.set_attend_kernel("auto")


# shapes the dense kernel takes with one routing-count plane per head (bf16, hd 32, R <= 64,
# H W <= 256): 4-token and one-token regions, two and eight 64-channel blocks
HEADS_DENSE = [WORKLOADS["stage3"].with_(B=4), WORKLOADS["stage4"].with_(B=4),
               _w("rs4_r16_c128", 3, 8, 8, 128, 4, 4, 5, "bf16")]


@pytest.mark.parametrize("w", HEADS_DENSE, ids=[w.name for w in HEADS_DENSE])
def test_heads_dense_kernel(w):
    inp, (q, k, v) = make(w)
    idx = bra.route_heads(q, k, w.n_win, w.topk, w.heads)
    torch.cuda.synchronize()
    ref = oracle.attend_heads(inp["q"], inp["k"], inp["v"], idx.cpu().numpy(), w.n_win)
    try:
        for kname in ("dense_mma", "simt"):
            bra.set_attend_kernel(kname)
            out = bra.attend_heads(q, k, v, idx, w.n_win)
            torch.cuda.synchronize()
            assert bra.check_device_error() == 0
            check_output(host_values(out), ref, w.dtype, f"{w.name} per-head / {kname}")
        # given rows with duplicates and one bad entry per row: skipped and flagged
        rng = np.random.Generator(np.random.PCG64(23))
        given = rng.integers(0, w.R, size=(w.B, w.heads, w.R, 3)).astype(np.int32)
        given[..., 2] = given[..., 0]
        gref = oracle.attend_heads(inp["q"], inp["k"], inp["v"], given, w.n_win)
        bad = np.concatenate([given, np.full((w.B, w.heads, w.R, 1), w.R, np.int32)], axis=-1)
        bra.set_attend_kernel("dense_mma")
        out = bra.attend_heads(q, k, v, torch.from_numpy(bad).cuda(), w.n_win)
        assert bra.check_device_error() == 4
        check_output(host_values(out), gref, w.dtype, f"{w.name} per-head dense, given rows")
    finally:
        bra.set_attend_kernel("auto")


def test_heads_topk_clamp_and_one_head():
    w = _w("clamp", 2, 16, 16, 64, 2, 4, 20, "bf16")  # topk 20 > R = 16: clamped to 16
    inp, (q, k, v) = make(w)
    out, idx = bra.forward_heads(q, k, v, w.n_win, w.topk, w.heads)
    assert idx.shape == (2, 2, 16, 16)
    check_routing_heads(idx.cpu().numpy(), inp["q"], inp["k"], w.n_win, w.topk, w.heads)
    check_output(host_values(out), oracle.attend_heads(inp["q"], inp["k"], inp["v"], idx.cpu().numpy(), w.n_win),
                 w.dtype, "clamped topk")
    # one head over all channels routes like the shared routing
    w1 = _w("one_head", 2, 16, 16, 64, 1, 4, 3, "bf16")
    inp, (q, k, v) = make(w1)
    assert torch.equal(bra.route_heads(q, k, 4, 3, 1)[:, 0], bra.route(q, k, 4, 3))


def test_attend_heads_given_rows_with_bad_entries():
    w = _w("given", 2, 16, 16, 64, 2, 4, 3, "bf16", "iid", 77)
    inp, (q, k, v) = make(w)
    rng = np.random.Generator(np.random.PCG64(8))
    good = rng.integers(0, w.R, size=(w.B, w.heads, w.R, w.topk)).astype(np.int32)
    ref = oracle.attend_heads(inp["q"], inp["k"], inp["v"], good, w.n_win)
    out = bra.attend_heads(q, k, v, torch.from_numpy(good).cuda(), w.n_win)
    assert bra.check_device_error() == 0
    check_output(host_values(out), ref, w.dtype, "given per-head rows")
    bad = np.concatenate([good, np.full((w.B, w.heads, w.R, 1), -5, np.int32)], axis=-1)
    out = bra.attend_heads(q, k, v, torch.from_numpy(bad).cuda(), w.n_win)
    assert bra.check_device_error() == 4
    check_output(host_values(out), ref, w.dtype, "bad entries skipped")


# ------------------------------------------------------------------ LePE

def _lepe_params(C, seed=5):
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.standard_normal((C, 5, 5)) * 0.2, rng.standard_normal(C) * 0.1


LEPE_SHAPES = [WORKLOADS["stage1"].with_(B=8), WORKLOADS["stage3"].with_(B=4), WORKLOADS["tiny_f32"],
               _w("odd_f32", 2, 7, 9, 12, 3, 1, 1, "f32"), _w("odd_bf16", 3, 13, 6, 40, 5, 1, 1, "bf16"),
               _w("ragged_bf16_c64", 3, 21, 13, 64, 2, 1, 1, "bf16")]


@pytest.mark.parametrize("w", LEPE_SHAPES, ids=[w.name for w in LEPE_SHAPES])
def test_lepe(w):
    inp, (x, _, _) = make(w)
    wt, bias = _lepe_params(w.C)
    y = bra.lepe(x, torch.from_numpy(wt).float().cuda(), torch.from_numpy(bias).float().cuda())
    ref = oracle.lepe(inp["q"], wt.astype(np.float32), bias.astype(np.float32))
    check_output(host_values(y), ref, w.dtype, f"{w.name} lepe")


@pytest.mark.parametrize("name", ["stage1", "stage2", "highres"])
def test_forward_lepe(name):
    w = WORKLOADS[name].with_(B=4 if name != "highres" else 1)
    inp, (q, k, v) = make(w)
    wt, bias = _lepe_params(w.C, 6)
    out, attn, idx = bra.forward_lepe(q, k, v, w.n_win, w.topk, w.heads, torch.from_numpy(wt).float().cuda(),
                                      torch.from_numpy(bias).float().cuda())
    torch.cuda.synchronize()
    gidx = idx.cpu().numpy()
    check_routing(gidx, inp["q"], inp["k"], w.n_win, w.topk)
    check_output(host_values(attn), oracle.attend(inp["q"], inp["k"], inp["v"], gidx, w.heads, w.n_win), w.dtype,
                 "attention")
    # the epilogue against the oracle's LePE of the attention output the GPU wrote
    ref = oracle.lepe(host_values(attn), wt.astype(np.float32), bias.astype(np.float32))
    check_output(host_values(out), ref, w.dtype, f"{name} forward + lepe")


# ------------------------------------------------------------------ backward

BACK_SHAPES = [WORKLOADS["stage1"].with_(B=2), WORKLOADS["stage2"].with_(B=2), WORKLOADS["stage3"].with_(B=2),
               WORKLOADS["stage4"].with_(B=2), WORKLOADS["highres"].with_(B=1), WORKLOADS["tiny_f32"],
               _w("rs15_f32", 2, 12, 20, 32, 4, 4, 3, "f32"), _w("hd64_bf16", 1, 16, 16, 128, 2, 4, 3, "bf16"),
               # 64-token regions of 32-channel heads in fp32: the register-tiled CUDA-core kernel
               _w("rs64_f32", 2, 32, 32, 64, 2, 4, 3, "f32"), _w("rs64_f32_topk1", 3, 24, 24, 64, 2, 3, 1, "f32")]


@pytest.mark.parametrize("w", BACK_SHAPES, ids=[w.name for w in BACK_SHAPES])
def test_backward(w):
    inp, (q, k, v) = make(w)
    rng = np.random.Generator(np.random.PCG64(11))
    dout32 = rng.standard_normal((w.B, w.H, w.W, w.C)).astype(np.float32)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dout = torch.from_numpy(dout32).to(dt).cuda()
    idx = bra.route(q, k, w.n_win, w.topk)
    gidx = idx.cpu().numpy()
    dq, dk, dv = bra.attend_backward(q, k, v, idx, dout, w.heads, w.n_win)
    torch.cuda.synchronize()
    assert bra.check_device_error() == 0
    rq, rk, rv = oracle.attend_backward(inp["q"], inp["k"], inp["v"], gidx, host_values(dout), w.heads, w.n_win)
    for g, r, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        check_grad(g.cpu().numpy(), r, f"{w.name} {n}")


MANY_ITEMS = [WORKLOADS["stage1"].with_(B=24), WORKLOADS["highres"].with_(B=2)]


@pytest.mark.parametrize("w", MANY_ITEMS, ids=[w.name for w in MANY_ITEMS])
def test_backward_many_items_per_cta(w):
    """Batches large enough that each CTA of the tensor-core kernel (a persistent grid of a few
    CTAs per SM) takes several (image, region, head) items in turn, with one routed region
    (stage1, B = 24: 2352 items) and with four (highres, B = 2: 1024 items); every element."""
    inp, (q, k, v) = make(w)
    rng = np.random.Generator(np.random.PCG64(19))
    dout = torch.from_numpy(rng.standard_normal((w.B, w.H, w.W, w.C)).astype(np.float32)).to(torch.bfloat16).cuda()
    idx = bra.route(q, k, w.n_win, w.topk)
    dq, dk, dv = bra.attend_backward(q, k, v, idx, dout, w.heads, w.n_win)
    torch.cuda.synchronize()
    assert bra.check_device_error() == 0
    rq, rk, rv = oracle.attend_backward(inp["q"], inp["k"], inp["v"], idx.cpu().numpy(), host_values(dout), w.heads,
                                        w.n_win)
    for g, r, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        check_grad(g.cpu().numpy(), r, f"{w.name} B={w.B} {n}")


def test_backward_duplicates():
    w = _w("dup", 2, 16, 16, 64, 2, 4, 4, "bf16", "iid", 12)
    inp, (q, k, v) = make(w)
    rng = np.random.Generator(np.random.PCG64(13))
    idx = rng.integers(0, w.R, size=(w.B, w.R, w.topk)).astype(np.int32)
    idx[:, :, -1] = idx[:, :, 0]
    dout = torch.from_numpy(rng.standard_normal((w.B, w.H, w.W, w.C)).astype(np.float32)).to(torch.bfloat16).cuda()
    dq, dk, dv = bra.attend_backward(q, k, v, torch.from_numpy(idx).cuda(), dout, w.heads, w.n_win)
    rq, rk, rv = oracle.attend_backward(inp["q"], inp["k"], inp["v"], idx, host_values(dout), w.heads, w.n_win)
    for g, r, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        check_grad(g.cpu().numpy(), r, f"duplicates {n}")


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_backward_many_regions_and_bad_entries(dt):
    """The kernels of 64-token regions (tensor cores for bf16, register tiles for fp32): 18 routed
    regions (past the 16 they keep in shared memory), duplicates, then one out-of-range entry
    that is skipped and flagged."""
    w = _w("rs64_r25", 2, 40, 40, 64, 2, 5, 18, dt, "iid", 21)
    inp, (q, k, v) = make(w)
    rng = np.random.Generator(np.random.PCG64(17))
    idx = rng.integers(0, w.R, size=(w.B, w.R, w.topk)).astype(np.int32)
    idx[:, :, 5] = idx[:, :, 17]
    dout = torch.from_numpy(rng.standard_normal((w.B, w.H, w.W, w.C)).astype(np.float32)).to(q.dtype).cuda()
    rq, rk, rv = oracle.attend_backward(inp["q"], inp["k"], inp["v"], idx, host_values(dout), w.heads, w.n_win)
    dq, dk, dv = bra.attend_backward(q, k, v, torch.from_numpy(idx).cuda(), dout, w.heads, w.n_win)
    assert bra.check_device_error() == 0
    for g, r, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        check_grad(g.cpu().numpy(), r, f"{dt}, 18 regions {n}")
    for at in (9, 0):  # an out-of-range entry in the middle, and first (the region loaded with the item)
        bad = np.concatenate([idx[:, :, :at], np.full((w.B, w.R, 1), -3, np.int32), idx[:, :, at:]], axis=-1)
        dq, dk, dv = bra.attend_backward(q, k, v, torch.from_numpy(bad).cuda(), dout, w.heads, w.n_win)
        assert bra.check_device_error() == 4
        for g, r, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
            check_grad(g.cpu().numpy(), r, f"{dt}, bad entry {at} skipped {n}")


# ------------------------------------------------------------------ auto_pad

PAD_SHAPES = [_w("stage1_54", 8, 54, 54, 64, 2, 7, 1, "bf16"), _w("stage2_27x30", 4, 27, 30, 128, 4, 7, 4, "bf16"),
              _w("stage3_13", 8, 13, 13, 256, 8, 7, 16, "bf16"), _w("tiny_25x26_f32", 1, 25, 26, 64, 2, 7, 4, "f32"),
              _w("highres_125", 1, 125, 121, 64, 2, 16, 4, "bf16"), _w("divisible", 2, 28, 28, 64, 2, 7, 4, "bf16"),
              _w("stage4_6x5", 8, 6, 5, 512, 16, 7, 49, "bf16", "iid"), _w("rs4_13x12_c64", 4, 13, 12, 64, 2, 7, 9, "bf16")]


@pytest.mark.parametrize("w", PAD_SHAPES, ids=[w.name for w in PAD_SHAPES])
def test_forward_auto_pad(w):
    inp, (q, k, v) = make(w)
    out, idx = bra.forward_auto_pad(q, k, v, w.n_win, w.topk, w.heads)
    torch.cuda.synchronize()
    assert bra.check_device_error() == 0
    gidx = idx.cpu().numpy()
    Hp, Wp = -(-w.H // w.n_win) * w.n_win, -(-w.W // w.n_win) * w.n_win
    pad = lambda x: np.pad(x, ((0, 0), (0, Hp - w.H), (0, Wp - w.W), (0, 0)))
    check_routing(gidx, pad(inp["q"]), pad(inp["k"]), w.n_win, w.topk)
    ref = oracle.attend_auto_pad(inp["q"], inp["k"], inp["v"], gidx, w.heads, w.n_win)
    check_output(host_values(out), ref, w.dtype, f"{w.name} auto_pad")
    if Hp == w.H and Wp == w.W:
        out0, idx0 = bra.forward(q, k, v, w.n_win, w.topk, w.heads)
        assert torch.equal(idx0, idx) and torch.equal(out0, out)
