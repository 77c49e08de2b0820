"""CUDA path against the CPU oracle, through the C ABI (via the ctypes binding)."""
import json
import os

import numpy as np
import pytest
import torch

import bi_level_routing_b200 as bra
import oracle
from bi_level_routing_b200.workloads import WORKLOADS, Workload, make_inputs
from parity import check_output, check_routing, device_tensors, host_values, make, value_relative_rejects

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _auto_kernel():
    bra.set_attend_kernel("auto")
    yield
    bra.set_attend_kernel("auto")


# ------------------------------------------------------------------ the named workloads, full size

def _report(key: str, value: dict):
    """Adds a line to the JSON parity report named by $BRA_PARITY_REPORT (when set)."""
    path = os.environ.get("BRA_PARITY_REPORT")
    if not path:
        return
    data = {}
    if os.path.exists(path):
        with open(path) as f:
            data = json.load(f)
    data[key] = value
    with open(path, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_forward_full_size(name):
    """bra_forward at full size, in the configuration the benchmark times: every routing row
    checked (bit-exact outside near-ties) and every output element compared with the oracle's
    attention over the GPU's own index."""
    w = WORKLOADS[name]
    inp, (q, k, v) = make(w)
    out, idx = bra.forward(q, k, v, w.n_win, w.topk, w.heads)
    torch.cuda.synchronize()
    assert bra.check_device_error() == 0
    gidx = idx.cpu().numpy()
    orc_idx, near = check_routing(gidx, inp["q"], inp["k"], w.n_win, w.topk)
    assert near <= max(2, gidx.shape[0] * gidx.shape[1] // 1000), f"{near} near-tie rows"
    _, A = oracle.route(inp["q"], inp["k"], w.n_win, w.topk, want_affinity=True)
    strict = value_relative_rejects(gidx, orc_idx, A)
    ref = oracle.attend(inp["q"], inp["k"], inp["v"], gidx, w.heads, w.n_win)
    got = host_values(out)
    err = check_output(got, ref, w.dtype, f"{name} every element")
    _report(f"full_size/{name}", {"rows": int(gidx.shape[0] * gidx.shape[1]), "near_tie_rows": int(near),
                                  "value_relative_rejects": int(strict), "max_abs_err": err,
                                  "max_abs_oracle": float(np.abs(ref).max()), "elements": int(ref.size)})
    assert strict == 0, f"{strict} near-tie rows would fail a tolerance relative to the affinity values"


# ------------------------------------------------------------------ many work items per CTA, every element

# The persistent kernels split a call's work items evenly over their CTAs; with the grid capped
# at a few CTAs each one runs many consecutive items, so the state carried from item to item
# (ring slots and phases, the running softmax of the previous item, the deferred store) is
# exercised on inputs small enough to compare element by element.
MULTI = [
    # name, B, H, W, C, heads, n_win, topk, dtype, grid cap
    ("stage1_b2_topk1", 2, 56, 56, 64, 2, 7, 1, "bf16", 3),
    ("stage1_b2_topk4", 2, 56, 56, 64, 2, 7, 4, "bf16", 5),
    ("highres_b1_topk4", 1, 128, 128, 64, 2, 16, 4, "bf16", 7),
    ("rs64_c128_topk3", 2, 32, 32, 128, 4, 4, 3, "bf16", 2),
    ("stage2_b2", 2, 28, 28, 128, 4, 7, 4, "bf16", 3),
    ("rs16_c64_topk7", 3, 16, 16, 64, 2, 4, 7, "bf16", 4),
]


@pytest.mark.parametrize("spec", MULTI, ids=[s[0] for s in MULTI])
def test_many_items_per_cta(spec):
    *shape, cap = spec
    w = _small(tuple(shape))
    inp, (q, k, v) = make(w)
    idx = bra.route(q, k, w.n_win, w.topk)
    torch.cuda.synchronize()
    gidx = idx.cpu().numpy()
    check_routing(gidx, inp["q"], inp["k"], w.n_win, w.topk)
    ref = oracle.attend(inp["q"], inp["k"], inp["v"], gidx, w.heads, w.n_win)
    kernels = [kn for kn in _kernels_for(w) if kn in ("gather_umma", "gather_mma")]
    assert kernels, "no persistent kernel serves this shape"
    try:
        for kname in kernels:
            bra.set_attend_kernel(kname)
            for c in (cap, 1):
                bra.set_max_ctas(c)
                out = bra.attend(q, k, v, idx, w.heads, w.n_win)
                torch.cuda.synchronize()
                assert bra.check_device_error() == 0
                check_output(host_values(out), ref, w.dtype, f"{w.name} / {kname} / {c} CTAs")
    finally:
        bra.set_max_ctas(0)
        bra.set_attend_kernel("auto")


# ------------------------------------------------------------------ small shapes, every element

SMALL = [
    # name, B, H, W, C, heads, n_win, topk, dtype
    ("rect_rs15_bf16", 3, 12, 20, 64, 2, 4, 3, "bf16"),
    ("rs64_ring_bf16", 2, 32, 32, 128, 4, 4, 5, "bf16"),
    ("rs48_c192_bf16", 2, 16, 48, 192, 6, 4, 2, "bf16"),
    ("rs16_c320_bf16", 1, 8, 8, 320, 10, 2, 4, "bf16"),
    ("rs16_stage2_bf16", 2, 28, 28, 128, 4, 7, 4, "bf16"),
    ("rs4_stage3_bf16", 3, 14, 14, 256, 8, 7, 16, "bf16"),
    ("rs1_bf16", 2, 8, 8, 64, 2, 8, 5, "bf16"),
    ("one_region_bf16", 2, 8, 8, 64, 2, 1, 1, "bf16"),
    ("hd4_f32", 2, 9, 15, 12, 3, 3, 2, "f32"),
    ("hd64_f32", 1, 16, 16, 128, 2, 4, 3, "f32"),
    ("hd64_bf16", 1, 16, 16, 128, 2, 4, 3, "bf16"),
    ("hd128_bf16", 1, 8, 8, 256, 2, 2, 2, "bf16"),
    ("tiny_f32", 1, 28, 28, 64, 2, 7, 4, "f32"),
    ("max_regions_bf16", 1, 32, 32, 8, 1, 32, 7, "bf16"),
    ("topk_all_256_bf16", 1, 16, 16, 32, 1, 16, 256, "bf16"),
    # 64-token regions, 64 channels (the tcgen05 kernel) with topk > 1
    ("rs64_c64_bf16", 3, 32, 32, 64, 2, 4, 3, "bf16"),
    ("stage1_topk4_bf16", 2, 56, 56, 64, 2, 7, 4, "bf16"),
    # one-token regions in bf16 (the tensor-core routing kernel): ragged key tiles and row
    # blocks with a full sort, one 32-channel chunk, argmax rounds over 512 channels
    ("rs1_r25_c96_bf16", 3, 5, 5, 96, 3, 5, 25, "bf16"),
    ("rs1_r64_c32_bf16", 2, 8, 8, 32, 1, 8, 64, "bf16"),
    ("rs1_r49_c512_topk3_bf16", 2, 7, 7, 512, 16, 7, 3, "bf16"),
    # 64 < R <= 256 with fp32 means (the key-split 3xTF32 routing kernel): E = 4 and E = 8
    ("r100_rs4_f32", 2, 20, 20, 32, 1, 10, 7, "f32"),
    ("r144_rs4_bf16", 2, 24, 24, 64, 2, 12, 20, "bf16"),
    # 4-token regions in bf16 (the stacked-head kernel): 1 x 4 regions with padded keys, and
    # 160 routed keys in three chunks of the online softmax
    ("rs4_1x4_c128_bf16", 2, 4, 16, 128, 4, 4, 3, "bf16"),
    ("rs4_topk40_c256_bf16", 1, 16, 16, 256, 8, 8, 40, "bf16"),
]


def _small(spec, values="region_offset", seed=1234):
    name, B, H, W, C, heads, n, topk, dt = spec
    return Workload(name, B, H, W, C, heads, n, topk, dt, values, seed)


def _kernels_for(w):
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    out = []
    for kname in ("simt", "gather_mma", "dense_mma", "gather_umma", "region_mma"):
        bra.set_attend_kernel(kname)
        if bra.selected_attend_kernel(w.B, w.H, w.W, w.C, w.heads, w.n_win, w.topk, dt) == kname:
            out.append(kname)
    bra.set_attend_kernel("auto")
    return out


@pytest.mark.parametrize("spec", SMALL, ids=[s[0] for s in SMALL])
def test_small_shapes_every_kernel(spec):
    w = _small(spec)
    inp, (q, k, v) = make(w)
    idx = bra.route(q, k, w.n_win, w.topk)
    torch.cuda.synchronize()
    gidx = idx.cpu().numpy()
    check_routing(gidx, inp["q"], inp["k"], w.n_win, w.topk)
    ref = oracle.attend(inp["q"], inp["k"], inp["v"], gidx, w.heads, w.n_win)
    kernels = _kernels_for(w)
    assert kernels, "no kernel serves this shape"
    for kname in kernels:
        bra.set_attend_kernel(kname)
        out = bra.attend(q, k, v, idx, w.heads, w.n_win)
        torch.cuda.synchronize()
        assert bra.check_device_error() == 0
        check_output(host_values(out), ref, w.dtype, f"{w.name} / {kname}")
    bra.set_attend_kernel("auto")
    out, idx2 = bra.forward(q, k, v, w.n_win, w.topk, w.heads)
    assert torch.equal(idx2, idx), "forward's routing differs from route's"
    check_output(host_values(out), ref, w.dtype, f"{w.name} / forward")


# ------------------------------------------------------------------ given indices: duplicates, order, bad entries

GIVEN = [("rs64_bf16", 2, 16, 16, 64, 2, 2, 3, "bf16"),
         ("rs16_bf16", 2, 16, 16, 128, 4, 4, 4, "bf16"),
         ("rs4_bf16", 2, 14, 14, 128, 4, 7, 6, "bf16"),
         ("rs9_f32", 2, 12, 12, 16, 2, 4, 3, "f32")]


@pytest.mark.parametrize("spec", GIVEN, ids=[s[0] for s in GIVEN])
def test_duplicates_and_row_order(spec):
    w = _small(spec, values="iid", seed=99)
    inp, (q, k, v) = make(w)
    rng = np.random.Generator(np.random.PCG64(5))
    R = w.R
    dup = rng.integers(0, R, size=(w.B, R, w.topk)).astype(np.int32)
    dup[:, :, -1] = dup[:, :, 0]  # at least one duplicate per row
    ref = oracle.attend(inp["q"], inp["k"], inp["v"], dup, w.heads, w.n_win)
    perm = np.ascontiguousarray(dup[:, :, rng.permutation(w.topk)])
    for kname in _kernels_for(w):
        bra.set_attend_kernel(kname)
        out = bra.attend(q, k, v, torch.from_numpy(dup).cuda(), w.heads, w.n_win)
        out_p = bra.attend(q, k, v, torch.from_numpy(perm).cuda(), w.heads, w.n_win)
        torch.cuda.synchronize()
        check_output(host_values(out), ref, w.dtype, f"duplicates / {kname}")
        check_output(host_values(out_p), ref, w.dtype, f"permuted / {kname}")
    assert bra.check_device_error() == 0


@pytest.mark.parametrize("spec", GIVEN, ids=[s[0] for s in GIVEN])
def test_out_of_range_entries_are_skipped_and_flagged(spec):
    w = _small(spec, values="iid", seed=77)
    inp, (q, k, v) = make(w)
    rng = np.random.Generator(np.random.PCG64(6))
    good = np.stack([np.stack([rng.choice(w.R, w.topk - 1, replace=False) for _ in range(w.R)])
                     for _ in range(w.B)]).astype(np.int32)
    bad = np.concatenate([good, np.full((w.B, w.R, 1), w.R + 3, np.int32)], axis=-1)
    bad[:, ::2, -1] = -1
    ref = oracle.attend(inp["q"], inp["k"], inp["v"], good, w.heads, w.n_win)
    for kname in _kernels_for(w):
        bra.set_attend_kernel(kname)
        assert bra.check_device_error() == 0
        out = bra.attend(q, k, v, torch.from_numpy(bad).cuda(), w.heads, w.n_win)
        assert bra.check_device_error() == 4, f"{kname} did not flag BRA_ERR_INDEX"
        assert bra.check_device_error() == 0, "the error word must clear after reading"
        check_output(host_values(out), ref, w.dtype, f"bad entries skipped / {kname}")


# ------------------------------------------------------------------ routing edge cases

def test_route_exact_ties_go_to_the_lower_region():
    w = Workload("ties", 2, 16, 16, 64, 2, 4, 16, "bf16", "region_offset", 4321)
    inp = make_inputs(w)
    for t in ("k_bits", "k"):  # region (1,2)=6 and region (3,0)=12 copy region (0,1)=1
        inp[t][:, 4:8, 8:12, :] = inp[t][:, 0:4, 4:8, :]
        inp[t][:, 12:16, 0:4, :] = inp[t][:, 0:4, 4:8, :]
    q, k, _ = device_tensors(inp, w)
    gidx = bra.route(q, k, w.n_win, w.topk).cpu().numpy()
    orc = oracle.route(inp["q"], inp["k"], w.n_win, w.topk)
    assert np.array_equal(gidx, orc)
    for b in range(w.B):
        for r in range(w.R):
            row = list(gidx[b, r])
            assert row.index(1) < row.index(6) < row.index(12)


def test_route_exact_ties_one_token_regions():
    """One-token regions (routed on the tensor cores in bf16): keys that are copies of one another
    give exactly equal affinities in every row, and the lower region ranks first."""
    w = Workload("ties1", 2, 7, 7, 512, 16, 7, 49, "bf16", "iid", 4324)
    inp = make_inputs(w)
    for t in ("k_bits", "k"):  # regions (1,2)=9 and (4,2)=30 copy region (0,3)=3
        inp[t][:, 1, 2, :] = inp[t][:, 0, 3, :]
        inp[t][:, 4, 2, :] = inp[t][:, 0, 3, :]
    q, k, _ = device_tensors(inp, w)
    gidx = bra.route(q, k, w.n_win, w.topk).cpu().numpy()
    check_routing(gidx, inp["q"], inp["k"], w.n_win, w.topk)
    for b in range(w.B):
        for r in range(w.R):
            row = list(gidx[b, r])
            i3, i9, i30 = row.index(3), row.index(9), row.index(30)
            assert i9 == i3 + 1 and i30 == i3 + 2, (b, r, row)


def test_route_nan_ranks_last_one_token_regions():
    w = Workload("nan1", 1, 7, 7, 64, 2, 7, 49, "bf16", "iid", 4325)
    inp = make_inputs(w)
    inp["k"][0, 2, 3, 5] = np.nan  # token (2,3) = region 17: column 17 is NaN in every row
    inp["k_bits"][0, 2, 3, 5] = 0x7FC0
    q, k, _ = device_tensors(inp, w)
    gidx = bra.route(q, k, w.n_win, w.topk).cpu().numpy()
    assert np.all(gidx[0, :, -1] == 17)
    check_routing(gidx, inp["q"], inp["k"], w.n_win, w.topk)


def test_route_nan_ranks_last():
    w = Workload("nan", 1, 16, 16, 64, 2, 4, 16, "f32", "region_offset", 4322)
    inp = make_inputs(w)
    inp["k"][0, 4, 4, 3] = np.nan  # region (1,1) = 5 gets a NaN mean: column 5 is NaN in every row
    q, k, _ = device_tensors(inp, w)
    gidx = bra.route(q, k, w.n_win, w.topk).cpu().numpy()
    orc = oracle.route(inp["q"], inp["k"], w.n_win, w.topk)
    assert np.array_equal(gidx, orc)
    assert np.all(gidx[0, :, -1] == 5)


def test_empty_batch():
    q = torch.empty((0, 8, 8, 64), dtype=torch.bfloat16, device="cuda")
    out, idx = bra.forward(q, q, q, 2, 2, 2)
    assert out.shape == (0, 8, 8, 64) and idx.shape == (0, 4, 2)


def test_side_stream_and_host_entry_point():
    w = WORKLOADS["stage2"].with_(B=4)
    inp, (q, k, v) = make(w)
    ref_out, ref_idx = bra.forward(q, k, v, w.n_win, w.topk, w.heads)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out, idx = bra.forward(q, k, v, w.n_win, w.topk, w.heads)
    s.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(idx, ref_idx)
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hout, hidx = bra.forward_host(hq, hk, hv, w.n_win, w.topk, w.heads)
    assert torch.equal(hout, ref_out.cpu()) and torch.equal(hidx, ref_idx.cpu())


def test_host_entry_point_in_chunks():
    """bra_forward_host splits the batch into chunks whose copies overlap the computation: B = 5
    gives chunks of 2, 1, 1 and 1 images; every chunk must equal bra_forward on the whole batch."""
    w = WORKLOADS["stage1"].with_(B=5)
    inp, (q, k, v) = make(w)
    ref_out, ref_idx = bra.forward(q, k, v, w.n_win, w.topk, w.heads)
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hout, hidx = bra.forward_host(hq, hk, hv, w.n_win, w.topk, w.heads)
    assert torch.equal(hout, ref_out.cpu()) and torch.equal(hidx, ref_idx.cpu())
    # pageable host memory works too
    hout2, hidx2 = bra.forward_host(q.cpu(), k.cpu(), v.cpu(), w.n_win, w.topk, w.heads)
    assert torch.equal(hout2, ref_out.cpu()) and torch.equal(hidx2, ref_idx.cpu())


def test_repeatable():
    """Same inputs, same bits: the kernels use no atomics in their arithmetic."""
    w = WORKLOADS["highres"].with_(B=2)
    _, (q, k, v) = make(w)
    a = bra.forward(q, k, v, w.n_win, w.topk, w.heads)
    b = bra.forward(q, k, v, w.n_win, w.topk, w.heads)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
