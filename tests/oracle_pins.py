"""Pins of the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` handle and raises AssertionError when the
oracle disagrees with an independent statement of the same quantity:

* region means against a numpy reshape-and-average of the window partition (a different
  formulation of "从零构建BiFormer", §1 region_partition);
* affinities against numpy's matmul;
* top-k against a full numpy lexsort of the row (brute force), with forced ties, -0/+0
  and NaN;
* attention against dense N x N attention per head with a mask built from the routing
  index (multiplicity counts, so duplicated indices are covered);
* topk = R against global attention from torch's scaled_dot_product_attention;
* the identity index against non-overlapping window attention (torch SDPA per window);
* closed forms: rs = 1 and topk = 1 returns the routed token's value; constant values
  pass through; attention is linear in v; a worked 2x2 example with a tie
  (tests/golden/tie_break_2x2.json);
* invariance of the output to the order of a routing row;
* per-head routing against a numpy restatement (per-head window means, matmul / sqrt(head_dim),
  brute-force ranking, topk clamped to R) and, with one head, against the shared routing;
  per-head attention against masked dense attention with one mask per head;
* LePE against torch's depthwise conv2d (padding 2, bias) plus the input, and two closed forms;
* the backward pass against central finite differences of the forward oracle and against torch
  autograd of masked dense attention;
* auto_pad against numpy zero padding + window means + brute-force ranking + masked dense
  attention + crop, the ordinary forward on divisible sizes, and a one-token closed form.

The same functions run against mutated copies of the oracle in test_oracle_mutants.py, to
show that each plausible slip in the oracle fails at least one of them. Run as a script,
``python oracle_pins.py <path to liboracle.so>`` runs every pin and exits non-zero on the
first failure.
"""
from __future__ import annotations

import json
import math
import os
import sys

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
if os.path.dirname(_HERE) not in sys.path:
    sys.path.insert(0, os.path.dirname(_HERE))

TOL = 1e-11


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _close(a, b, tol=TOL, what=""):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = np.max(np.abs(a - b)) if a.size else 0.0
    scale = max(1.0, np.max(np.abs(b)) if b.size else 0.0)
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol * scale:.3e}"


# ---------------------------------------------------------------- independent restatements

def region_of_token(H, W, n_win):
    """[H*W] region id of every token in raster order: window (y // hr, x // wr), windows
    numbered row-major."""
    hr, wr = H // n_win, W // n_win
    ys, xs = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    return ((ys // hr) * n_win + (xs // wr)).reshape(-1)


def numpy_region_means(x, n_win):
    B, H, W, C = x.shape
    hr, wr = H // n_win, W // n_win
    return x.reshape(B, n_win, hr, n_win, wr, C).mean(axis=(2, 4)).reshape(B, n_win * n_win, C)


def numpy_topk(A, k):
    """Brute-force ranking of every row: lexsort by (NaN last, value descending, index)."""
    B, R, _ = A.shape
    out = np.empty((B, R, k), np.int64)
    s = np.arange(R)
    for b in range(B):
        for r in range(R):
            row = A[b, r]
            nan = np.isnan(row)
            neg = np.where(nan, 0.0, -row)
            order = np.lexsort((s, neg, nan))
            out[b, r] = order[:k]
    return out


def masked_dense_attention(q, k, v, idx, heads, n_win):
    """Full N x N attention per head where key t' counts cnt[region(t), region(t')] times,
    cnt[r, s] = #{j : idx[r, j] = s}. Equal to BRA's gather-then-attend by the definition of
    softmax over a concatenated key list."""
    B, H, W, C = q.shape
    R, N, hd = n_win * n_win, H * W, C // heads
    reg = region_of_token(H, W, n_win)
    out = np.empty((B, N, C))
    for b in range(B):
        cnt = np.zeros((R, R))
        for r in range(R):
            for s in idx[b, r]:
                cnt[r, s] += 1
        weight = cnt[reg][:, reg]  # [N, N]
        qb, kb, vb = (t[b].reshape(N, C) for t in (q, k, v))
        for h in range(heads):
            sl = slice(h * hd, (h + 1) * hd)
            logits = (qb[:, sl] @ kb[:, sl].T) / math.sqrt(hd)
            logits = np.where(weight > 0, logits, -np.inf)
            p = weight * np.exp(logits - logits.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            out[b, :, sl] = p @ vb[:, sl]
    return out.reshape(B, H, W, C)


def torch_global_attention(q, k, v, heads):
    import torch
    B, H, W, C = q.shape
    hd = C // heads
    t = [torch.from_numpy(np.ascontiguousarray(x)).reshape(B, H * W, heads, hd).transpose(1, 2)
         for x in (q, k, v)]
    o = torch.nn.functional.scaled_dot_product_attention(*t)
    return o.transpose(1, 2).reshape(B, H, W, C).numpy()


def torch_window_attention(q, k, v, heads, n_win):
    import torch
    B, H, W, C = q.shape
    hr, wr, hd = H // n_win, W // n_win, C // heads

    def windows(x):
        x = torch.from_numpy(np.ascontiguousarray(x)).view(B, n_win, hr, n_win, wr, C)
        x = x.permute(0, 1, 3, 2, 4, 5).reshape(B * n_win * n_win, hr * wr, heads, hd)
        return x.transpose(1, 2)

    o = torch.nn.functional.scaled_dot_product_attention(windows(q), windows(k), windows(v))
    o = o.transpose(1, 2).reshape(B, n_win, n_win, hr, wr, C).permute(0, 1, 3, 2, 4, 5)
    return o.reshape(B, H, W, C).numpy()


# ---------------------------------------------------------------- the pins

def pin_region_means(orc):
    rng = _rng(11)
    for (B, H, W, C, n) in [(2, 6, 8, 5, 2), (1, 9, 6, 3, 3), (1, 4, 4, 2, 4), (1, 3, 5, 4, 1)]:
        x = rng.standard_normal((B, H, W, C))
        _close(orc.region_means(x, n), numpy_region_means(x, n), what=f"means {B,H,W,C,n}")


def pin_affinity(orc):
    rng = _rng(12)
    qm, km = rng.standard_normal((2, 9, 6)), rng.standard_normal((2, 9, 6))
    _close(orc.affinity(qm, km), np.matmul(qm, km.transpose(0, 2, 1)) / math.sqrt(6), what="affinity")


def pin_topk_bruteforce(orc):
    rng = _rng(13)
    # values from a small set force many exact ties; -0.0 and +0.0 must tie too
    A = rng.integers(-3, 4, size=(3, 40, 40)).astype(np.float64)
    A[0, 0, 5] = -0.0
    A[0, 0, 6] = 0.0
    A[1, 2, :] = np.nan
    A[1, 3, ::3] = np.nan
    A[2, 4, 7] = -np.inf
    A[2, 4, 8] = np.nan
    for k in (1, 5, 40):
        got = orc.topk(A, k)
        assert np.array_equal(got, numpy_topk(A, k)), f"topk k={k} differs from brute force"
    B2 = rng.standard_normal((2, 17, 17))
    assert np.array_equal(orc.topk(B2, 3), numpy_topk(B2, 3)), "topk on distinct values"


def pin_route_ties(orc):
    """Regions with identical key content tie exactly; the lower region wins."""
    rng = _rng(14)
    q = rng.standard_normal((1, 8, 8, 4))
    k = rng.standard_normal((1, 8, 8, 4))
    k[:, 4:6, 2:4, :] = k[:, 0:2, 2:4, :]  # region (2,1)=9 copies region (0,1)=1
    idx, A = orc.route(q, k, 4, 16, want_affinity=True)
    assert np.array_equal(A[..., 1], A[..., 9])
    for r in range(16):
        row = list(idx[0, r])
        assert row.index(1) < row.index(9), "tie must go to the lower region index"
    assert np.array_equal(idx, numpy_topk(np.matmul(numpy_region_means(q, 4),
                                                    numpy_region_means(k, 4).transpose(0, 2, 1)), 16))


def pin_masked_dense(orc):
    rng = _rng(15)
    for (B, H, W, C, heads, n, topk) in [(2, 6, 8, 8, 2, 2, 2), (1, 4, 4, 6, 3, 4, 3), (1, 9, 6, 4, 1, 3, 4)]:
        q, k, v = (rng.standard_normal((B, H, W, C)) for _ in range(3))
        R = n * n
        idx = np.stack([np.stack([rng.choice(R, topk, replace=False) for _ in range(R)]) for _ in range(B)])
        _close(orc.attend(q, k, v, idx, heads, n), masked_dense_attention(q, k, v, idx, heads, n),
               what=f"masked dense {B,H,W,C,heads,n,topk}")
        # duplicated regions in a row count once per occurrence (gather semantics)
        dup = idx.copy()
        dup[..., -1] = dup[..., 0]
        _close(orc.attend(q, k, v, dup, heads, n), masked_dense_attention(q, k, v, dup, heads, n),
               what="masked dense with duplicates")
        # and the routed path: route then attend equals masked dense over the oracle's own idx,
        # whose rows must also equal the brute-force ranking of numpy's affinities
        out, ridx = orc.forward(q, k, v, n, topk, heads)
        A = np.matmul(numpy_region_means(q, n), numpy_region_means(k, n).transpose(0, 2, 1)) / math.sqrt(C)
        assert np.array_equal(ridx, numpy_topk(A, topk)), "forward's routing differs from brute force"
        _close(out, masked_dense_attention(q, k, v, ridx, heads, n), what="forward")


def pin_global_attention(orc):
    rng = _rng(16)
    for (B, H, W, C, heads, n) in [(1, 9, 6, 4, 1, 3), (2, 4, 4, 8, 2, 4), (1, 6, 6, 12, 3, 2)]:
        q, k, v = (rng.standard_normal((B, H, W, C)) for _ in range(3))
        out, _ = orc.forward(q, k, v, n, n * n, heads)
        _close(out, torch_global_attention(q, k, v, heads), what=f"topk=R vs SDPA {B,H,W,C,heads,n}")


def pin_window_attention(orc):
    rng = _rng(17)
    for (B, H, W, C, heads, n) in [(2, 6, 8, 8, 2, 2), (1, 9, 6, 6, 3, 3)]:
        q, k, v = (rng.standard_normal((B, H, W, C)) for _ in range(3))
        R = n * n
        idx = np.broadcast_to(np.arange(R, dtype=np.int32)[None, :, None], (B, R, 1))
        _close(orc.attend(q, k, v, idx, heads, n), torch_window_attention(q, k, v, heads, n),
               what="identity idx vs window attention")


def pin_closed_forms(orc):
    rng = _rng(18)
    # one token per region, one routed region: softmax over a single key is 1
    B, H, W, C, heads, n = 2, 4, 4, 6, 3, 4
    q, k, v = (rng.standard_normal((B, H, W, C)) for _ in range(3))
    idx = rng.integers(0, 16, size=(B, 16, 1)).astype(np.int32)
    out = orc.attend(q, k, v, idx, heads, n)
    vflat = v.reshape(B, 16, C)  # with rs = 1, region r is token r
    _close(out.reshape(B, 16, C), np.take_along_axis(vflat, idx.astype(np.int64), axis=1),
           what="rs=1, topk=1")
    # constant values pass through any softmax
    B, H, W, C, heads, n, topk = 1, 6, 6, 4, 2, 3, 3
    q, k = rng.standard_normal((B, H, W, C)), rng.standard_normal((B, H, W, C))
    cval = rng.standard_normal(C)
    v = np.broadcast_to(cval, (B, H, W, C)).copy()
    out, _ = orc.forward(q, k, v, n, topk, heads)
    _close(out, v, what="constant v")
    # linear in v for a fixed routing
    v1, v2 = rng.standard_normal((B, H, W, C)), rng.standard_normal((B, H, W, C))
    idx = orc.route(q, k, n, topk)
    _close(orc.attend(q, k, v1 + 2.0 * v2, idx, heads, n),
           orc.attend(q, k, v1, idx, heads, n) + 2.0 * orc.attend(q, k, v2, idx, heads, n),
           what="linearity in v")


def pin_golden_2x2(orc):
    with open(os.path.join(_HERE, "golden", "tie_break_2x2.json")) as f:
        g = json.load(f)
    c = math.sqrt(2.0) * math.log(3.0)
    q = np.array(g["q_over_c"], np.float64).reshape(1, 2, 2, 2) * c
    k = np.array(g["k"], np.float64).reshape(1, 2, 2, 2)
    v = np.array(g["v"], np.float64).reshape(1, 2, 2, 2)
    out, idx = orc.forward(q, k, v, g["n_win"], g["topk"], g["heads"])
    assert idx.reshape(4, 2).tolist() == g["idx"], f"golden idx {idx.reshape(4, 2).tolist()}"
    vt = v.reshape(4, 2)
    expect = np.stack([(3.0 * vt[a] + vt[b]) / 4.0 for a, b in g["idx"]])
    _close(out.reshape(4, 2), expect, tol=1e-12, what="golden 2x2 weights 3/4, 1/4")


def pin_row_order_invariance(orc):
    rng = _rng(19)
    B, H, W, C, heads, n, topk = 2, 8, 8, 8, 2, 4, 5
    q, k, v = (rng.standard_normal((B, H, W, C)) for _ in range(3))
    idx = orc.route(q, k, n, topk)
    perm = np.stack([np.stack([rng.permutation(row) for row in img]) for img in idx])
    _close(orc.attend(q, k, v, idx, heads, n), orc.attend(q, k, v, perm, heads, n), what="row order")


def pin_attend_tokens(orc):
    rng = _rng(20)
    B, H, W, C, heads, n, topk = 2, 6, 8, 8, 2, 2, 3
    q, k, v = (rng.standard_normal((B, H, W, C)) for _ in range(3))
    idx = orc.route(q, k, n, topk)
    toks = np.array([0, 5, 47, 48, 95])
    full = orc.attend(q, k, v, idx, heads, n).reshape(B * H * W, C)
    _close(orc.attend_tokens(q, k, v, idx, heads, n, toks), full[toks], tol=0.0, what="attend_tokens")


# ---------------------------------------------------------------- per-head routing, LePE, backward, auto_pad

def numpy_route_heads(q, k, n_win, topk, heads):
    """Per-head routing restated with numpy: head h's region means are its head_dim channels of
    the window means, affinities (qm_h km_h^T) / sqrt(head_dim), rows ranked by brute force,
    min(topk, R) kept."""
    B, H, W, C = q.shape
    R, hd = n_win * n_win, C // heads
    qm = numpy_region_means(q, n_win).reshape(B, R, heads, hd).transpose(0, 2, 1, 3)
    km = numpy_region_means(k, n_win).reshape(B, R, heads, hd).transpose(0, 2, 1, 3)
    A = np.matmul(qm, km.transpose(0, 1, 3, 2)) / math.sqrt(hd)
    kk = min(topk, R)
    return numpy_topk(A.reshape(B * heads, R, R), kk).reshape(B, heads, R, kk), A


def masked_dense_attention_heads(q, k, v, idx, n_win):
    """masked_dense_attention with one index per head: idx [B, heads, R, topk]."""
    B, H, W, C = q.shape
    heads = idx.shape[1]
    hd = C // heads
    out = np.empty_like(np.asarray(q, np.float64))
    for h in range(heads):
        sl = slice(h * hd, (h + 1) * hd)
        out[..., sl] = masked_dense_attention(q[..., sl], k[..., sl], v[..., sl], idx[:, h], 1, n_win)
    return out


def pin_route_heads(orc):
    rng = _rng(21)
    for (B, H, W, C, heads, n, topk) in [(2, 6, 8, 8, 2, 2, 3), (1, 9, 6, 12, 3, 3, 4), (1, 8, 8, 6, 3, 4, 7)]:
        q, k = rng.standard_normal((B, H, W, C)), rng.standard_normal((B, H, W, C))
        idx, A = orc.route_heads(q, k, n, topk, heads, want_affinity=True)
        nidx, nA = numpy_route_heads(q, k, n, topk, heads)
        _close(A, nA, what=f"per-head affinity {B,H,W,C,heads,n}")
        assert np.array_equal(idx, nidx), "per-head routing differs from brute force"
    # topk above R is clamped to R: every row is the full ranking
    idx = orc.route_heads(q, k, 4, 20, 3)
    assert idx.shape == (1, 3, 16, 16) and np.array_equal(idx, numpy_route_heads(q, k, 4, 16, 3)[0])
    # one head over all channels is the shared routing (same scale C^-1/2)
    q, k = rng.standard_normal((2, 6, 6, 5)), rng.standard_normal((2, 6, 6, 5))
    idx1, A1 = orc.route_heads(q, k, 3, 4, 1, want_affinity=True)
    idx0, A0 = orc.route(q, k, 3, 4, want_affinity=True)
    assert np.array_equal(idx1[:, 0], idx0)
    _close(A1[:, 0], A0, what="one head = shared routing")


def pin_attend_heads(orc):
    rng = _rng(22)
    for (B, H, W, C, heads, n, topk) in [(2, 6, 8, 8, 2, 2, 2), (1, 9, 6, 6, 3, 3, 4)]:
        q, k, v = (rng.standard_normal((B, H, W, C)) for _ in range(3))
        R = n * n
        idx = rng.integers(0, R, size=(B, heads, R, topk)).astype(np.int32)
        _close(orc.attend_heads(q, k, v, idx, n), masked_dense_attention_heads(q, k, v, idx, n),
               what=f"per-head masked dense {B,H,W,C,heads,n,topk}")
        # every head given the same rows: the shared-index attention
        same = np.repeat(idx[:, :1], heads, axis=1)
        _close(orc.attend_heads(q, k, v, same, n), orc.attend(q, k, v, idx[:, 0], heads, n), what="same rows")
        # per-head routing end to end against masked dense over the brute-force index
        ridx = orc.route_heads(q, k, n, topk, heads)
        _close(orc.attend_heads(q, k, v, ridx, n),
               masked_dense_attention_heads(q, k, v, numpy_route_heads(q, k, n, topk, heads)[0], n),
               what="per-head route + attend")


def torch_lepe(x, w, bias):
    import torch
    B, H, W, C = x.shape
    t = torch.from_numpy(np.ascontiguousarray(x)).permute(0, 3, 1, 2)
    conv = torch.nn.functional.conv2d(t, torch.from_numpy(np.ascontiguousarray(w)).reshape(C, 1, 5, 5),
                                      torch.from_numpy(np.ascontiguousarray(bias)), padding=2, groups=C)
    return (t + conv).permute(0, 2, 3, 1).numpy()


def pin_lepe(orc):
    rng = _rng(23)
    for (B, H, W, C) in [(2, 7, 9, 3), (1, 4, 3, 5), (1, 1, 6, 2)]:
        x, w, bias = rng.standard_normal((B, H, W, C)), rng.standard_normal((C, 5, 5)), rng.standard_normal(C)
        _close(orc.lepe(x, w, bias), torch_lepe(x, w, bias), what=f"lepe vs torch conv2d {B,H,W,C}")
    # a filter that is 1 at the centre doubles x; a zero filter adds the bias
    x = rng.standard_normal((1, 5, 6, 4))
    centre = np.zeros((4, 5, 5))
    centre[:, 2, 2] = 1.0
    _close(orc.lepe(x, centre, np.zeros(4)), 2.0 * x, what="centre tap")
    bias = rng.standard_normal(4)
    _close(orc.lepe(x, np.zeros((4, 5, 5)), bias), x + bias, what="bias only")


def torch_masked_attention_grads(q, k, v, idx, dout, heads, n_win):
    """Gradients of sum(dout * masked dense attention) by torch autograd, float64."""
    import torch
    B, H, W, C = q.shape
    R, N, hd = n_win * n_win, H * W, C // heads
    reg = torch.from_numpy(region_of_token(H, W, n_win))
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x)).requires_grad_(True) for x in (q, k, v))
    outs = []
    for b in range(B):
        cnt = torch.zeros((R, R), dtype=torch.float64)
        for r in range(R):
            for s in idx[b, r]:
                cnt[r, s] += 1
        weight = cnt[reg][:, reg]
        qb, kb, vb = (t[b].reshape(N, C) for t in (tq, tk, tv))
        heads_out = []
        for h in range(heads):
            sl = slice(h * hd, (h + 1) * hd)
            logits = (qb[:, sl] @ kb[:, sl].T) / math.sqrt(hd)
            logits = torch.where(weight > 0, logits, torch.tensor(-math.inf, dtype=torch.float64))
            p = weight * torch.exp(logits - logits.max(dim=1, keepdim=True).values)
            p = p / p.sum(dim=1, keepdim=True)
            heads_out.append(p @ vb[:, sl])
        outs.append(torch.cat(heads_out, dim=1))
    out = torch.stack(outs).reshape(B, H, W, C)
    (out * torch.from_numpy(np.ascontiguousarray(dout))).sum().backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


def pin_backward(orc):
    rng = _rng(24)
    # central differences of sum(dout * out) on every coordinate of a tiny case
    B, H, W, C, heads, n, topk = 1, 4, 4, 4, 2, 2, 2
    q, k, v = (rng.standard_normal((B, H, W, C)) for _ in range(3))
    idx = rng.integers(0, n * n, size=(B, n * n, topk)).astype(np.int32)
    dout = rng.standard_normal((B, H, W, C))
    grads = orc.attend_backward(q, k, v, idx, dout, heads, n)
    eps = 1e-6
    for which, g in enumerate(grads):
        num = np.zeros_like(g)
        for i in range(g.size):
            args = [q.copy(), k.copy(), v.copy()]
            args[which].reshape(-1)[i] += eps
            fp = np.sum(dout * orc.attend(*args, idx, heads, n))
            args[which].reshape(-1)[i] -= 2 * eps
            fm = np.sum(dout * orc.attend(*args, idx, heads, n))
            num.reshape(-1)[i] = (fp - fm) / (2 * eps)
        _close(g, num, tol=1e-7, what=f"finite differences of {'qkv'[which]}")
    # torch autograd of masked dense attention, duplicated regions included
    B, H, W, C, heads, n, topk = 2, 6, 8, 8, 2, 2, 3
    q, k, v, dout = (rng.standard_normal((B, H, W, C)) for _ in range(4))
    idx = rng.integers(0, n * n, size=(B, n * n, topk)).astype(np.int32)
    idx[:, :, -1] = idx[:, :, 0]
    for g, t, name in zip(orc.attend_backward(q, k, v, idx, dout, heads, n),
                          torch_masked_attention_grads(q, k, v, idx, dout, heads, n), "qkv"):
        _close(g, t, what=f"autograd d{name}")


def pin_auto_pad(orc):
    rng = _rng(25)
    # sizes that divide: the ordinary forward pass
    q, k, v = (rng.standard_normal((2, 6, 9, 4)) for _ in range(3))
    out, idx = orc.forward_auto_pad(q, k, v, 3, 2, 2)
    out0, idx0 = orc.forward(q, k, v, 3, 2, 2)
    assert np.array_equal(idx, idx0)
    _close(out, out0, tol=0.0, what="auto_pad on divisible sizes")
    # numpy: zero padding at the bottom and right, window means over the padded windows,
    # brute-force ranking, masked dense attention, crop
    for (B, H, W, C, heads, n, topk) in [(2, 5, 7, 4, 2, 3, 2), (1, 9, 4, 6, 3, 4, 5), (1, 3, 3, 2, 1, 2, 4)]:
        q, k, v = (rng.standard_normal((B, H, W, C)) for _ in range(3))
        Hp, Wp = -(-H // n) * n, -(-W // n) * n
        pad = lambda x: np.pad(x, ((0, 0), (0, Hp - H), (0, Wp - W), (0, 0)))
        qp, kp, vp = pad(q), pad(k), pad(v)
        A = np.matmul(numpy_region_means(qp, n), numpy_region_means(kp, n).transpose(0, 2, 1)) / math.sqrt(C)
        nidx = numpy_topk(A, topk)
        out, idx = orc.forward_auto_pad(q, k, v, n, topk, heads)
        assert np.array_equal(idx, nidx), f"auto_pad routing {B,H,W,C,n}"
        _close(out, masked_dense_attention(qp, kp, vp, nidx, heads, n)[:, :H, :W],
               what=f"auto_pad {B,H,W,C,heads,n,topk}")
        _close(orc.attend_auto_pad(q, k, v, idx, heads, n), out, tol=0.0, what="attend_auto_pad")
    # one real token in a 2 x 2 grid of one-token regions: its three routed neighbours are zero
    # keys (logit 0) with zero values, so out = e^l / (e^l + 3) v, l = q . k / sqrt(C)
    q, k, v = (rng.standard_normal((1, 1, 1, 3)) for _ in range(3))
    out, idx = orc.forward_auto_pad(q, k, v, 2, 4, 1)
    l = float(q.ravel() @ k.ravel()) / math.sqrt(3)
    _close(out, math.exp(l) / (math.exp(l) + 3.0) * v, tol=1e-14, what="one token, three zero keys")


PINS = [pin_region_means, pin_affinity, pin_topk_bruteforce, pin_route_ties, pin_masked_dense,
        pin_global_attention, pin_window_attention, pin_closed_forms, pin_golden_2x2,
        pin_row_order_invariance, pin_attend_tokens, pin_route_heads, pin_attend_heads, pin_lepe,
        pin_backward, pin_auto_pad]


def run_all(orc):
    for pin in PINS:
        pin(orc)


if __name__ == "__main__":
    import oracle
    run_all(oracle.Oracle(sys.argv[1]))
    print("all pins hold")
