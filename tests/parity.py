"""Comparison rules between the CUDA path and the CPU oracle.

Routing indices: bit-exact, except at near-ties. A GPU row is accepted when it holds topk
distinct regions in [0, R) and, at every position j, the oracle's affinity of the GPU's
region equals the oracle's j-th largest affinity within
    tol = 1e-5 * C^-1/2 * max(sum_c |qm_r,c km_a,c|, sum_c |qm_r,c km_b,c|)
(a relative tolerance measured against the size of the dot product's terms, which is what
bounds its rounding error). Wherever the k-th and (k+1)-th affinities are further apart
than that, this is bit-exact equality. The output is always compared against the oracle
run on the GPU's own indices.

Outputs: fp32 max |gpu - oracle| <= 1e-4; bf16 max |gpu - oracle| <= 2e-2 * max |oracle|
(the relative bound read normwise).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from bi_level_routing_b200.workloads import Workload, make_inputs

ROUTE_REL_TOL = 1e-5
F32_ABS_TOL = 1e-4
BF16_REL_TOL = 2e-2


def device_tensors(inp: dict, w: Workload, device="cuda"):
    """q, k, v as CUDA tensors holding exactly the generated values."""
    out = []
    for name in ("q", "k", "v"):
        if w.dtype == "bf16":
            t = torch.from_numpy(inp[name + "_bits"].view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(inp[name])
        out.append(t.to(device).contiguous())
    return out


def host_values(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_routing(gpu_idx: np.ndarray, q: np.ndarray, k: np.ndarray, n_win: int, topk: int):
    """Returns (oracle idx, number of rows accepted through a near-tie). Raises on a mismatch."""
    orc_idx, A = oracle.route(q, k, n_win, topk, want_affinity=True)
    gpu_idx = np.asarray(gpu_idx)
    assert gpu_idx.shape == orc_idx.shape, (gpu_idx.shape, orc_idx.shape)
    if np.array_equal(gpu_idx, orc_idx):
        return orc_idx, 0
    B, R, _ = orc_idx.shape
    C = q.shape[-1]
    qm, km = oracle.region_means(q, n_win), oracle.region_means(k, n_win)
    near = 0
    bad_rows = np.argwhere(np.any(gpu_idx != orc_idx, axis=-1))
    for b, r in bad_rows:
        row = gpu_idx[b, r]
        assert np.all((row >= 0) & (row < R)), f"row {b},{r}: index out of range {row}"
        assert len(set(row.tolist())) == topk, f"row {b},{r}: repeated region {row}"
        mag = np.abs(qm[b, r]) @ np.abs(km[b]).T / math.sqrt(C)  # [R] term magnitude per candidate
        for j in range(topk):
            a, o = row[j], orc_idx[b, r, j]
            if a == o:
                continue
            va, vo = A[b, r, a], A[b, r, o]
            tol = ROUTE_REL_TOL * max(mag[a], mag[o])
            assert abs(va - vo) <= tol or (np.isnan(va) and np.isnan(vo)), (
                f"row {b},{r} position {j}: GPU region {a} (affinity {va!r}) vs oracle region {o} "
                f"({vo!r}), difference {abs(va - vo):.3e} > tolerance {tol:.3e}")
        near += 1
    return orc_idx, near


def value_relative_rejects(gpu_idx: np.ndarray, orc_idx: np.ndarray, A: np.ndarray) -> int:
    """Rows the acceptance rule took as near-ties that a rule relative to the affinity VALUES,
    |A_gpu - A_orc| <= 1e-5 * max(|A_gpu|, |A_orc|) at every differing position, would reject
    (a report of how much looser the terms-magnitude measure is on real inputs)."""
    gpu_idx = np.asarray(gpu_idx)
    rejects = 0
    for b, r in np.argwhere(np.any(gpu_idx != orc_idx, axis=-1)):
        for a, o in zip(gpu_idx[b, r], orc_idx[b, r]):
            if a == o:
                continue
            va, vo = A[b, r, a], A[b, r, o]
            if not abs(va - vo) <= ROUTE_REL_TOL * max(abs(va), abs(vo)):
                rejects += 1
                break
    return rejects


def check_output(gpu: np.ndarray, ref: np.ndarray, dtype: str, what: str = "out"):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite values"
    err = float(np.max(np.abs(gpu - ref))) if gpu.size else 0.0
    if dtype == "f32":
        assert err <= F32_ABS_TOL, f"{what}: max abs err {err:.3e} > {F32_ABS_TOL}"
        return err
    bound = BF16_REL_TOL * float(np.max(np.abs(ref)))
    assert err <= bound, f"{what}: max abs err {err:.3e} > {bound:.3e} (2e-2 of max |oracle|)"
    return err


def make(w: Workload, seed=None):
    inp = make_inputs(w, seed)
    return inp, device_tensors(inp, w)


def check_routing_heads(gpu_idx: np.ndarray, q: np.ndarray, k: np.ndarray, n_win: int, topk: int, heads: int):
    """check_routing for per-head routing: idx [B, heads, R, k]; the tolerance of a near-tie is
    measured on head h's channels with its scale head_dim^-1/2. Returns (oracle idx, near rows)."""
    orc_idx, A = oracle.route_heads(q, k, n_win, topk, heads, want_affinity=True)
    gpu_idx = np.asarray(gpu_idx)
    assert gpu_idx.shape == orc_idx.shape, (gpu_idx.shape, orc_idx.shape)
    if np.array_equal(gpu_idx, orc_idx):
        return orc_idx, 0
    B, _, R, kk = orc_idx.shape
    C = q.shape[-1]
    hd = C // heads
    qm, km = oracle.region_means(q, n_win), oracle.region_means(k, n_win)
    near = 0
    for b, h, r in np.argwhere(np.any(gpu_idx != orc_idx, axis=-1)):
        row = gpu_idx[b, h, r]
        assert np.all((row >= 0) & (row < R)) and len(set(row.tolist())) == kk, f"row {b},{h},{r}: {row}"
        sl = slice(h * hd, (h + 1) * hd)
        mag = np.abs(qm[b, r, sl]) @ np.abs(km[b, :, sl]).T / math.sqrt(hd)
        for j in range(kk):
            a, o = row[j], orc_idx[b, h, r, j]
            if a != o:
                va, vo = A[b, h, r, a], A[b, h, r, o]
                tol = ROUTE_REL_TOL * max(mag[a], mag[o])
                assert abs(va - vo) <= tol, f"row {b},{h},{r} pos {j}: {a} ({va!r}) vs {o} ({vo!r}), tol {tol:.3e}"
        near += 1
    return orc_idx, near


# Backward: fp32 arithmetic on the GPU, float64 in the oracle. Each gradient element is a sum of
# at most topk * rs * (queries of a region) terms of O(1) size formed in fp32 (relative rounding
# 2^-24 per operation), so its error stays below about 1e-5 of the largest gradient; the bound is
# 1e-4 of the largest oracle gradient.
GRAD_REL_TOL = 1e-4


def check_grad(gpu: np.ndarray, ref: np.ndarray, what: str):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape and np.all(np.isfinite(gpu)), what
    err = float(np.max(np.abs(gpu - ref)))
    bound = GRAD_REL_TOL * float(np.max(np.abs(ref)))
    assert err <= bound, f"{what}: max abs err {err:.3e} > {bound:.3e}"
    return err
