"""Python binding of libbra.so: argument marshalling only.

Every step of the forward pass runs in the library's CUDA kernels; these functions only
check tensor metadata, allocate outputs with torch and pass raw pointers and the current
CUDA stream through ctypes. If libbra.so is missing the first call raises: there is no
CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

LIBRARY = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbra.so")
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "bra.h")

STATUS = {0: "BRA_OK", 1: "BRA_ERR_INVALID_ARG", 2: "BRA_ERR_UNSUPPORTED", 3: "BRA_ERR_CUDA",
          4: "BRA_ERR_INDEX", 5: "BRA_ERR_TIMEOUT"}
DTYPES = {torch.float32: 0, torch.bfloat16: 1}
ATTEND_KERNELS = {"auto": 0, "simt": 1, "gather_mma": 2, "dense_mma": 3, "gather_umma": 4, "region_mma": 5}

_lib = None


class BraError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        self.status = status
        name = STATUS.get(status, f"status {status}")
        super().__init__(f"{what}: {name}" + (f" ({detail})" if detail else ""))


def lib() -> ctypes.CDLL:
    """The loaded libbra.so (argument and result types set)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIBRARY):
        raise RuntimeError(f"{LIBRARY} is missing; build it with `python -m bi_level_routing_b200.build` "
                           "(there is no CPU fallback)")
    L = ctypes.CDLL(LIBRARY)
    vp, i32p, I = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_int
    L.bra_route.argtypes = [vp, vp, vp, I, I, I, I, I, I, I, vp]
    L.bra_attend.argtypes = [vp, vp, vp, vp, vp, I, I, I, I, I, I, I, I, vp]
    L.bra_forward.argtypes = [vp, vp, vp, vp, vp, I, I, I, I, I, I, I, I, vp]
    L.bra_forward_host.argtypes = [vp, vp, vp, vp, vp, I, I, I, I, I, I, I, I, vp]
    L.bra_route_heads.argtypes = [vp, vp, vp, I, I, I, I, I, I, I, I, vp]
    L.bra_attend_heads.argtypes = [vp, vp, vp, vp, vp, I, I, I, I, I, I, I, I, vp]
    L.bra_forward_heads.argtypes = [vp, vp, vp, vp, vp, I, I, I, I, I, I, I, I, vp]
    L.bra_forward_auto_pad.argtypes = [vp, vp, vp, vp, vp, I, I, I, I, I, I, I, I, vp]
    L.bra_lepe.argtypes = [vp, vp, vp, vp, I, I, I, I, I, vp]
    L.bra_forward_lepe.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, I, I, I, I, I, I, I, I, vp]
    L.bra_attend_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, I, I, I, I, I, I, I, I, vp]
    L.bra_selftest_wait_timeout.argtypes = [ctypes.c_uint, vp]
    L.bra_set_attend_kernel.argtypes = [I]
    L.bra_set_max_ctas.argtypes = [I]
    L.bra_selected_attend_kernel.argtypes = [I, I, I, I, I, I, I, I]
    L.bra_check_device_error.argtypes = [vp]
    L.bra_route_scratch_bytes.argtypes = [I, I, I, I, I]
    L.bra_route_scratch_bytes.restype = ctypes.c_size_t
    L.bra_kernels_per_call.argtypes = [ctypes.c_char_p, I, I, I, I, I, I, I, I]
    L.bra_status_string.argtypes = [I]
    L.bra_status_string.restype = ctypes.c_char_p
    L.bra_last_error_message.restype = ctypes.c_char_p
    for name in ("bra_route", "bra_attend", "bra_forward", "bra_forward_host", "bra_set_attend_kernel", "bra_set_max_ctas",
                 "bra_route_heads", "bra_attend_heads", "bra_forward_heads", "bra_forward_auto_pad", "bra_lepe",
                 "bra_forward_lepe", "bra_attend_backward", "bra_selftest_wait_timeout",
                 "bra_selected_attend_kernel", "bra_check_device_error", "bra_kernels_per_call"):
        getattr(L, name).restype = I
    _lib = L
    return L


def declared_symbols() -> list[str]:
    """Names of the functions include/bra.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(bra_\w+)\s*\(", text, flags=re.M)))


def _check(status: int, what: str):
    if status != 0:
        detail = lib().bra_last_error_message().decode() if status == 3 else ""
        raise BraError(status, what, detail)


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _shape(x: torch.Tensor, name: str):
    if x.dim() != 4:
        raise ValueError(f"{name} must be [B, H, W, C], got shape {tuple(x.shape)}")
    if not x.is_cuda or not x.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if x.dtype not in DTYPES:
        raise ValueError(f"{name} must be float32 or bfloat16, got {x.dtype}")
    return tuple(x.shape)


def _same(ref: torch.Tensor, *others):
    for name, t in others:
        if t.shape != ref.shape or t.dtype != ref.dtype or t.device != ref.device:
            raise ValueError(f"{name} must match q in shape, dtype and device")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def route(q: torch.Tensor, k: torch.Tensor, n_win: int, topk: int, idx: torch.Tensor | None = None) -> torch.Tensor:
    """Routing index int32 [B, n_win^2, topk] (region means, affinity, top-k)."""
    B, H, W, C = _shape(q, "q")
    _same(q, ("k", k))
    R = n_win * n_win
    if idx is None:
        idx = torch.empty((B, R, topk), dtype=torch.int32, device=q.device)
    elif idx.shape != (B, R, topk) or idx.dtype != torch.int32 or not idx.is_contiguous():
        raise ValueError("idx must be a contiguous int32 [B, n_win^2, topk] tensor")
    _check(lib().bra_route(q.data_ptr(), k.data_ptr(), idx.data_ptr(), B, H, W, C, n_win, topk, DTYPES[q.dtype],
                           _stream(q.device)), "bra_route")
    return idx


def attend(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor, heads: int, n_win: int,
           out: torch.Tensor | None = None) -> torch.Tensor:
    """Attention of every query over its region's routed keys; out has q's shape and dtype."""
    B, H, W, C = _shape(q, "q")
    _same(q, ("k", k), ("v", v))
    if idx.dim() != 3 or idx.dtype != torch.int32 or not idx.is_contiguous() or idx.device != q.device:
        raise ValueError("idx must be a contiguous int32 [B, n_win^2, topk] tensor on q's device")
    if out is None:
        out = torch.empty_like(q)
    _same(q, ("out", out))
    _check(lib().bra_attend(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), out.data_ptr(), B, H, W, C,
                            heads, n_win, idx.shape[-1], DTYPES[q.dtype], _stream(q.device)), "bra_attend")
    return out


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_win: int, topk: int, heads: int,
            out: torch.Tensor | None = None, idx: torch.Tensor | None = None):
    """The whole forward pass. Returns (out, idx)."""
    B, H, W, C = _shape(q, "q")
    _same(q, ("k", k), ("v", v))
    R = n_win * n_win
    if out is None:
        out = torch.empty_like(q)
    _same(q, ("out", out))
    if idx is None:
        idx = torch.empty((B, R, topk), dtype=torch.int32, device=q.device)
    elif idx.shape != (B, R, topk) or idx.dtype != torch.int32 or not idx.is_contiguous():
        raise ValueError("idx must be a contiguous int32 [B, n_win^2, topk] tensor")
    _check(lib().bra_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), out.data_ptr(), B, H, W, C,
                             heads, n_win, topk, DTYPES[q.dtype], _stream(q.device)), "bra_forward")
    return out, idx


def forward_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_win: int, topk: int, heads: int,
                 out: torch.Tensor | None = None, idx: torch.Tensor | None = None, device=None):
    """The forward pass on HOST tensors (pinned for full-speed copies): the library copies the
    inputs to the current CUDA device, runs the pass and copies out and idx back. Synchronous."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.is_cuda or not t.is_contiguous() or t.dim() != 4 or t.dtype not in DTYPES:
            raise ValueError(f"{name} must be a contiguous host [B, H, W, C] float32/bfloat16 tensor")
    if k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k and v must match")
    B, H, W, C = q.shape
    R = n_win * n_win
    if out is None:
        out = torch.empty_like(q, pin_memory=q.is_pinned())
    if idx is None:
        idx = torch.empty((B, R, topk), dtype=torch.int32, pin_memory=q.is_pinned())
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(device):
        _check(lib().bra_forward_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), out.data_ptr(), B, H,
                                      W, C, heads, n_win, topk, DTYPES[q.dtype], _stream(device)), "bra_forward_host")
    return out, idx


def route_heads(q: torch.Tensor, k: torch.Tensor, n_win: int, topk: int, heads: int,
                idx: torch.Tensor | None = None) -> torch.Tensor:
    """Per-head routing index int32 [B, heads, n_win^2, min(topk, n_win^2)] (topk clamped to the
    number of regions, as the pages do)."""
    B, H, W, C = _shape(q, "q")
    _same(q, ("k", k))
    R = n_win * n_win
    topk = min(topk, R)
    if idx is None:
        idx = torch.empty((B, heads, R, topk), dtype=torch.int32, device=q.device)
    elif idx.shape != (B, heads, R, topk) or idx.dtype != torch.int32 or not idx.is_contiguous():
        raise ValueError("idx must be a contiguous int32 [B, heads, n_win^2, min(topk, n_win^2)] tensor")
    _check(lib().bra_route_heads(q.data_ptr(), k.data_ptr(), idx.data_ptr(), B, H, W, C, heads, n_win, topk,
                                 DTYPES[q.dtype], _stream(q.device)), "bra_route_heads")
    return idx


def attend_heads(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor, n_win: int,
                 out: torch.Tensor | None = None) -> torch.Tensor:
    """Attention where head h gathers the regions of its own rows idx [B, heads, R, topk]."""
    B, H, W, C = _shape(q, "q")
    _same(q, ("k", k), ("v", v))
    if idx.dim() != 4 or idx.dtype != torch.int32 or not idx.is_contiguous() or idx.device != q.device:
        raise ValueError("idx must be a contiguous int32 [B, heads, n_win^2, topk] tensor on q's device")
    if out is None:
        out = torch.empty_like(q)
    _same(q, ("out", out))
    _check(lib().bra_attend_heads(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), out.data_ptr(), B, H, W,
                                  C, idx.shape[1], n_win, idx.shape[-1], DTYPES[q.dtype], _stream(q.device)),
           "bra_attend_heads")
    return out


def forward_heads(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_win: int, topk: int, heads: int,
                  out: torch.Tensor | None = None, idx: torch.Tensor | None = None):
    """The forward pass with per-head routing. Returns (out, idx [B, heads, R, min(topk, R)])."""
    B, H, W, C = _shape(q, "q")
    _same(q, ("k", k), ("v", v))
    R = n_win * n_win
    topk = min(topk, R)
    if out is None:
        out = torch.empty_like(q)
    _same(q, ("out", out))
    if idx is None:
        idx = torch.empty((B, heads, R, topk), dtype=torch.int32, device=q.device)
    _check(lib().bra_forward_heads(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), out.data_ptr(), B, H,
                                   W, C, heads, n_win, topk, DTYPES[q.dtype], _stream(q.device)), "bra_forward_heads")
    return out, idx


def forward_auto_pad(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_win: int, topk: int, heads: int,
                     out: torch.Tensor | None = None, idx: torch.Tensor | None = None):
    """The forward pass on any H x W: the map is taken as zero-padded at the bottom and right to
    multiples of n_win (nothing is copied), and out has q's shape. Returns (out, idx)."""
    B, H, W, C = _shape(q, "q")
    _same(q, ("k", k), ("v", v))
    R = n_win * n_win
    if out is None:
        out = torch.empty_like(q)
    _same(q, ("out", out))
    if idx is None:
        idx = torch.empty((B, R, topk), dtype=torch.int32, device=q.device)
    _check(lib().bra_forward_auto_pad(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), out.data_ptr(), B, H,
                                      W, C, heads, n_win, topk, DTYPES[q.dtype], _stream(q.device)),
           "bra_forward_auto_pad")
    return out, idx


def lepe(x: torch.Tensor, weight: torch.Tensor, bias: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """x + 5x5 depthwise convolution of x (zero padding 2) + bias; weight fp32 [C, 5, 5], bias fp32 [C]."""
    B, H, W, C = _shape(x, "x")
    for name, t, shape in (("weight", weight, (C, 5, 5)), ("bias", bias, (C,))):
        if t.dtype != torch.float32 or tuple(t.shape) != shape or not t.is_contiguous() or t.device != x.device:
            raise ValueError(f"{name} must be a contiguous float32 {shape} tensor on x's device")
    if out is None:
        out = torch.empty_like(x)
    _same(x, ("out", out))
    _check(lib().bra_lepe(x.data_ptr(), weight.data_ptr(), bias.data_ptr(), out.data_ptr(), B, H, W, C,
                          DTYPES[x.dtype], _stream(x.device)), "bra_lepe")
    return out


def forward_lepe(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_win: int, topk: int, heads: int,
                 weight: torch.Tensor, bias: torch.Tensor, attn: torch.Tensor | None = None,
                 out: torch.Tensor | None = None, idx: torch.Tensor | None = None):
    """The forward pass followed by the LePE epilogue. Returns (out, attn, idx): attn is the
    attention output, out = attn + lepe(attn)."""
    B, H, W, C = _shape(q, "q")
    _same(q, ("k", k), ("v", v))
    R = n_win * n_win
    attn = torch.empty_like(q) if attn is None else attn
    out = torch.empty_like(q) if out is None else out
    _same(q, ("attn", attn), ("out", out))
    if idx is None:
        idx = torch.empty((B, R, topk), dtype=torch.int32, device=q.device)
    _check(lib().bra_forward_lepe(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), attn.data_ptr(),
                                  out.data_ptr(), weight.data_ptr(), bias.data_ptr(), B, H, W, C, heads, n_win, topk,
                                  DTYPES[q.dtype], _stream(q.device)), "bra_forward_lepe")
    return out, attn, idx


def attend_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor, dout: torch.Tensor,
                    heads: int, n_win: int, dq: torch.Tensor | None = None, dk: torch.Tensor | None = None,
                    dv: torch.Tensor | None = None):
    """(dq, dk, dv), float32 [B, H, W, C]: gradients of sum(dout * attend(q, k, v, idx)), idx fixed."""
    B, H, W, C = _shape(q, "q")
    _same(q, ("k", k), ("v", v), ("dout", dout))
    if idx.dim() != 3 or idx.dtype != torch.int32 or not idx.is_contiguous() or idx.device != q.device:
        raise ValueError("idx must be a contiguous int32 [B, n_win^2, topk] tensor on q's device")
    grads = []
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        if g is None:
            g = torch.empty((B, H, W, C), dtype=torch.float32, device=q.device)
        elif g.shape != (B, H, W, C) or g.dtype != torch.float32 or not g.is_contiguous() or g.device != q.device:
            raise ValueError(f"{name} must be a contiguous float32 [B, H, W, C] tensor on q's device")
        grads.append(g)
    dq, dk, dv = grads
    _check(lib().bra_attend_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), dout.data_ptr(),
                                     dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, W, C, heads, n_win,
                                     idx.shape[-1], DTYPES[q.dtype], _stream(q.device)), "bra_attend_backward")
    return dq, dk, dv


def check_device_error(device=None) -> int:
    """Synchronises the current stream and returns (and clears) the device error status."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(device):
        return lib().bra_check_device_error(_stream(device))


def set_attend_kernel(name: str):
    """Force one attention kernel ("simt", "gather_mma", "dense_mma", "gather_umma") or release ("auto")."""
    _check(lib().bra_set_attend_kernel(ATTEND_KERNELS[name]), "bra_set_attend_kernel")


def set_max_ctas(n: int):
    """Cap the persistent attention kernels' grid at n CTAs (0 = no cap); the result does not change."""
    _check(lib().bra_set_max_ctas(int(n)), "bra_set_max_ctas")


def selected_attend_kernel(B, H, W, C, heads, n_win, topk, dtype) -> str | None:
    code = lib().bra_selected_attend_kernel(B, H, W, C, heads, n_win, topk, DTYPES[dtype])
    return {v: k for k, v in ATTEND_KERNELS.items()}.get(code)


def kernels_per_call(entry_point: str, B, H, W, C, heads, n_win, topk, dtype) -> int:
    return lib().bra_kernels_per_call(entry_point.encode(), B, H, W, C, heads, n_win, topk, DTYPES[dtype])


def route_scratch_bytes(B, H, W, C, n_win) -> int:
    return int(lib().bra_route_scratch_bytes(B, H, W, C, n_win))
