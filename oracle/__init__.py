"""CPU oracle for the forward pass of Bi-Level Routing Attention (BRA).

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline / reference legs may import this package. The product path (the CUDA library
and its binding) never imports, links or executes anything here, and this package imports
nothing from the product.

The arithmetic lives in ``bra_oracle.c`` (plain C, float64); this module only builds it with
gcc and marshals numpy arrays through ctypes. Each function states the page passage it
restates; the C file's header lists the readings taken where the pages are silent.

All array inputs are converted to contiguous float64 (bf16 and fp32 values convert
exactly). Layouts: q, k, v, out ``[B, H, W, C]``; means ``[B, R, C]``; affinities
``[B, R, R]``; idx int32 ``[B, R, topk]``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "bra_oracle.c")
LIBRARY = os.path.join(_HERE, "libbra_oracle.so")

_DP = ctypes.POINTER(ctypes.c_double)
_IP = ctypes.POINTER(ctypes.c_int32)
_LP = ctypes.POINTER(ctypes.c_int64)
_I = ctypes.c_int


def compile_oracle(source: str = SOURCE, output: str = LIBRARY, extra_flags=()) -> str:
    """Compile the oracle's C source into a shared library with gcc (OpenMP, -O2)."""
    cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp", *extra_flags,
           source, "-o", output, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return output


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


class OracleError(RuntimeError):
    pass


class Oracle:
    """ctypes handle on one compiled copy of the oracle (tests may load mutated copies)."""

    def __init__(self, path: str = LIBRARY):
        if path == LIBRARY and (not os.path.exists(LIBRARY)
                                or os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE)):
            compile_oracle()
        lib = ctypes.CDLL(path)
        lib.oracle_max_threads.restype = _I
        lib.oracle_region_means.argtypes = [_DP, _I, _I, _I, _I, _I, _DP]
        lib.oracle_affinity.argtypes = [_DP, _DP, _I, _I, _I, _DP]
        lib.oracle_topk.argtypes = [_DP, _I, _I, _I, _IP]
        lib.oracle_route.argtypes = [_DP, _DP, _I, _I, _I, _I, _I, _I, _IP, _DP]
        lib.oracle_attend.argtypes = [_DP, _DP, _DP, _IP, _I, _I, _I, _I, _I, _I, _I, _DP]
        lib.oracle_attend_tokens.argtypes = [_DP, _DP, _DP, _IP, _I, _I, _I, _I, _I, _I, _I, _LP,
                                             ctypes.c_int64, _DP]
        lib.oracle_forward.argtypes = [_DP, _DP, _DP, _I, _I, _I, _I, _I, _I, _I, _IP, _DP]
        lib.oracle_route_heads.argtypes = [_DP, _DP, _I, _I, _I, _I, _I, _I, _I, _IP, _DP]
        lib.oracle_attend_heads.argtypes = [_DP, _DP, _DP, _IP, _I, _I, _I, _I, _I, _I, _I, _DP]
        lib.oracle_lepe.argtypes = [_DP, _DP, _DP, _I, _I, _I, _I, _DP]
        lib.oracle_attend_backward.argtypes = [_DP, _DP, _DP, _IP, _DP, _I, _I, _I, _I, _I, _I, _I, _DP, _DP, _DP]
        lib.oracle_forward_auto_pad.argtypes = [_DP, _DP, _DP, _I, _I, _I, _I, _I, _I, _I, _IP, _DP]
        lib.oracle_attend_auto_pad.argtypes = [_DP, _DP, _DP, _IP, _I, _I, _I, _I, _I, _I, _I, _DP]
        for name in ("oracle_region_means", "oracle_affinity", "oracle_topk", "oracle_route",
                     "oracle_attend", "oracle_attend_tokens", "oracle_forward", "oracle_route_heads",
                     "oracle_attend_heads", "oracle_lepe", "oracle_attend_backward", "oracle_forward_auto_pad",
                     "oracle_attend_auto_pad"):
            getattr(lib, name).restype = _I
        self._lib = lib
        self.path = path

    @staticmethod
    def _check(status: int, what: str):
        if status == 1:
            raise OracleError(f"{what}: invalid argument")
        if status == 2:
            raise OracleError(f"{what}: routing index outside [0, R)")
        if status != 0:
            raise OracleError(f"{what}: status {status}")

    def max_threads(self) -> int:
        return int(self._lib.oracle_max_threads())

    def region_means(self, x, n_win: int) -> np.ndarray:
        """Region-mean descriptors ("手把手带你读懂BiFormer源码", §1.2 step 1)."""
        x = _f64(x)
        B, H, W, C = x.shape
        out = np.empty((B, n_win * n_win, C), np.float64)
        self._check(self._lib.oracle_region_means(x.ctypes.data_as(_DP), B, H, W, C, n_win,
                                                  out.ctypes.data_as(_DP)), "region_means")
        return out

    def affinity(self, qm, km) -> np.ndarray:
        """Region affinity C^-1/2 Q_r K_r^T ("手把手带你读懂BiFormer源码", §1.2 step 2)."""
        qm, km = _f64(qm), _f64(km)
        B, R, C = qm.shape
        out = np.empty((B, R, R), np.float64)
        self._check(self._lib.oracle_affinity(qm.ctypes.data_as(_DP), km.ctypes.data_as(_DP), B, R, C,
                                              out.ctypes.data_as(_DP)), "affinity")
        return out

    def topk(self, A, topk: int) -> np.ndarray:
        """Per-row top-k, affinity descending, ties to the lower region, NaN last
        ("手把手带你读懂BiFormer源码", §1.2 step 3)."""
        A = _f64(A)
        B, R, _ = A.shape
        out = np.empty((B, R, topk), np.int32)
        self._check(self._lib.oracle_topk(A.ctypes.data_as(_DP), B, R, topk, out.ctypes.data_as(_IP)),
                    "topk")
        return out

    def route(self, q, k, n_win: int, topk: int, want_affinity: bool = False):
        """Routing index (and optionally the affinities) from q and k."""
        q, k = _f64(q), _f64(k)
        B, H, W, C = q.shape
        R = n_win * n_win
        idx = np.empty((B, R, topk), np.int32)
        A = np.empty((B, R, R), np.float64) if want_affinity else None
        self._check(self._lib.oracle_route(q.ctypes.data_as(_DP), k.ctypes.data_as(_DP), B, H, W, C, n_win,
                                           topk, idx.ctypes.data_as(_IP),
                                           A.ctypes.data_as(_DP) if A is not None else None), "route")
        return (idx, A) if want_affinity else idx

    def attend(self, q, k, v, idx, heads: int, n_win: int) -> np.ndarray:
        """Gather + token-to-token attention ("从零构建BiFormer", §2.2 TokenAttention;
        "医学图像分割模块", §五 steps ⑤-⑦)."""
        q, k, v, idx = _f64(q), _f64(k), _f64(v), _i32(idx)
        B, H, W, C = q.shape
        topk = idx.shape[-1]
        out = np.empty_like(q)
        self._check(self._lib.oracle_attend(q.ctypes.data_as(_DP), k.ctypes.data_as(_DP),
                                            v.ctypes.data_as(_DP), idx.ctypes.data_as(_IP), B, H, W, C,
                                            heads, n_win, topk, out.ctypes.data_as(_DP)), "attend")
        return out

    def attend_tokens(self, q, k, v, idx, heads: int, n_win: int, tokens) -> np.ndarray:
        """Attention output of the listed tokens only (tokens[i] = b*H*W + y*W + x)."""
        q, k, v, idx = _f64(q), _f64(k), _f64(v), _i32(idx)
        tokens = np.ascontiguousarray(np.asarray(tokens, dtype=np.int64))
        B, H, W, C = q.shape
        topk = idx.shape[-1]
        out = np.empty((tokens.shape[0], C), np.float64)
        self._check(self._lib.oracle_attend_tokens(
            q.ctypes.data_as(_DP), k.ctypes.data_as(_DP), v.ctypes.data_as(_DP), idx.ctypes.data_as(_IP),
            B, H, W, C, heads, n_win, topk, tokens.ctypes.data_as(_LP), tokens.shape[0],
            out.ctypes.data_as(_DP)), "attend_tokens")
        return out

    def forward(self, q, k, v, n_win: int, topk: int, heads: int):
        """Route then attend. Returns (out float64 [B,H,W,C], idx int32 [B,R,topk])."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, W, C = q.shape
        idx = np.empty((B, n_win * n_win, topk), np.int32)
        out = np.empty_like(q)
        self._check(self._lib.oracle_forward(q.ctypes.data_as(_DP), k.ctypes.data_as(_DP),
                                             v.ctypes.data_as(_DP), B, H, W, C, heads, n_win, topk,
                                             idx.ctypes.data_as(_IP), out.ctypes.data_as(_DP)), "forward")
        return out, idx

    def route_heads(self, q, k, n_win: int, topk: int, heads: int, want_affinity: bool = False):
        """Per-head routing ("医学图像分割模块", §五 steps ③④): idx int32 [B, heads, R, min(topk, R)]
        (and optionally the per-head affinities [B, heads, R, R], scale head_dim^-1/2)."""
        q, k = _f64(q), _f64(k)
        B, H, W, C = q.shape
        R = n_win * n_win
        kk = min(topk, R)
        idx = np.empty((B, heads, R, kk), np.int32)
        A = np.empty((B, heads, R, R), np.float64) if want_affinity else None
        self._check(self._lib.oracle_route_heads(q.ctypes.data_as(_DP), k.ctypes.data_as(_DP), B, H, W, C, heads,
                                                 n_win, topk, idx.ctypes.data_as(_IP),
                                                 A.ctypes.data_as(_DP) if A is not None else None), "route_heads")
        return (idx, A) if want_affinity else idx

    def attend_heads(self, q, k, v, idx, n_win: int) -> np.ndarray:
        """Attention with per-head index rows idx [B, heads, R, topk] ("医学图像分割模块", §五 ⑤-⑦)."""
        q, k, v, idx = _f64(q), _f64(k), _f64(v), _i32(idx)
        B, H, W, C = q.shape
        heads, topk = idx.shape[1], idx.shape[-1]
        out = np.empty_like(q)
        self._check(self._lib.oracle_attend_heads(q.ctypes.data_as(_DP), k.ctypes.data_as(_DP),
                                                  v.ctypes.data_as(_DP), idx.ctypes.data_as(_IP), B, H, W, C,
                                                  heads, n_win, topk, out.ctypes.data_as(_DP)), "attend_heads")
        return out

    def lepe(self, x, weight, bias) -> np.ndarray:
        """x + 5x5 depthwise convolution of x (zero padding 2) + bias ("医学图像分割模块", §五 ⑧);
        x [B, H, W, C], weight [C, 5, 5], bias [C]."""
        x, weight, bias = _f64(x), _f64(weight), _f64(bias)
        B, H, W, C = x.shape
        assert weight.shape == (C, 5, 5) and bias.shape == (C,)
        y = np.empty_like(x)
        self._check(self._lib.oracle_lepe(x.ctypes.data_as(_DP), weight.ctypes.data_as(_DP),
                                          bias.ctypes.data_as(_DP), B, H, W, C, y.ctypes.data_as(_DP)), "lepe")
        return y

    def attend_backward(self, q, k, v, idx, dout, heads: int, n_win: int):
        """(dq, dk, dv): gradients of sum(dout * attend(q, k, v, idx)) with idx held fixed."""
        q, k, v, idx, dout = _f64(q), _f64(k), _f64(v), _i32(idx), _f64(dout)
        B, H, W, C = q.shape
        dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
        self._check(self._lib.oracle_attend_backward(
            q.ctypes.data_as(_DP), k.ctypes.data_as(_DP), v.ctypes.data_as(_DP), idx.ctypes.data_as(_IP),
            dout.ctypes.data_as(_DP), B, H, W, C, heads, n_win, idx.shape[-1], dq.ctypes.data_as(_DP),
            dk.ctypes.data_as(_DP), dv.ctypes.data_as(_DP)), "attend_backward")
        return dq, dk, dv

    def forward_auto_pad(self, q, k, v, n_win: int, topk: int, heads: int):
        """auto_pad ("从静态到动态", §4.2): zero-pad to multiples of n_win, route + attend, crop.
        Returns (out [B, H, W, C], idx [B, R, topk] of the padded map)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, W, C = q.shape
        idx = np.empty((B, n_win * n_win, topk), np.int32)
        out = np.empty_like(q)
        self._check(self._lib.oracle_forward_auto_pad(q.ctypes.data_as(_DP), k.ctypes.data_as(_DP),
                                                      v.ctypes.data_as(_DP), B, H, W, C, heads, n_win, topk,
                                                      idx.ctypes.data_as(_IP), out.ctypes.data_as(_DP)),
                    "forward_auto_pad")
        return out, idx

    def attend_auto_pad(self, q, k, v, idx, heads: int, n_win: int) -> np.ndarray:
        """Step 5 of auto_pad with a given index of the padded map."""
        q, k, v, idx = _f64(q), _f64(k), _f64(v), _i32(idx)
        B, H, W, C = q.shape
        out = np.empty_like(q)
        self._check(self._lib.oracle_attend_auto_pad(q.ctypes.data_as(_DP), k.ctypes.data_as(_DP),
                                                     v.ctypes.data_as(_DP), idx.ctypes.data_as(_IP), B, H, W, C,
                                                     heads, n_win, idx.shape[-1], out.ctypes.data_as(_DP)),
                    "attend_auto_pad")
        return out


_default: Oracle | None = None


def default() -> Oracle:
    """The oracle compiled from this directory's source (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def region_means(x, n_win):
    return default().region_means(x, n_win)


def affinity(qm, km):
    return default().affinity(qm, km)


def topk(A, k):
    return default().topk(A, k)


def route(q, k, n_win, topk, want_affinity=False):
    return default().route(q, k, n_win, topk, want_affinity)


def attend(q, k, v, idx, heads, n_win):
    return default().attend(q, k, v, idx, heads, n_win)


def attend_tokens(q, k, v, idx, heads, n_win, tokens):
    return default().attend_tokens(q, k, v, idx, heads, n_win, tokens)


def forward(q, k, v, n_win, topk, heads):
    return default().forward(q, k, v, n_win, topk, heads)


def max_threads():
    return default().max_threads()


def route_heads(q, k, n_win, topk, heads, want_affinity=False):
    return default().route_heads(q, k, n_win, topk, heads, want_affinity)


def attend_heads(q, k, v, idx, n_win):
    return default().attend_heads(q, k, v, idx, n_win)


def lepe(x, weight, bias):
    return default().lepe(x, weight, bias)


def attend_backward(q, k, v, idx, dout, heads, n_win):
    return default().attend_backward(q, k, v, idx, dout, heads, n_win)


def forward_auto_pad(q, k, v, n_win, topk, heads):
    return default().forward_auto_pad(q, k, v, n_win, topk, heads)


def attend_auto_pad(q, k, v, idx, heads, n_win):
    return default().attend_auto_pad(q, k, v, idx, heads, n_win)
