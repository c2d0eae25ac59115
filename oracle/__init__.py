"""CPU oracle for the K-quant dequant-GEMV — TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (``libkq``) never uses it
and shares no code with it.

The arithmetic lives in ``kq_oracle.c`` (plain C, double precision): every
super-block is dequantised to double by its block formula and dotted with x
in natural index order.  Sources, by page:
 - "Out-of-core LLM inference engine written from scratch in Rust",
   Approach (weights dequantised inside fused matmul kernels; speculative
   decoding verifies several positions in one pass) and Results (Q4_K_M).
 - "Kortex: Streaming 70B Models on Consumer GPUs", Key components 2-3
   (layers copied into device slots while others compute; dequantise only in registers).
 - "RunNburn - Run a 295B MoE ...": selected experts per token, native
   K-quant kernels.

The multi-column, MoE and chain forms below are literal loops over the
single-matrix product: column c of the verify GEMV is the GEMV of column c;
the MoE GEMV for routed id e is the GEMV of expert e's matrix; a chain is its
matrices one after another.  The fused forms apply the textbook RMSNorm or
SiLU-gated unit to each column in double, then take the same product.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkq_oracle.so")
_lib = None

Q4_K, Q6_K, Q5_K, Q2_K, Q3_K, Q8_0 = 1, 2, 3, 4, 5, 6
FMT = {"q4_k": Q4_K, "q6_k": Q6_K, "q5_k": Q5_K, "q2_k": Q2_K, "q3_k": Q3_K, "q8_0": Q8_0}
# bytes per 256 weights (Q8_0: eight 34-byte blocks)
BLOCK_BYTES = {Q4_K: 144, Q6_K: 210, Q5_K: 176, Q2_K: 84, Q3_K: 110, Q8_0: 272}


def build(force: bool = False) -> str:
    """Compile kq_oracle.c with gcc (-O1, no fast-math: plain IEEE double)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O1", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
                               "-shared", "-fPIC", "-std=c11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        lib.kqo_f16.restype = ctypes.c_double
        lib.kqo_f16.argtypes = [ctypes.c_uint16]
        lib.kqo_dequant_row.restype = i32
        lib.kqo_dequant_row.argtypes = [i32, vp, i64, vp]
        lib.kqo_gemv.restype = i32
        lib.kqo_gemv.argtypes = [i32, vp, i64, i64, vp, vp, vp, i32]
        lib.kqo_gemv_rows.restype = i32
        lib.kqo_gemv_rows.argtypes = [i32, vp, i64, vp, i64, vp, vp, vp, i32]
        lib.kqo_unpack.restype = i32
        lib.kqo_unpack.argtypes = [i32, vp, i64, vp, vp, vp]
        lib.kqo_rmsnorm.restype = None
        lib.kqo_rmsnorm.argtypes = [vp, vp, i64, ctypes.c_double, vp]
        lib.kqo_swiglu.restype = None
        lib.kqo_swiglu.argtypes = [vp, i64, vp]
        lib.kqo_gemv_x64.restype = i32
        lib.kqo_gemv_x64.argtypes = [i32, vp, i64, i64, vp, vp, vp, i32]
        _lib = lib
    return _lib


def _fmt(fmt) -> int:
    return FMT[fmt] if isinstance(fmt, str) else int(fmt)


def _u8(W) -> np.ndarray:
    W = np.ascontiguousarray(W)
    assert W.dtype == np.uint8
    return W


def _threads(nthreads):
    if nthreads is None:
        return 1
    if nthreads <= 0:
        return max(1, len(os.sched_getaffinity(0)))
    return nthreads


def f16(bits: int) -> float:
    """fp16 bit pattern -> value (exact)."""
    return float(_load().kqo_f16(bits))


def dequant(fmt, W, N: int, K: int) -> np.ndarray:
    """Dense (N, K) float64 dequantised weights (small matrices only)."""
    f = _fmt(fmt)
    W = _u8(W)
    rb = K // 256 * BLOCK_BYTES[f]
    out = np.empty((N, K), np.float64)
    for r in range(N):
        rc = _load().kqo_dequant_row(f, W.ctypes.data + r * rb, K, out[r].ctypes.data)
        if rc:
            raise ValueError("dequant: bad format or K")
    return out


def gemv(fmt, W, N: int, K: int, x, nthreads=None):
    """(y, s): y_r = sum_i w_ri x_i and s_r = sum_i |w_ri x_i|, float64."""
    f = _fmt(fmt)
    W = _u8(W)
    x = np.ascontiguousarray(x, np.float32)
    assert x.size >= K and W.size >= N * (K // 256) * BLOCK_BYTES[f]
    y = np.empty(N, np.float64)
    s = np.empty(N, np.float64)
    rc = _load().kqo_gemv(f, W.ctypes.data, N, K, x.ctypes.data, y.ctypes.data, s.ctypes.data,
                          _threads(nthreads))
    if rc:
        raise RuntimeError(f"kqo_gemv failed ({rc})")
    return y, s


def gemv_rows(fmt, W, K: int, rows, x, nthreads=None):
    """(y, s) for a subset of rows (sampled checks on full-size matrices)."""
    f = _fmt(fmt)
    W = _u8(W)
    rows = np.ascontiguousarray(rows, np.int64)
    x = np.ascontiguousarray(x, np.float32)
    y = np.empty(rows.size, np.float64)
    s = np.empty(rows.size, np.float64)
    rc = _load().kqo_gemv_rows(f, W.ctypes.data, K, rows.ctypes.data, rows.size, x.ctypes.data,
                               y.ctypes.data, s.ctypes.data, _threads(nthreads))
    if rc:
        raise RuntimeError(f"kqo_gemv_rows failed ({rc})")
    return y, s


def gemv_multi(fmt, W, N: int, K: int, X, nthreads=None):
    """k-column form: X is (k, K) (column c contiguous); returns (k, N) y and s.
    Each column is an independent GEMV (one weight read serves k columns in
    the fused kernel; the result is the same as k separate products)."""
    X = np.ascontiguousarray(X, np.float32).reshape(-1, K)
    ys, ss = zip(*(gemv(fmt, W, N, K, X[c], nthreads) for c in range(X.shape[0])))
    return np.stack(ys), np.stack(ss)


def rmsnorm(x, gamma, eps: float) -> np.ndarray:
    """x_i * gamma_i / sqrt(mean(x^2) + eps) in float64 (kq_oracle.c)."""
    x = np.ascontiguousarray(x, np.float32)
    g = np.ascontiguousarray(gamma, np.float32)
    out = np.empty(x.size, np.float64)
    _load().kqo_rmsnorm(x.ctypes.data, g.ctypes.data, x.size, ctypes.c_double(eps), out.ctypes.data)
    return out


def swiglu(gu) -> np.ndarray:
    """silu(g_i) * u_i for gu = [g; u] (2K floats), float64 (kq_oracle.c)."""
    gu = np.ascontiguousarray(gu, np.float32)
    K = gu.size // 2
    out = np.empty(K, np.float64)
    _load().kqo_swiglu(gu.ctypes.data, K, out.ctypes.data)
    return out


def gemv_x64(fmt, W, N: int, K: int, x, nthreads=None):
    """(y, s) for float64 activations (a prologue's output)."""
    f = _fmt(fmt)
    W = _u8(W)
    x = np.ascontiguousarray(x, np.float64)
    assert x.size >= K
    y = np.empty(N, np.float64)
    s = np.empty(N, np.float64)
    rc = _load().kqo_gemv_x64(f, W.ctypes.data, N, K, x.ctypes.data, y.ctypes.data, s.ctypes.data,
                              _threads(nthreads))
    if rc:
        raise RuntimeError(f"kqo_gemv_x64 failed ({rc})")
    return y, s


def gemv_fused(fmt, W, N: int, K: int, X, kind: str, gamma=None, eps: float = 1e-5, nthreads=None):
    """k-column GEMV of prologue(X): kind "none", "rmsnorm" (X is (k, K)) or
    "swiglu" (X is (k, 2K), each row [g; u]).  Returns (k, N) y and s, with
    s = sum |w x'| over the transformed activations."""
    width = 2 * K if kind == "swiglu" else K
    X = np.ascontiguousarray(X, np.float32).reshape(-1, width)
    ys, ss = [], []
    for c in range(X.shape[0]):
        if kind == "rmsnorm":
            xt = rmsnorm(X[c], gamma, eps)
        elif kind == "swiglu":
            xt = swiglu(X[c])
        else:
            xt = X[c].astype(np.float64)
        y, s = gemv_x64(fmt, W, N, K, xt, nthreads)
        ys.append(y)
        ss.append(s)
    return np.stack(ys), np.stack(ss)


def moe_gemv(fmt, W_experts, E: int, N: int, K: int, ids, X, nthreads=None):
    """Routed-expert form: for the i-th id e, y[i] = W_e x_i, where W_e is
    the e-th (N x K) matrix of the contiguous expert stack and x_i = X[i] if X
    has one row per id, else the shared X."""
    f = _fmt(fmt)
    W_experts = _u8(W_experts)
    stride = N * (K // 256) * BLOCK_BYTES[f]
    X = np.ascontiguousarray(X, np.float32).reshape(-1, K)
    ys, ss = [], []
    for i, e in enumerate(np.asarray(ids).tolist()):
        if not (0 <= e < E):
            raise ValueError(f"expert id {e} out of range")
        x = X[i] if X.shape[0] > 1 else X[0]
        y, s = gemv(fmt, W_experts[e * stride:(e + 1) * stride], N, K, x, nthreads)
        ys.append(y)
        ss.append(s)
    return np.stack(ys), np.stack(ss)


def unpack(fmt, W, nblocks: int):
    """Logical fields (q, sc, d) of consecutive blocks; see kq_oracle.c."""
    f = _fmt(fmt)
    W = _u8(W)
    q = np.empty(nblocks * 256, np.uint8)
    sc = np.empty(nblocks * 16, np.uint8)
    d = np.empty(nblocks * 2, np.float32)
    rc = _load().kqo_unpack(f, W.ctypes.data, nblocks, q.ctypes.data, sc.ctypes.data, d.ctypes.data)
    if rc:
        raise ValueError("unpack: bad format")
    return q, sc, d


def within_tolerance(y_gpu, y_ref, s_ref, rel: float = 1e-3, abs_: float = 1e-6):
    """Per-output acceptance: |y - y_ref| <= rel * sum|w x| + abs."""
    y_gpu = np.asarray(y_gpu, np.float64)
    err = np.abs(y_gpu - y_ref)
    bound = rel * s_ref + abs_
    return bool(np.all(err <= bound)), err, bound
