"""Seeded synthetic inputs for the K-quant GEMV workloads (shared by the
oracle side and the CUDA side; holds no dequantisation or dot-product
arithmetic).

The C source ``kqgen.c`` draws logical values with a counter-based
SplitMix64 stream and encodes them into the GGUF K-quant super-block layout
(Q2_K: 84 bytes, Q3_K: 110, Q4_K: 144, Q5_K: 176, Q6_K: 210; 256 weights each;
Q8_0 in units of eight 34-byte blocks, 272 bytes per 256 weights).  This wrapper builds it
with gcc on first use and returns numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kqgen.c")
_LIB_PATH = os.path.join(_HERE, "libkqgen.so")
_lib = None

Q4_K_BLOCK_BYTES = 144
Q5_K_BLOCK_BYTES = 176
Q2_K_BLOCK_BYTES = 84
Q3_K_BLOCK_BYTES = 110
Q6_K_BLOCK_BYTES = 210
Q8_0_UNIT_BYTES = 272  # eight 34-byte Q8_0 blocks: 256 weights
QK = 256  # weights per super-block


def build(force: bool = False) -> str:
    """Compile kqgen.c into libkqgen.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, i64, i32, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        lib.kqg_splitmix64.restype = u64
        lib.kqg_splitmix64.argtypes = [u64, u64]
        lib.kqg_tensor_seed.restype = u64
        lib.kqg_tensor_seed.argtypes = [u64, u64, u64]
        lib.kqg_f16_bits.restype = ctypes.c_uint16
        lib.kqg_f16_bits.argtypes = [ctypes.c_double]
        lib.kqg_q4k_draw.argtypes = [u64, i64, vp, vp, vp, vp, vp]
        lib.kqg_q4k_pack.argtypes = [i64, vp, vp, vp, vp, vp, vp]
        lib.kqg_q4k_fill.argtypes = [u64, i64, i64, vp, i32]
        lib.kqg_q5k_draw.argtypes = [u64, i64, vp, vp, vp, vp, vp]
        lib.kqg_q5k_pack.argtypes = [i64, vp, vp, vp, vp, vp, vp]
        lib.kqg_q5k_fill.argtypes = [u64, i64, i64, vp, i32]
        lib.kqg_q2k_draw.argtypes = [u64, i64, vp, vp, vp, vp, vp]
        lib.kqg_q2k_pack.argtypes = [i64, vp, vp, vp, vp, vp, vp]
        lib.kqg_q2k_fill.argtypes = [u64, i64, i64, vp, i32]
        lib.kqg_q3k_draw.argtypes = [u64, i64, vp, vp, vp]
        lib.kqg_q3k_pack.argtypes = [i64, vp, vp, vp, vp]
        lib.kqg_q3k_fill.argtypes = [u64, i64, i64, vp, i32]
        lib.kqg_q6k_draw.argtypes = [u64, i64, vp, vp, vp]
        lib.kqg_q6k_pack.argtypes = [i64, vp, vp, vp, vp]
        lib.kqg_q6k_fill.argtypes = [u64, i64, i64, vp, i32]
        lib.kqg_q80_draw.argtypes = [u64, i64, vp, vp]
        lib.kqg_q80_pack.argtypes = [i64, vp, vp, vp]
        lib.kqg_q80_fill.argtypes = [u64, i64, i64, vp, i32]
        lib.kqg_normal_f32.argtypes = [u64, i64, vp, i32]
        lib.kqg_topk_ids.restype = i32
        lib.kqg_topk_ids.argtypes = [u64, i32, i32, vp]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def splitmix64(key: int, ctr: int) -> int:
    return int(_load().kqg_splitmix64(key & (2**64 - 1), ctr))


def tensor_seed(base: int, layer: int, matrix: int) -> int:
    return int(_load().kqg_tensor_seed(base & (2**64 - 1), layer, matrix))


def f16_bits(v: float) -> int:
    return int(_load().kqg_f16_bits(float(v)))


def block_bytes(fmt: str) -> int:
    return {"q4_k": Q4_K_BLOCK_BYTES, "q5_k": Q5_K_BLOCK_BYTES, "q6_k": Q6_K_BLOCK_BYTES, "q2_k": Q2_K_BLOCK_BYTES,
            "q3_k": Q3_K_BLOCK_BYTES, "q8_0": Q8_0_UNIT_BYTES}[fmt]


def row_bytes(fmt: str, K: int) -> int:
    assert K % QK == 0
    return K // QK * block_bytes(fmt)


# ----------------------------------------------------------------- Q4_K
def q4k_draw(key: int, nblocks: int) -> dict:
    """Logical values of ``nblocks`` Q4_K super-blocks: q (nb,256) u8 in 0..15,
    sc/m (nb,8) u8 in 0..63, d/dmin (nb,) fp16 bit patterns (uint16)."""
    q = np.empty((nblocks, 256), np.uint8)
    sc = np.empty((nblocks, 8), np.uint8)
    m = np.empty((nblocks, 8), np.uint8)
    d = np.empty(nblocks, np.uint16)
    dmin = np.empty(nblocks, np.uint16)
    _load().kqg_q4k_draw(key, nblocks, _ptr(q), _ptr(sc), _ptr(m), _ptr(d), _ptr(dmin))
    return dict(q=q, sc=sc, m=m, d=d, dmin=dmin)


def q4k_pack(q, sc, m, d, dmin) -> np.ndarray:
    """Encode logical Q4_K values (see :func:`q4k_draw`) into bytes (nb*144,)."""
    q = np.ascontiguousarray(q, np.uint8).reshape(-1, 256)
    nb = q.shape[0]
    sc = np.ascontiguousarray(sc, np.uint8).reshape(nb, 8)
    m = np.ascontiguousarray(m, np.uint8).reshape(nb, 8)
    d = np.ascontiguousarray(d, np.uint16).reshape(nb)
    dmin = np.ascontiguousarray(dmin, np.uint16).reshape(nb)
    out = np.empty(nb * Q4_K_BLOCK_BYTES, np.uint8)
    _load().kqg_q4k_pack(nb, _ptr(q), _ptr(sc), _ptr(m), _ptr(d), _ptr(dmin), _ptr(out))
    return out


def q4k_fill(key: int, nblocks: int, out: np.ndarray | None = None, b0: int = 0,
             nthreads: int | None = None) -> np.ndarray:
    """Draw + encode super-blocks [b0, b0+nblocks) of stream ``key``."""
    if out is None:
        out = np.empty(nblocks * Q4_K_BLOCK_BYTES, np.uint8)
    assert out.nbytes >= nblocks * Q4_K_BLOCK_BYTES and out.dtype == np.uint8
    _load().kqg_q4k_fill(key, b0, nblocks, _ptr(out), nthreads or default_threads())
    return out


# ----------------------------------------------------------------- Q5_K
def q5k_draw(key: int, nblocks: int) -> dict:
    """Logical values of ``nblocks`` Q5_K super-blocks: q (nb,256) u8 in 0..31,
    sc/m (nb,8) u8 in 0..63, d/dmin (nb,) fp16 bit patterns (uint16)."""
    q = np.empty((nblocks, 256), np.uint8)
    sc = np.empty((nblocks, 8), np.uint8)
    m = np.empty((nblocks, 8), np.uint8)
    d = np.empty(nblocks, np.uint16)
    dmin = np.empty(nblocks, np.uint16)
    _load().kqg_q5k_draw(key, nblocks, _ptr(q), _ptr(sc), _ptr(m), _ptr(d), _ptr(dmin))
    return dict(q=q, sc=sc, m=m, d=d, dmin=dmin)


def q5k_pack(q, sc, m, d, dmin) -> np.ndarray:
    """Encode logical Q5_K values (see :func:`q5k_draw`) into bytes (nb*176,)."""
    q = np.ascontiguousarray(q, np.uint8).reshape(-1, 256)
    nb = q.shape[0]
    sc = np.ascontiguousarray(sc, np.uint8).reshape(nb, 8)
    m = np.ascontiguousarray(m, np.uint8).reshape(nb, 8)
    d = np.ascontiguousarray(d, np.uint16).reshape(nb)
    dmin = np.ascontiguousarray(dmin, np.uint16).reshape(nb)
    out = np.empty(nb * Q5_K_BLOCK_BYTES, np.uint8)
    _load().kqg_q5k_pack(nb, _ptr(q), _ptr(sc), _ptr(m), _ptr(d), _ptr(dmin), _ptr(out))
    return out


def q5k_fill(key: int, nblocks: int, out: np.ndarray | None = None, b0: int = 0,
             nthreads: int | None = None) -> np.ndarray:
    """Draw + encode Q5_K super-blocks [b0, b0+nblocks) of stream ``key``."""
    if out is None:
        out = np.empty(nblocks * Q5_K_BLOCK_BYTES, np.uint8)
    assert out.nbytes >= nblocks * Q5_K_BLOCK_BYTES and out.dtype == np.uint8
    _load().kqg_q5k_fill(key, b0, nblocks, _ptr(out), nthreads or default_threads())
    return out


# ----------------------------------------------------------------- Q2_K
def q2k_draw(key: int, nblocks: int) -> dict:
    """Logical values of Q2_K super-blocks: q (nb,256) u8 in 0..3, sc/m
    (nb,16) u8 in 0..15, d/dmin (nb,) fp16 bit patterns."""
    q = np.empty((nblocks, 256), np.uint8)
    sc = np.empty((nblocks, 16), np.uint8)
    m = np.empty((nblocks, 16), np.uint8)
    d = np.empty(nblocks, np.uint16)
    dmin = np.empty(nblocks, np.uint16)
    _load().kqg_q2k_draw(key, nblocks, _ptr(q), _ptr(sc), _ptr(m), _ptr(d), _ptr(dmin))
    return dict(q=q, sc=sc, m=m, d=d, dmin=dmin)


def q2k_pack(q, sc, m, d, dmin) -> np.ndarray:
    q = np.ascontiguousarray(q, np.uint8).reshape(-1, 256)
    nb = q.shape[0]
    sc = np.ascontiguousarray(sc, np.uint8).reshape(nb, 16)
    m = np.ascontiguousarray(m, np.uint8).reshape(nb, 16)
    d = np.ascontiguousarray(d, np.uint16).reshape(nb)
    dmin = np.ascontiguousarray(dmin, np.uint16).reshape(nb)
    out = np.empty(nb * Q2_K_BLOCK_BYTES, np.uint8)
    _load().kqg_q2k_pack(nb, _ptr(q), _ptr(sc), _ptr(m), _ptr(d), _ptr(dmin), _ptr(out))
    return out


def q2k_fill(key: int, nblocks: int, out: np.ndarray | None = None, b0: int = 0,
             nthreads: int | None = None) -> np.ndarray:
    if out is None:
        out = np.empty(nblocks * Q2_K_BLOCK_BYTES, np.uint8)
    assert out.nbytes >= nblocks * Q2_K_BLOCK_BYTES and out.dtype == np.uint8
    _load().kqg_q2k_fill(key, b0, nblocks, _ptr(out), nthreads or default_threads())
    return out


# ----------------------------------------------------------------- Q3_K
def q3k_draw(key: int, nblocks: int) -> dict:
    """Logical values of Q3_K super-blocks: q (nb,256) int8 in -4..3, v
    (nb,16) u8 6-bit scales (used as v - 32), d (nb,) fp16 bit patterns."""
    q = np.empty((nblocks, 256), np.int8)
    v = np.empty((nblocks, 16), np.uint8)
    d = np.empty(nblocks, np.uint16)
    _load().kqg_q3k_draw(key, nblocks, _ptr(q), _ptr(v), _ptr(d))
    return dict(q=q, v=v, d=d)


def q3k_pack(q, v, d) -> np.ndarray:
    q = np.ascontiguousarray(q, np.int8).reshape(-1, 256)
    nb = q.shape[0]
    v = np.ascontiguousarray(v, np.uint8).reshape(nb, 16)
    d = np.ascontiguousarray(d, np.uint16).reshape(nb)
    out = np.empty(nb * Q3_K_BLOCK_BYTES, np.uint8)
    _load().kqg_q3k_pack(nb, _ptr(q), _ptr(v), _ptr(d), _ptr(out))
    return out


def q3k_fill(key: int, nblocks: int, out: np.ndarray | None = None, b0: int = 0,
             nthreads: int | None = None) -> np.ndarray:
    if out is None:
        out = np.empty(nblocks * Q3_K_BLOCK_BYTES, np.uint8)
    assert out.nbytes >= nblocks * Q3_K_BLOCK_BYTES and out.dtype == np.uint8
    _load().kqg_q3k_fill(key, b0, nblocks, _ptr(out), nthreads or default_threads())
    return out


# ----------------------------------------------------------------- Q6_K
def q6k_draw(key: int, nblocks: int) -> dict:
    """Logical values of Q6_K super-blocks: q (nb,256) u8 in 0..63,
    s (nb,16) int8 in -64..63, d (nb,) fp16 bit patterns."""
    q = np.empty((nblocks, 256), np.uint8)
    s = np.empty((nblocks, 16), np.int8)
    d = np.empty(nblocks, np.uint16)
    _load().kqg_q6k_draw(key, nblocks, _ptr(q), _ptr(s), _ptr(d))
    return dict(q=q, s=s, d=d)


def q6k_pack(q, s, d) -> np.ndarray:
    q = np.ascontiguousarray(q, np.uint8).reshape(-1, 256)
    nb = q.shape[0]
    s = np.ascontiguousarray(s, np.int8).reshape(nb, 16)
    d = np.ascontiguousarray(d, np.uint16).reshape(nb)
    out = np.empty(nb * Q6_K_BLOCK_BYTES, np.uint8)
    _load().kqg_q6k_pack(nb, _ptr(q), _ptr(s), _ptr(d), _ptr(out))
    return out


def q6k_fill(key: int, nblocks: int, out: np.ndarray | None = None, b0: int = 0,
             nthreads: int | None = None) -> np.ndarray:
    if out is None:
        out = np.empty(nblocks * Q6_K_BLOCK_BYTES, np.uint8)
    assert out.nbytes >= nblocks * Q6_K_BLOCK_BYTES and out.dtype == np.uint8
    _load().kqg_q6k_fill(key, b0, nblocks, _ptr(out), nthreads or default_threads())
    return out


# ----------------------------------------------------------------- Q8_0
def q80_draw(key: int, nunits: int) -> dict:
    """Logical values of Q8_0 data in units of 8 blocks (256 weights): q
    (nu,256) int8 over -128..127, d (nu,8) fp16 bit patterns (one per block
    of 32)."""
    q = np.empty((nunits, 256), np.int8)
    d = np.empty((nunits, 8), np.uint16)
    _load().kqg_q80_draw(key, nunits, _ptr(q), _ptr(d))
    return dict(q=q, d=d)


def q80_pack(q, d) -> np.ndarray:
    q = np.ascontiguousarray(q, np.int8).reshape(-1, 256)
    nu = q.shape[0]
    d = np.ascontiguousarray(d, np.uint16).reshape(nu, 8)
    out = np.empty(nu * Q8_0_UNIT_BYTES, np.uint8)
    _load().kqg_q80_pack(nu, _ptr(q), _ptr(d), _ptr(out))
    return out


def q80_fill(key: int, nunits: int, out: np.ndarray | None = None, b0: int = 0,
             nthreads: int | None = None) -> np.ndarray:
    if out is None:
        out = np.empty(nunits * Q8_0_UNIT_BYTES, np.uint8)
    assert out.nbytes >= nunits * Q8_0_UNIT_BYTES and out.dtype == np.uint8
    _load().kqg_q80_fill(key, b0, nunits, _ptr(out), nthreads or default_threads())
    return out


def fill(fmt: str, key: int, nblocks: int, out: np.ndarray | None = None,
         nthreads: int | None = None) -> np.ndarray:
    if fmt == "q4_k":
        return q4k_fill(key, nblocks, out, nthreads=nthreads)
    if fmt == "q5_k":
        return q5k_fill(key, nblocks, out, nthreads=nthreads)
    if fmt == "q2_k":
        return q2k_fill(key, nblocks, out, nthreads=nthreads)
    if fmt == "q3_k":
        return q3k_fill(key, nblocks, out, nthreads=nthreads)
    if fmt == "q6_k":
        return q6k_fill(key, nblocks, out, nthreads=nthreads)
    if fmt == "q8_0":
        return q80_fill(key, nblocks, out, nthreads=nthreads)
    raise ValueError(fmt)


def matrix(fmt: str, key: int, N: int, K: int, out: np.ndarray | None = None,
           nthreads: int | None = None) -> np.ndarray:
    """An N x K weight matrix: N rows of K/256 contiguous super-blocks."""
    return fill(fmt, key, N * (K // QK), out, nthreads)


# ---------------------------------------------------------- activations
def normal_f32(key: int, n: int, out: np.ndarray | None = None, nthreads: int | None = None) -> np.ndarray:
    """x ~ N(0,1) as fp32 (Box-Muller on the SplitMix64 stream ``key``)."""
    if out is None:
        out = np.empty(n, np.float32)
    assert out.dtype == np.float32 and out.size >= n
    _load().kqg_normal_f32(key, n, _ptr(out), nthreads or default_threads())
    return out


def topk_ids(key: int, E: int, k: int) -> np.ndarray:
    """k distinct expert ids uniform over 0..E-1 (partial Fisher-Yates)."""
    out = np.empty(k, np.int32)
    rc = _load().kqg_topk_ids(key, E, k, _ptr(out))
    if rc != 0:
        raise ValueError(f"topk_ids: bad E={E} k={k}")
    return out
