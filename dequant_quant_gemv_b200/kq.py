"""Python binding of libkq (argument marshalling only).

Every computation runs in the CUDA kernels of ``libkq.so``; this module only
passes device pointers, sizes and the current torch stream through the C
ABI declared in ``include/kq.h``.  There is no CPU fallback: if the library
is missing or fails to load, the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkq.so")

Q4_K = 1
Q6_K = 2
Q5_K = 3
Q2_K = 4
Q3_K = 5
Q8_0 = 6
FORMATS = {"q4_k": Q4_K, "q6_k": Q6_K, "q5_k": Q5_K, "q2_k": Q2_K, "q3_k": Q3_K, "q8_0": Q8_0}
BLOCK_BYTES = {Q4_K: 144, Q6_K: 210, Q5_K: 176, Q2_K: 84, Q3_K: 110, Q8_0: 272}  # per 256 weights

OK = 0
STATUS = {0: "KQ_OK", 1: "KQ_ERR_INVALID_ARG", 2: "KQ_ERR_UNSUPPORTED", 3: "KQ_ERR_NOT_PINNED",
          4: "KQ_ERR_OOM", 5: "KQ_ERR_CUDA", 6: "KQ_ERR_TIMEOUT", 7: "KQ_ERR_DEVICE_CHECK",
          8: "KQ_ERR_INJECTED"}

_lib = None


class KQError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str):
        super().__init__(f"{what}: {STATUS.get(status, status)} ({detail})")
        self.status = status


class Prologue(ctypes.Structure):
    """kq_prologue: the activation prologue of kq_gemv_fused."""
    _fields_ = [("kind", ctypes.c_int), ("gamma", ctypes.c_void_p), ("eps", ctypes.c_float)]


PROLOGUE = {"none": 0, "rmsnorm": 1, "swiglu": 2}


class Step(ctypes.Structure):
    """kq_step: one GEMV of kq_gemv_steps."""
    _fields_ = [("W", ctypes.c_void_p), ("fmt", ctypes.c_int), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("x", ctypes.c_void_p), ("y", ctypes.c_void_p), ("pro", Prologue), ("after", ctypes.c_int)]


def lib() -> ctypes.CDLL:
    """Load libkq.so (built in-tree by ``dequant_quant_gemv_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libkq.so not built at {LIB_PATH}; run python -m dequant_quant_gemv_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        i64, i32, vp, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
        L.kq_version.restype = i32
        L.kq_status_str.restype = ctypes.c_char_p
        L.kq_status_str.argtypes = [i32]
        L.kq_last_error.restype = ctypes.c_char_p
        L.kq_device_fault.restype = i32
        L.kq_device_fault.argtypes = [ctypes.POINTER(ctypes.c_int)]
        L.kq_block_bytes.restype = sz
        L.kq_block_bytes.argtypes = [i32]
        L.kq_row_bytes.restype = sz
        L.kq_row_bytes.argtypes = [i32, i64]
        L.kq_gemv.restype = i32
        L.kq_gemv.argtypes = [vp, i32, i64, i64, vp, vp, vp]
        L.kq_gemv_multi.restype = i32
        L.kq_gemv_multi.argtypes = [vp, i32, i64, i64, vp, i64, i32, vp, i64, vp]
        L.kq_moe_gemv.restype = i32
        L.kq_moe_gemv.argtypes = [vp, i32, i32, i64, i64, sz, vp, i32, vp, i64, vp, vp, vp]
        L.kq_unpack.restype = i32
        L.kq_unpack.argtypes = [vp, i32, i64, vp, vp, vp, vp, vp, vp]
        L.kq_unpack_fields.restype = i32
        L.kq_unpack_fields.argtypes = [vp, i32, i64, vp, vp, vp, vp]
        L.kq_gemv_fused.restype = i32
        L.kq_gemv_fused.argtypes = [vp, i32, i64, i64, vp, i64, i32, ctypes.POINTER(Prologue), vp, i64, vp]
        L.kq_gemv_steps.restype = i32
        L.kq_gemv_steps.argtypes = [ctypes.POINTER(Step), i32, vp]
        _lib = L
    return _lib


def _fmt(fmt) -> int:
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


def _check(status: int, what: str) -> None:
    if status != OK:
        raise KQError(status, what, lib().kq_last_error().decode())


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def row_bytes(fmt, K: int) -> int:
    return int(lib().kq_row_bytes(_fmt(fmt), K))


def gemv(W: torch.Tensor, fmt, N: int, K: int, x: torch.Tensor, y: torch.Tensor | None = None,
         stream=None) -> torch.Tensor:
    """y = W x.  W: uint8 device tensor of N*row_bytes; x: K float32."""
    if y is None:
        y = torch.empty(N, dtype=torch.float32, device=x.device)
    _check(lib().kq_gemv(_dev(W, "W"), _fmt(fmt), N, K, _dev(x, "x", torch.float32),
                         _dev(y, "y", torch.float32), _stream(stream)), "kq_gemv")
    return y


def gemv_multi(W: torch.Tensor, fmt, N: int, K: int, X: torch.Tensor, Y: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """Y[c] = W X[c] for the k rows of X (shape (k, K), rows may be strided)."""
    k = X.shape[0]
    if Y is None:
        Y = torch.empty((k, N), dtype=torch.float32, device=X.device)
    _check(lib().kq_gemv_multi(_dev(W, "W"), _fmt(fmt), N, K, _dev(X, "X", torch.float32), X.stride(0), k,
                               _dev(Y, "Y", torch.float32), Y.stride(0), _stream(stream)), "kq_gemv_multi")
    return Y


def gemv_fused(W: torch.Tensor, fmt, N: int, K: int, X: torch.Tensor, kind: str = "none",
               gamma: torch.Tensor | None = None, eps: float = 1e-5, Y: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """Y[c] = W P(X[c]) for the k rows of X: P = "none", "rmsnorm" (with gamma,
    eps; rows of K) or "swiglu" (rows of 2K: [gate; up])."""
    if X.dim() == 1:
        X = X[None, :]
    k = X.shape[0]
    if Y is None:
        Y = torch.empty((k, N), dtype=torch.float32, device=X.device)
    pro = Prologue(PROLOGUE[kind], _dev(gamma, "gamma", torch.float32) if gamma is not None else None, eps)
    _check(lib().kq_gemv_fused(_dev(W, "W"), _fmt(fmt), N, K, _dev(X, "X", torch.float32), X.stride(0), k,
                               ctypes.byref(pro), _dev(Y, "Y", torch.float32), Y.stride(0), _stream(stream)),
           "kq_gemv_fused")
    return Y


def make_step(W: torch.Tensor, fmt, N: int, K: int, x: torch.Tensor, y: torch.Tensor, kind: str = "none",
              gamma: torch.Tensor | None = None, eps: float = 1e-5, after: bool = False) -> Step:
    """A kq_step for gemv_steps: y = W P(x), one column (x of K floats, 2K for
    "swiglu"); `after`: x is written by an earlier step of the same call."""
    pro = Prologue(PROLOGUE[kind], _dev(gamma, "gamma", torch.float32) if gamma is not None else None, eps)
    return Step(_dev(W, "W"), _fmt(fmt), N, K, _dev(x, "x", torch.float32), _dev(y, "y", torch.float32), pro,
                1 if after else 0)


def gemv_steps(steps, stream=None) -> None:
    """kq_gemv_steps over a list of Step (see make_step), in order."""
    arr = (Step * max(1, len(steps)))(*steps)
    _check(lib().kq_gemv_steps(arr, len(steps), _stream(stream)), "kq_gemv_steps")


def _splitk_sigs(L):
    if not getattr(L, "_splitk_ready", False):
        L.kq_splitk_workspace_bytes.restype = ctypes.c_size_t
        L.kq_splitk_workspace_bytes.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int]
        L.kq_gemv_splitk.restype = ctypes.c_int
        L.kq_gemv_splitk.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                     ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                     ctypes.c_size_t, ctypes.c_void_p]
        L._splitk_ready = True
    return L


def splitk_workspace_bytes(fmt, N: int, K: int, k: int = 1) -> int:
    return int(_splitk_sigs(lib()).kq_splitk_workspace_bytes(_fmt(fmt), N, K, k))


def gemv_splitk(W: torch.Tensor, fmt, N: int, K: int, X: torch.Tensor, Y: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """kq_gemv_splitk: X is (K,) or (k, K); the workspace is allocated here
    (torch) when not given."""
    L = _splitk_sigs(lib())
    X2 = X.view(1, -1) if X.dim() == 1 else X
    k = X2.shape[0]
    if Y is None:
        Y = torch.empty((k, N), dtype=torch.float32, device=X.device)
    Y2 = Y.view(1, -1) if Y.dim() == 1 else Y
    need = splitk_workspace_bytes(fmt, N, K, k)
    if workspace is None:
        workspace = torch.empty(max(1, (need + 3) // 4), dtype=torch.float32, device=X.device)
    _check(L.kq_gemv_splitk(_dev(W, "W"), _fmt(fmt), N, K, _dev(X2, "X", torch.float32), X2.stride(0), k,
                            _dev(Y2, "Y", torch.float32), Y2.stride(0), _dev(workspace, "workspace"),
                            workspace.numel() * workspace.element_size(), _stream(stream)), "kq_gemv_splitk")
    return Y


def gemv_splitk_noalloc(W: torch.Tensor, fmt, N: int, K: int, X: torch.Tensor, Y: torch.Tensor,
                        stream=None) -> torch.Tensor:
    """kq_gemv_splitk_noalloc: split-K GEMV with its partial sums in the
    library's built-in scratch, for callers that cannot allocate device
    memory.  X is (K,) or (k, K); Y must be given (this call allocates
    nothing)."""
    L = lib()
    if not getattr(L, "_noalloc_ready", False):
        L.kq_gemv_splitk_noalloc.restype = ctypes.c_int
        L.kq_gemv_splitk_noalloc.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                             ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p,
                                             ctypes.c_int64, ctypes.c_void_p]
        L._noalloc_ready = True
    X2 = X.view(1, -1) if X.dim() == 1 else X
    Y2 = Y.view(1, -1) if Y.dim() == 1 else Y
    _check(L.kq_gemv_splitk_noalloc(_dev(W, "W"), _fmt(fmt), N, K, _dev(X2, "X", torch.float32), X2.stride(0),
                                    X2.shape[0], _dev(Y2, "Y", torch.float32), Y2.stride(0), _stream(stream)),
           "kq_gemv_splitk_noalloc")
    return Y


def moe_gemv(W_experts: torch.Tensor, fmt, E: int, N: int, K: int, ids: torch.Tensor, x: torch.Tensor,
             y: torch.Tensor | None = None, status: torch.Tensor | None = None, expert_stride: int | None = None,
             stream=None) -> torch.Tensor:
    """y[i] = W_{ids[i]} x_i; x is (K,) shared or (n_ids, K) per id."""
    n = ids.numel()
    if expert_stride is None:
        expert_stride = N * row_bytes(fmt, K)
    if y is None:
        y = torch.empty((n, N), dtype=torch.float32, device=x.device)
    x_stride = 0 if x.dim() == 1 else x.stride(0)
    _check(lib().kq_moe_gemv(_dev(W_experts, "W_experts"), _fmt(fmt), E, N, K, expert_stride,
                             _dev(ids, "ids", torch.int32), n, _dev(x, "x", torch.float32), x_stride,
                             _dev(y, "y", torch.float32), None if status is None else _dev(status, "status"),
                             _stream(stream)), "kq_moe_gemv")
    return y


def unpack(W: torch.Tensor, fmt, n_blocks: int, stream=None):
    """(q, sc, d) integer fields as decoded on the GPU, packed form
    (kq_unpack_fields in kq.h)."""
    q = torch.empty(n_blocks * 256, dtype=torch.uint8, device=W.device)
    sc = torch.empty(n_blocks * 16, dtype=torch.uint8, device=W.device)
    d = torch.empty(n_blocks * 2, dtype=torch.float32, device=W.device)
    _check(lib().kq_unpack_fields(_dev(W, "W"), _fmt(fmt), n_blocks, q.data_ptr(), sc.data_ptr(), d.data_ptr(),
                                  _stream(stream)), "kq_unpack_fields")
    return q, sc, d


def unpack_split(W: torch.Tensor, fmt, n_blocks: int, stream=None):
    """(q, sc_or_s, m, d, dmin) as decoded on the GPU (kq_unpack in kq.h):
    q int8 (n_blocks*256), sc_or_s and m uint8 (n_blocks*16 each), d and
    dmin float32 (n_blocks each)."""
    q = torch.empty(n_blocks * 256, dtype=torch.int8, device=W.device)
    sc = torch.empty(n_blocks * 16, dtype=torch.uint8, device=W.device)
    m = torch.empty(n_blocks * 16, dtype=torch.uint8, device=W.device)
    d = torch.empty(n_blocks, dtype=torch.float32, device=W.device)
    dmin = torch.empty(n_blocks, dtype=torch.float32, device=W.device)
    _check(lib().kq_unpack(_dev(W, "W"), _fmt(fmt), n_blocks, q.data_ptr(), sc.data_ptr(), m.data_ptr(),
                           d.data_ptr(), dmin.data_ptr(), _stream(stream)), "kq_unpack")
    return q, sc, m, d, dmin


def read_probe(buf: torch.Tensor, mode: int, out: torch.Tensor, stream=None) -> None:
    """kq_read_probe: read `buf` once (mode 0 loads, mode 1 the bulk-copy
    ring of the GEMV kernels); XOR of the data into out (int32, 1 element)."""
    L = lib()
    L.kq_read_probe.restype = ctypes.c_int
    L.kq_read_probe.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    _check(L.kq_read_probe(_dev(buf, "buf"), buf.numel() * buf.element_size(), mode, _dev(out, "out"),
                           _stream(stream)), "kq_read_probe")


def inject(spec: str | None) -> None:
    """kq_inject: test hook ("hold@S" withholds one weight stage of the next
    single-column launch so that its bounded wait runs out)."""
    L = lib()
    L.kq_inject.restype = ctypes.c_int
    L.kq_inject.argtypes = [ctypes.c_char_p]
    _check(L.kq_inject(spec.encode() if spec else None), "kq_inject")


def device_fault() -> int:
    out = ctypes.c_int(0)
    _check(lib().kq_device_fault(ctypes.byref(out)), "kq_device_fault")
    return out.value


# --------------------------------------------------------------- chain
class MatrixDesc(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("fmt", ctypes.c_int), ("N", ctypes.c_int64), ("K", ctypes.c_int64)]


def _chain_sigs(L):
    if getattr(L, "_chain_ready", False):
        return
    vp = ctypes.c_void_p
    L.kq_chain_create.restype = ctypes.c_int
    L.kq_chain_create.argtypes = [ctypes.POINTER(MatrixDesc), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                  ctypes.POINTER(vp)]
    L.kq_chain_create_resident.restype = ctypes.c_int
    L.kq_chain_create_resident.argtypes = [ctypes.POINTER(MatrixDesc), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.POINTER(vp)]
    L.kq_chain_plan.restype = ctypes.c_int
    L.kq_chain_plan.argtypes = [ctypes.POINTER(MatrixDesc), ctypes.c_int, ctypes.c_int, ctypes.c_size_t,
                                ctypes.c_int, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
    L.kq_chain_resident_layers.restype = ctypes.c_int
    L.kq_chain_resident_layers.argtypes = [vp]
    L.kq_chain_slot_bytes.restype = ctypes.c_size_t
    L.kq_chain_slot_bytes.argtypes = [vp]
    L.kq_chain_run.restype = ctypes.c_int
    L.kq_chain_run.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), vp]
    L.kq_chain_wait.restype = ctypes.c_int
    L.kq_chain_wait.argtypes = [vp, ctypes.c_int64]
    L.kq_chain_last_error.restype = ctypes.c_char_p
    L.kq_chain_destroy.restype = None
    L.kq_chain_destroy.argtypes = [vp]
    L._chain_ready = True


def chain_plan(layers, budget_bytes: int, max_slots: int = 4):
    """kq_chain_plan: (n_resident, n_slots) for a device-memory budget.
    layers: list over layers of lists of (W, fmt, N, K) (W unused here)."""
    L = lib()
    _chain_sigs(L)
    flat = [m for layer in layers for m in layer]
    arr = (MatrixDesc * len(flat))()
    for i, (W, fmt, N, K) in enumerate(flat):
        arr[i] = MatrixDesc(None if W is None else W.data_ptr(), _fmt(fmt), N, K)
    r, s = ctypes.c_int(), ctypes.c_int()
    st = L.kq_chain_plan(arr, len(layers), len(layers[0]), budget_bytes, max_slots, ctypes.byref(r), ctypes.byref(s))
    if st != OK:
        raise KQError(st, "kq_chain_plan", L.kq_chain_last_error().decode())
    return int(r.value), int(s.value)


def _moe_stream_sigs(L):
    if getattr(L, "_moe_stream_sigs", False):
        return
    i64, i32, vp, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
    L.kq_moe_stream_create.restype = i32
    L.kq_moe_stream_create.argtypes = [vp, i32, i32, i64, i64, sz, i32, i32, ctypes.POINTER(vp)]
    L.kq_moe_stream_run.restype = i32
    L.kq_moe_stream_run.argtypes = [vp, vp, i32, vp, i64, vp, vp]
    L.kq_moe_stream_wait.restype = i32
    L.kq_moe_stream_wait.argtypes = [vp, i64]
    L.kq_moe_stream_destroy.restype = None
    L.kq_moe_stream_destroy.argtypes = [vp]
    L.kq_moe_stream_last_error.restype = ctypes.c_char_p
    L._moe_stream_sigs = True


class MoEStream:
    """Routed experts kept in pinned host memory and copied to the device on
    demand (kq_moe_stream_* in kq.h).

    W_host: pinned uint8 tensor holding E expert matrices (N x K in fmt),
    expert e at byte e * stride (default N * row_bytes)."""

    def __init__(self, W_host, fmt, E: int, N: int, K: int, max_ids: int, n_sets: int = 2,
                 stride: int | None = None):
        L = lib()
        _moe_stream_sigs(L)
        self._L = L
        if W_host.is_cuda:
            raise ValueError("streamed experts must be host memory")
        self._keep = W_host
        self.N, self.K, self.max_ids = N, K, max_ids
        stride = stride if stride is not None else N * row_bytes(fmt, K)
        h = ctypes.c_void_p()
        st = L.kq_moe_stream_create(W_host.data_ptr(), _fmt(fmt), E, N, K, stride, max_ids, n_sets,
                                    ctypes.byref(h))
        if st != OK:
            raise KQError(st, "kq_moe_stream_create", L.kq_moe_stream_last_error().decode())
        self._h = h

    def run(self, ids_host, x, x_stride: int = 0, y=None, stream=None):
        """ids_host: int32 numpy array or CPU tensor; x, y: device tensors."""
        ids = np.ascontiguousarray(np.asarray(ids_host, dtype=np.int32))
        n = int(ids.size)
        if y is None:
            y = torch.empty((n, self.N), dtype=torch.float32, device=x.device)
        st = self._L.kq_moe_stream_run(self._h, ids.ctypes.data, n, _dev(x, "x", torch.float32), x_stride,
                                       _dev(y, "y", torch.float32), _stream(stream))
        if st != OK:
            raise KQError(st, "kq_moe_stream_run", self._L.kq_moe_stream_last_error().decode())
        return y

    def wait(self, timeout_ms: int = -1) -> None:
        st = self._L.kq_moe_stream_wait(self._h, timeout_ms)
        if st != OK:
            raise KQError(st, "kq_moe_stream_wait", self._L.kq_moe_stream_last_error().decode())

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._L.kq_moe_stream_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def gguf_format(ggml_type: int) -> int:
    """libkq format id of a ggml type id (0 if none): kq_gguf_kq_format."""
    L = lib()
    L.kq_gguf_kq_format.restype = ctypes.c_int
    L.kq_gguf_kq_format.argtypes = [ctypes.c_int]
    return int(L.kq_gguf_kq_format(int(ggml_type)))


class GGUF:
    """Tensor table and tensor bytes of a GGUF file (kq_gguf_* in kq.h)."""

    def __init__(self, path: str):
        L = lib()
        if not getattr(L, "_gguf_sigs", False):
            i32, vp, u64 = ctypes.c_int, ctypes.c_void_p, ctypes.c_uint64
            L.kq_gguf_open.restype = i32
            L.kq_gguf_open.argtypes = [ctypes.c_char_p, ctypes.POINTER(vp)]
            L.kq_gguf_tensor_count.restype = i32
            L.kq_gguf_tensor_count.argtypes = [vp]
            L.kq_gguf_tensor_info.restype = i32
            L.kq_gguf_tensor_info.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(i32),
                                              ctypes.POINTER(i32), ctypes.POINTER(ctypes.c_int64),
                                              ctypes.POINTER(u64), ctypes.POINTER(u64)]
            L.kq_gguf_find.restype = i32
            L.kq_gguf_find.argtypes = [vp, ctypes.c_char_p]
            L.kq_gguf_kq_format.restype = i32
            L.kq_gguf_kq_format.argtypes = [i32]
            L.kq_gguf_read.restype = i32
            L.kq_gguf_read.argtypes = [vp, i32, vp, u64]
            L.kq_gguf_close.restype = None
            L.kq_gguf_close.argtypes = [vp]
            L.kq_gguf_last_error.restype = ctypes.c_char_p
            L._gguf_sigs = True
        self._L = L
        h = ctypes.c_void_p()
        st = L.kq_gguf_open(os.fsencode(path), ctypes.byref(h))
        if st != OK:
            raise KQError(st, "kq_gguf_open", L.kq_gguf_last_error().decode())
        self._h = h

    def __len__(self) -> int:
        return int(self._L.kq_gguf_tensor_count(self._h))

    def info(self, i: int) -> dict:
        name, t, nd = ctypes.c_char_p(), ctypes.c_int(), ctypes.c_int()
        dims = (ctypes.c_int64 * 4)()
        off, nb = ctypes.c_uint64(), ctypes.c_uint64()
        st = self._L.kq_gguf_tensor_info(self._h, i, ctypes.byref(name), ctypes.byref(t), ctypes.byref(nd), dims,
                                         ctypes.byref(off), ctypes.byref(nb))
        if st != OK:
            raise KQError(st, "kq_gguf_tensor_info", self._L.kq_gguf_last_error().decode())
        return dict(name=name.value.decode(), type=t.value, dims=list(dims)[:nd.value], offset=off.value,
                    nbytes=nb.value, fmt=int(self._L.kq_gguf_kq_format(t.value)))

    def find(self, name: str) -> int:
        return int(self._L.kq_gguf_find(self._h, name.encode()))

    def read(self, name_or_index) -> np.ndarray:
        i = name_or_index if isinstance(name_or_index, int) else self.find(name_or_index)
        nb = self.info(i)["nbytes"]
        out = np.empty(nb, np.uint8)
        st = self._L.kq_gguf_read(self._h, i, out.ctypes.data, nb)
        if st != OK:
            raise KQError(st, "kq_gguf_read", self._L.kq_gguf_last_error().decode())
        return out

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._L.kq_gguf_close(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Chain:
    """Layer chain whose weights stay in pinned host memory and stream
    through ``n_slots`` device slots (kq_chain_* in kq.h).

    mats: list over layers of lists of (W_host_pinned_uint8_tensor, fmt, N, K).
    n_resident: leading layers copied once into device memory of their own
    (kq_chain_create_resident); the rest stream.
    """

    def __init__(self, mats, n_slots: int = 4, n_resident: int = 0):
        L = lib()
        _chain_sigs(L)
        self._L = L
        self.n_layers = len(mats)
        self.per_layer = len(mats[0])
        flat = [m for layer in mats for m in layer]
        self._keep = [m[0] for m in flat]  # keep the host tensors alive
        arr = (MatrixDesc * len(flat))()
        for i, (W, fmt, N, K) in enumerate(flat):
            if W.is_cuda:
                raise ValueError("chain weights must be host memory")
            arr[i] = MatrixDesc(W.data_ptr(), _fmt(fmt), N, K)
        h = ctypes.c_void_p()
        st = L.kq_chain_create_resident(arr, self.n_layers, self.per_layer, n_resident, n_slots, ctypes.byref(h))
        if st != OK:
            raise KQError(st, "kq_chain_create_resident", L.kq_chain_last_error().decode())
        self._h = h

    @property
    def slot_bytes(self) -> int:
        return int(self._L.kq_chain_slot_bytes(self._h))

    @property
    def resident_layers(self) -> int:
        return int(self._L.kq_chain_resident_layers(self._h))

    def run(self, xs, ys, stream=None) -> None:
        n = self.n_layers * self.per_layer
        assert len(xs) == n and len(ys) == n
        xa = (ctypes.c_void_p * n)(*[_dev(x, "x", torch.float32) for x in xs])
        ya = (ctypes.c_void_p * n)(*[_dev(y, "y", torch.float32) for y in ys])
        st = self._L.kq_chain_run(self._h, xa, ya, _stream(stream))
        if st != OK:
            raise KQError(st, "kq_chain_run", self._L.kq_chain_last_error().decode())

    def wait(self, timeout_ms: int = -1) -> None:
        st = self._L.kq_chain_wait(self._h, timeout_ms)
        if st != OK:
            raise KQError(st, "kq_chain_wait", self._L.kq_chain_last_error().decode())

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._L.kq_chain_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class LayerDesc(ctypes.Structure):
    """kq_layer_desc: one layer's matrices for kq_stream_chain_create."""
    _fields_ = [("mats", ctypes.POINTER(MatrixDesc)), ("n_mats", ctypes.c_int)]


class StreamChain(Chain):
    """The streamed chain through the per-layer entry points
    kq_stream_chain_create / kq_stream_chain / kq_stream_chain_destroy."""

    def __init__(self, mats, n_slots: int = 4):
        L = lib()
        _chain_sigs(L)
        if not getattr(L, "_stream_chain_ready", False):
            vp = ctypes.c_void_p
            L.kq_stream_chain_create.restype = ctypes.c_int
            L.kq_stream_chain_create.argtypes = [ctypes.POINTER(LayerDesc), ctypes.c_int, ctypes.c_int,
                                                 ctypes.POINTER(vp)]
            L.kq_stream_chain.restype = ctypes.c_int
            L.kq_stream_chain.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), vp, ctypes.c_int64]
            L.kq_stream_chain_destroy.restype = None
            L.kq_stream_chain_destroy.argtypes = [vp]
            L._stream_chain_ready = True
        self._L = L
        self.n_layers = len(mats)
        self.per_layer = len(mats[0])
        self._keep = [m[0] for layer in mats for m in layer]
        self._arrays = []
        layers = (LayerDesc * self.n_layers)()
        for l, layer in enumerate(mats):
            arr = (MatrixDesc * len(layer))()
            for i, (W, fmt, N, K) in enumerate(layer):
                if W.is_cuda:
                    raise ValueError("chain weights must be host memory")
                arr[i] = MatrixDesc(W.data_ptr(), _fmt(fmt), N, K)
            self._arrays.append(arr)
            layers[l] = LayerDesc(arr, len(layer))
        h = ctypes.c_void_p()
        st = L.kq_stream_chain_create(layers, self.n_layers, n_slots, ctypes.byref(h))
        if st != OK:
            raise KQError(st, "kq_stream_chain_create", L.kq_chain_last_error().decode())
        self._h = h

    def run_wait(self, xs, ys, timeout_ms: int = -1, stream=None) -> None:
        """kq_stream_chain: one pass, waited for on the host (bounded)."""
        n = self.n_layers * self.per_layer
        assert len(xs) == n and len(ys) == n
        xa = (ctypes.c_void_p * n)(*[_dev(x, "x", torch.float32) for x in xs])
        ya = (ctypes.c_void_p * n)(*[_dev(y, "y", torch.float32) for y in ys])
        st = self._L.kq_stream_chain(self._h, xa, ya, _stream(stream), timeout_ms)
        if st != OK:
            raise KQError(st, "kq_stream_chain", self._L.kq_chain_last_error().decode())

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._L.kq_stream_chain_destroy(self._h)
            self._h = None
