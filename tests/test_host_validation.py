"""Argument validation of the C ABI, on the host.

Each call below carries exactly one invalid argument, which the library
rejects before it touches a device; the library is loaded but no kernel
runs.  Pointers stand in as aligned addresses.  On a machine with a GPU
this file is skipped (the GPU tests check the same rejections with real
buffers)."""
import ctypes

import pytest
import torch

kq = pytest.importorskip("dequant_quant_gemv_b200.kq")

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="host-only checks; the GPU tests cover these")

P = 0x10000  # an aligned stand-in address (never dereferenced: every call below fails first)
INVALID, UNSUPPORTED = 1, 2


def multi(fmt=1, N=64, K=4096, x=P, ldx=4096, k=1, y=P, ldy=64, W=P):
    return kq.lib().kq_gemv_multi(W, fmt, N, K, x, ldx, k, y, ldy, None)


@pytest.mark.parametrize("args,status", [
    (dict(fmt=0), INVALID), (dict(fmt=7), INVALID),           # unknown formats
    (dict(K=4000), INVALID),                                   # K not a multiple of 256
    (dict(N=-1), INVALID), (dict(K=-256), INVALID),           # negative sizes
    (dict(W=0), INVALID), (dict(W=P + 8), INVALID),           # NULL or misaligned weights
    (dict(k=0), INVALID), (dict(k=9), INVALID),               # column count outside 1..8
    (dict(y=0), INVALID), (dict(y=P + 2), INVALID),           # NULL or misaligned y
    (dict(x=0), INVALID), (dict(x=P + 1), INVALID),           # NULL or misaligned x
    (dict(k=2, ldx=100), INVALID), (dict(k=2, ldy=10), INVALID),  # strides below a column
])
def test_gemv_multi_rejects(args, status):
    assert multi(**args) == status
    assert kq.lib().kq_last_error() != b""


def test_rows_off_the_16_byte_grid_pass_validation():
    # Q6_K, Q3_K and Q2_K rows need not be 16-byte aligned: such shapes are
    # not rejected as invalid (on a host without CUDA the device query fails)
    for fmt, K in ((2, 2304), (5, 1024), (4, 2304), (2, 5120)):
        for k in (1, 8):
            st = multi(fmt=fmt, K=K, ldx=K, k=k)
            assert st not in (INVALID, UNSUPPORTED), (fmt, K, k, st)


def test_n_zero_is_a_no_op():
    assert multi(N=0) == 0


@pytest.mark.parametrize("kind,gamma,eps", [(7, P, 1e-5), (1, 0, 1e-5), (1, P, 0.0), (1, P, -1.0), (1, P + 2, 1e-5)])
def test_fused_prologue_rejects(kind, gamma, eps):
    pro = kq.Prologue(kind, gamma, eps)
    st = kq.lib().kq_gemv_fused(P, 1, 64, 4096, P, 4096, 1, ctypes.byref(pro), P, 64, None)
    assert st == INVALID


def test_steps_reject_bad_lists():
    L = kq.lib()
    assert L.kq_gemv_steps(None, -1, None) == INVALID
    assert L.kq_gemv_steps(None, 2, None) == INVALID
    assert L.kq_gemv_steps(None, 0, None) == 0


def test_moe_rejects():
    L = kq.lib()
    ids = P
    # E < 1, n_ids < 0, stride below one expert, NULL ids
    assert L.kq_moe_gemv(P, 1, 0, 64, 4096, 64 * 2304, ids, 8, P, 0, P, None, None) == INVALID
    assert L.kq_moe_gemv(P, 1, 8, 64, 4096, 64 * 2304, ids, -1, P, 0, P, None, None) == INVALID
    assert L.kq_moe_gemv(P, 1, 8, 64, 4096, 64 * 2304 - 16, ids, 8, P, 0, P, None, None) == INVALID
    assert L.kq_moe_gemv(P, 1, 8, 64, 4096, 64 * 2304, 0, 8, P, 0, P, None, None) == INVALID
    assert L.kq_moe_gemv(P, 1, 8, 64, 4096, 64 * 2304, ids, 0, P, 0, P, None, None) == 0   # nothing routed


def test_unpack_and_workspace_sizes():
    L = kq.lib()
    L.kq_splitk_workspace_bytes.restype = ctypes.c_size_t
    L.kq_splitk_workspace_bytes.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int]
    assert L.kq_unpack_fields(P, 9, 4, P, P, P, None) == INVALID
    assert L.kq_unpack_fields(P, 1, -1, P, P, P, None) == INVALID
    assert L.kq_unpack_fields(P, 1, 0, P, P, P, None) == 0
    # the separate-array form: unknown format, negative count, NULL q / sc / d,
    # misaligned d or dmin; m and dmin may be NULL
    assert L.kq_unpack(P, 9, 4, P, P, P, P, P, None) == INVALID
    assert L.kq_unpack(P, 1, -1, P, P, P, P, P, None) == INVALID
    assert L.kq_unpack(P, 1, 4, 0, P, P, P, P, None) == INVALID
    assert L.kq_unpack(P, 1, 4, P, 0, P, P, P, None) == INVALID
    assert L.kq_unpack(P, 1, 4, P, P, P, 0, P, None) == INVALID
    assert L.kq_unpack(P, 1, 4, P, P, P, P + 2, P, None) == INVALID
    assert L.kq_unpack(P, 1, 4, P, P, P, P, P + 2, None) == INVALID
    assert L.kq_unpack(P, 1, 0, P, P, None, P, None, None) == 0
    for bad in ((9, 64, 4096, 1), (1, 0, 4096, 1), (1, 64, 100, 1), (1, 64, 4096, 0), (1, 64, 4096, 9)):
        assert L.kq_splitk_workspace_bytes(*bad) == 0
