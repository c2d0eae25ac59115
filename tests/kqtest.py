"""Shared helpers for the GPU parity tests (inputs come from kqgen, expected
values from the oracle; nothing here computes the method)."""
from __future__ import annotations

import numpy as np
import torch

import kqgen
import oracle

REL, ABS = 1e-3, 1e-6   # |y - y_ref| <= REL * sum_i |w_i x_i| + ABS, per output


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def assert_close(y_gpu, y_ref, s_ref, what=""):
    y = y_gpu.detach().cpu().numpy().astype(np.float64) if isinstance(y_gpu, torch.Tensor) else np.asarray(y_gpu)
    err = np.abs(y - y_ref)
    bound = REL * s_ref + ABS
    bad = np.nonzero(~(err <= bound))[0]
    assert bad.size == 0, (f"{what}: {bad.size} outputs out of tolerance; first {bad[:5].tolist()} "
                           f"err={err[bad[:5]].tolist()} bound={bound[bad[:5]].tolist()}")
    return float(np.max(err / bound)) if err.size else 0.0


def matrix(fmt: str, seed: int, N: int, K: int) -> np.ndarray:
    return kqgen.matrix(fmt, seed, N, K)


def x_vec(seed: int, K: int) -> np.ndarray:
    return kqgen.normal_f32(seed, K)


def oracle_gemv(fmt, W, N, K, x):
    return oracle.gemv(fmt, W, N, K, x, nthreads=0)
