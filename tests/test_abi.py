"""The C-ABI library builds, loads and exports every entry point that
include/kq.h declares (host-only calls; no GPU needed)."""
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^KQ_API\s+[\w\s\*]+?\b(kq_\w+)\s*\(", src, re.M)
    return names


@pytest.fixture(scope="module")
def libkq():
    from dequant_quant_gemv_b200 import build
    build.build()
    from dequant_quant_gemv_b200 import kq
    return kq


def test_header_declares_entry_points():
    names = declared_symbols()
    for n in ("kq_gemv", "kq_gemv_multi", "kq_moe_gemv", "kq_unpack", "kq_row_bytes", "kq_status_str",
              "kq_stream_chain_create", "kq_stream_chain", "kq_stream_chain_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol(libkq):
    out = subprocess.check_output(["nm", "-D", "--defined-only", libkq.LIB_PATH]).decode()
    exported = set(re.findall(r"\sT\s(kq_\w+)$", out, re.M))
    missing = [n for n in declared_symbols() if n not in exported]
    assert not missing, missing
    L = libkq.lib()
    for n in declared_symbols():
        assert hasattr(L, n)


def test_host_only_helpers(libkq):
    L = libkq.lib()
    assert L.kq_row_bytes(1, 4096) == 16 * 144
    assert L.kq_row_bytes(2, 14336) == 56 * 210
    assert L.kq_row_bytes(1, 300) == 0
    assert L.kq_block_bytes(3) == 176                 # Q5_K
    assert L.kq_row_bytes(3, 4096) == 16 * 176
    assert L.kq_block_bytes(4) == 84                  # Q2_K
    assert L.kq_block_bytes(5) == 110                 # Q3_K
    assert L.kq_row_bytes(5, 2048) == 8 * 110
    assert L.kq_block_bytes(6) == 272                 # Q8_0, per 8 blocks of 32
    assert L.kq_row_bytes(6, 4096) == 16 * 272
    assert L.kq_block_bytes(7) == 0                   # no such format
    assert L.kq_block_bytes(0) == 0
    assert L.kq_status_str(0) == b"ok"
    assert L.kq_version() >= 100


def test_no_cpu_fallback_in_product():
    """The product package never imports the oracle or the generator."""
    pkg = os.path.join(ROOT, "dequant_quant_gemv_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in src.replace("the oracle", ""), f
                assert "kqgen" not in src, f
