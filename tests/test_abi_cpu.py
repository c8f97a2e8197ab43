"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol the header declares, and rejects bad arguments before touching a
device."""

import ctypes
import os
import re

import pytest

from bit_weight_only_lcvq_b200 import lcvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "lcvq.h")).read()
    return sorted(set(re.findall(r"LCVQ_API\s+[\w\s\*]+?\b(lcvq_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = lcvq.lib()
    declared = _header_functions()
    assert set(declared) == set(lcvq.EXPORTS)
    for name in declared:
        assert hasattr(L, name), name


def test_status_strings():
    L = lcvq.lib()
    for code, name in lcvq.STATUS.items():
        assert L.lcvq_status_string(code).decode() == name


def test_workspace_size_rules():
    ws = lcvq.workspace_size(lcvq.OP_GEMM, __import__("torch").bfloat16, 16, 4096, 4096, 8)
    assert ws >= 256 + 16 * 4096 * 2 + 16 * 4
    assert lcvq.lib().lcvq_workspace_size(lcvq.OP_GEMM, 1, -1, 8, 64, 8) == 0
    assert lcvq.lib().lcvq_workspace_size(lcvq.OP_GEMM, 1, 1, 8, 64, 3) == 0


def test_invalid_arguments_rejected_without_device():
    L = lcvq.lib()
    # bad d, bad shapes: rejected by validation (before any CUDA call)
    assert L.lcvq_assign_pack(None, 4, 12, 4, None, None, None) == 1      # d_in % 8
    assert L.lcvq_assign_pack(None, 4, 64, 3, None, None, None) == 1      # d not in {1,2,4,8}
    assert L.lcvq_assign_pack(None, 0, 64, 8, None, None, None) == 0      # empty: no-op
    assert L.lcvq_decode(None, 4, 24, 8, None, None, None, 1, None) == 1  # d_in % 16
    assert L.lcvq_gemm(None, 1, 4, None, 8, 96, 8, None, None, None, 0, None, 0, None) == 1
    assert L.lcvq_gemm(None, 1, 4, None, 12, 64, 8, None, None, None, 0, None, 0, None) == 1
    assert L.lcvq_gemm(None, 1, 0, None, 8, 64, 8, None, None, None, 0, None, 0, None) == 0
    assert L.lcvq_gemm(None, 7, 4, None, 8, 64, 8, None, None, None, 0, None, 0, None) == 1
    assert L.lcvq_gemm(None, 1, 4, None, 8, 64, 8, None, None, None, 9, None, 0, None) == 1
    # misaligned output pointer is caught before the device check
    assert L.lcvq_gemm(None, 1, 4, None, 8, 64, 8, None, None, 8, 0, None, 0, None) == 3
    assert L.lcvq_gemm_backward(None, None, 1, 4, None, None, 8, 64, 8, None, None, None,
                                None, None, None, None, 0, None) == 1      # dA/dB required
