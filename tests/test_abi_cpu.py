"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol the header declares, and rejects bad arguments before touching a
device."""

import ctypes
import os
import re

import pytest
import torch

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


def test_grouped_gemm_rejects_bad_groups_without_device():
    L = lcvq.lib()
    Item = lcvq.GemmItem

    def items(*shapes):
        arr = (Item * len(shapes))()
        for i, (d_out, d_in) in enumerate(shapes):
            arr[i] = Item(16, 16, 16, 16, 16, d_out, d_in)  # aligned dummy pointers
        return arr

    good = items((4096, 4096), (11008, 4096), (4096, 11008))
    need = L.lcvq_workspace_size_grouped(good, 3, 8, 8)
    # per item: X'' (M d_in bf16), then corr [M] and the int8 path's scales [M][8] (fp32)
    per = [256 * -(-(8 * k * 2) // 256) + 256 * -(-(8 * 36) // 256)
           for _, k in ((0, 4096), (0, 4096), (0, 11008))]
    assert need == 256 + sum(per)
    assert L.lcvq_workspace_size_grouped(good, 3, 33, 8) == 0                 # M > 32
    assert L.lcvq_workspace_size_grouped(good, 3, 0, 8) == 0                  # M < 1
    assert L.lcvq_workspace_size_grouped(good, 0, 8, 8) == 0                  # empty group
    assert L.lcvq_workspace_size_grouped(good, 3, 8, 3) == 0                  # d
    assert L.lcvq_workspace_size_grouped(items((4096, 4000)), 1, 8, 8) == 0   # d_in % 64
    assert L.lcvq_workspace_size_grouped(items((4100, 4096)), 1, 8, 8) == 0   # d_out % 8
    assert L.lcvq_workspace_size_grouped(items((0, 4096)), 1, 8, 8) == 0      # empty matrix
    # every failure is reported before any device call
    assert L.lcvq_gemm_grouped(good, 3, 33, 8, 256, need, None) == 1
    assert L.lcvq_gemm_grouped(good, 3, 8, 8, None, need, None) == 1          # no workspace
    assert L.lcvq_gemm_grouped(good, 3, 8, 8, 8, need, None) == 3             # misaligned
    assert L.lcvq_gemm_grouped(good, 3, 8, 8, 256, need - 1, None) == 4       # too small
    bad = items((4096, 4096), (4096, 4096))
    bad[1].Y = 8                                                              # one bad item
    assert L.lcvq_gemm_grouped(bad, 2, 8, 8, 256, 1 << 30, None) == 3
    bad[1].Y = None
    assert L.lcvq_gemm_grouped(bad, 2, 8, 8, 256, 1 << 30, None) == 1


def test_fit_affine_rejects_bad_arguments_without_device():
    L = lcvq.lib()
    assert L.lcvq_workspace_size(lcvq.OP_FIT_AFFINE, 0, 0, 4096, 4096, 8) > 256
    assert L.lcvq_workspace_size(lcvq.OP_FIT_AFFINE, 0, 0, 4096, 4096, 3) == 0
    assert L.lcvq_fit_affine(16, 16, 8, 24, 8, None, 16, 16, 256, 1 << 20, None) == 1  # d_in % 16
    assert L.lcvq_fit_affine(16, 16, 8, 64, 3, None, 16, 16, 256, 1 << 20, None) == 1  # d
    assert L.lcvq_fit_affine(16, 16, 8, 64, 8, None, None, 16, 256, 1 << 20, None) == 1  # no A
    assert L.lcvq_fit_affine(16, 16, 8, 64, 8, 8, 16, 16, 256, 1 << 20, None) == 3     # h misaligned
    assert L.lcvq_fit_affine(16, 16, 8, 64, 8, None, 16, 16, 256, 16, None) == 4       # workspace


def test_dge_scale_rejects_bad_arguments_without_device():
    L = lcvq.lib()
    assert L.lcvq_dge_scale(16, 16, 6, 2.0, None) == 1            # n % 4
    assert L.lcvq_dge_scale(16, 16, 8, 0.0, None) == 1            # k <= 0
    assert L.lcvq_dge_scale(16, 16, 8, float("nan"), None) == 1   # k not finite
    assert L.lcvq_dge_scale(None, 16, 8, 2.0, None) == 1
    assert L.lcvq_dge_scale(8, 16, 8, 2.0, None) == 3             # misaligned
    assert L.lcvq_dge_scale(None, None, 0, 2.0, None) == 0        # empty: no-op


def test_assign_ldlq_rejects_bad_arguments_without_device():
    L = lcvq.lib()
    ws = L.lcvq_workspace_size(lcvq.OP_ASSIGN_LDLQ, 0, 0, 50, 256, 8)
    assert ws == 256 + 64 * 256 * 4                                     # rows padded to 32
    assert L.lcvq_workspace_size(lcvq.OP_ASSIGN_LDLQ, 0, 0, 50, 256, 3) == 0
    assert L.lcvq_assign_ldlq(16, 16, 8, 96, 8, 16, 256, 1 << 20, None) == 1    # d_in % 64
    assert L.lcvq_assign_ldlq(16, 16, 8, 64, 3, 16, 256, 1 << 20, None) == 1    # d
    assert L.lcvq_assign_ldlq(16, 16, 8, (1 << 20) + 64, 8, 16, 256, 1 << 40, None) == 1  # d_in
    assert L.lcvq_assign_ldlq(16, None, 8, 64, 8, 16, 256, 1 << 20, None) == 1  # no U
    assert L.lcvq_assign_ldlq(16, 16, 8, 64, 8, 16, None, 1 << 20, None) == 1   # no workspace
    assert L.lcvq_assign_ldlq(16, 8, 8, 64, 8, 16, 256, 1 << 20, None) == 3     # U misaligned
    assert L.lcvq_assign_ldlq(16, 16, 8, 64, 8, 16, 256, 1024, None) == 4       # workspace
    assert L.lcvq_assign_ldlq(None, None, 0, 64, 8, None, 256, 0, None) == 0    # empty: no-op


def test_gemm_dimension_limits_without_device():
    """Matrix dimensions above 2^30 are refused before anything runs (the GEMV
    kernels index rows and columns in 32 bits)."""
    L = lcvq.lib()
    big = (1 << 30) + 64
    assert L.lcvq_gemm(None, 1, 4, None, 8, big, 8, None, None, None, 0, None, 0, None) == 1
    assert L.lcvq_gemm(None, 1, 4, None, big - 56, 64, 8, None, None, None, 0, None, 0, None) == 1
    assert L.lcvq_gemm_backward(None, None, 1, 4, None, None, 8, big, 8, None, None, None,
                                None, None, None, None, 0, None) == 1


def test_binding_refuses_host_tensors():
    """The binding hands kernels device addresses only: a host tensor is
    refused before any call reaches the library (no CPU fallback either)."""
    with pytest.raises(ValueError, match="CUDA tensor"):
        lcvq._ptr(torch.zeros(4))
    assert lcvq._ptr(None) is None
