"""The seeded generators: reproducible, bf16 storage exact, and the
distribution parameters each workload states."""

import numpy as np

from bit_weight_only_lcvq_b200 import synth


def test_bf16_rounding_ties_to_even_and_roundtrip():
    a = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e38], dtype=np.float32)
    r = synth.round_to_bf16(a)
    assert r[0] == 1.0 and r[1] == 1.0 and r[2] == 1.0 + 2 ** -6 and r[3] == -2.5
    bits = synth.bf16_bits(r)
    assert np.array_equal(synth.from_bf16_bits(bits), r)


def test_workloads_are_reproducible_and_shaped():
    a = synth.workload(2, M=4, d_in=256, d_out=128)
    b = synth.workload(2, M=4, d_in=256, d_out=128)
    for k in ("Wp", "A", "B", "X", "dY"):
        assert np.array_equal(a[k], b[k])
    assert a["Wp"].shape == (128, 256) and a["X"].shape == (4, 256)
    # B = -1.5 A 1, formed in fp64 before A is rounded to fp32
    assert np.allclose(a["B"], -1.5 * a["A"].astype(np.float64).sum(1), rtol=1e-6, atol=1e-9)
    synth.bf16_bits(a["X"])           # raises if not bf16-representable
    # 1% outlier channels scaled x20
    big = np.abs(a["X"]).max(axis=0) > 8
    assert 1 <= big.sum() <= 3


def test_stack_matrix_shapes():
    m = synth.stack_matrix(0, 6, 8)
    assert m["packed"].shape == (4096, 11008 // 4) and m["X"].shape == (8, 11008)
