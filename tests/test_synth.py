"""The seeded generators' storage-format roundings, on hand-worked values.

bf16 keeps 7 explicit mantissa bits and tf32 10 (the mHC paper's section 4.3.1,
Eq.(10)-(11) dtype table); both round to nearest with ties to the even mantissa."""
from __future__ import annotations

import numpy as np

import synth


def test_tf32_rounding_hand_worked():
    u = 2.0 ** -10                               # one tf32 ulp at 1.0
    cases = [
        (1.0 + u / 2, 1.0),                      # tie, 1.0 has the even mantissa
        (1.0 + 3 * u / 2, 1.0 + 2 * u),          # tie, rounds up to the even mantissa
        (1.0 + u / 2 + 2.0 ** -20, 1.0 + u),     # just above the tie
        (1.0 + u / 2 - 2.0 ** -20, 1.0),         # just below the tie
        (-(1.0 + 3 * u / 2), -(1.0 + 2 * u)),    # sign symmetric
        (2.0 - u / 4, 2.0),                      # rounds into the next binade
        (0.0, 0.0),
    ]
    got = synth.f32_to_tf32(np.array([c[0] for c in cases], dtype=np.float32))
    np.testing.assert_array_equal(got, np.array([c[1] for c in cases], dtype=np.float32))
    r = synth.f32_to_tf32(np.random.default_rng(0).normal(size=1000).astype(np.float32))
    assert ((r.view(np.uint32) & np.uint32(0x1FFF)) == 0).all()
    assert np.isinf(synth.f32_to_tf32(np.array([np.inf], dtype=np.float32)))[0]


def test_bf16_rounding_hand_worked():
    u = 2.0 ** -7
    x = np.array([1.0 + u / 2, 1.0 + 3 * u / 2, 1.0 + u / 2 + 2.0 ** -20], dtype=np.float32)
    want = np.array([1.0, 1.0 + 2 * u, 1.0 + u], dtype=np.float32)
    got = (synth.f32_to_bf16_bits(x).astype(np.uint32) << 16).view(np.float32)
    np.testing.assert_array_equal(got, want)


def test_tf32_phi_is_the_same_draw_rounded():
    a = synth.mhc_inputs(8, 2, 64, "bf16", seed=3, phi_dtype="tf32")
    b = synth.mhc_inputs(8, 2, 64, "f32", seed=3)
    np.testing.assert_array_equal(a["phi"], synth.f32_to_tf32(b["phi"]))
    c = synth.mhc_inputs(8, 2, 64, "bf16", seed=3)
    np.testing.assert_array_equal(a["X"], c["X"])
