"""The CPU oracle, pinned to facts outside itself (runs without a GPU)."""
import numpy as np
import pytest

import oracle
from selective_ssm_scan_mamba_b200 import inputs as I
from tests import oracle_pins as P


@pytest.mark.parametrize("check", P.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(check):
    ok, detail = check(0)
    assert ok, detail


@pytest.mark.parametrize("mutant", range(1, 13))
def test_planted_mistake_is_caught(mutant):
    """Each planted mistake in the oracle must fail at least one pin."""
    assert oracle.load(mutant).oracle_mutant_id() == mutant
    failed = []
    for check in P.ALL_CHECKS:
        try:
            ok, _ = check(mutant)
        except Exception:  # a mutant may also break an argument contract
            ok = False
        if not ok:
            failed.append(check.__name__)
    assert failed, f"mutant {mutant} passed every pin"


def test_block_step_leaves_cache_untouched():
    s = P._small(19, 2, 8, 3, 4)
    h = I.make_state(5, 2, 3, 4)
    h_copy = h.copy()
    oracle.block_step(s["x"], s["dt"], s["A"], s["B"], s["C"], s["Dskip"], h)
    assert np.array_equal(h, h_copy)


def test_bf16_decode_is_exact():
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x8000, 0x3F81, 0x7F7F], np.uint16)
    want = np.array([1.0, -2.0, 0.0, -0.0, 1.0 + 2 ** -7, 3.3895313892515355e38])
    assert np.array_equal(oracle.decode(bits), want)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -9, 1.0 + 2 ** -8 + 2 ** -20], np.float32)
    want = np.array([1.0, 1.0 + 2 ** -6, -1.0, 1.0 + 2 ** -7])
    assert np.array_equal(oracle.decode(I.f32_to_bf16_bits(x)), want)


def test_inputs_are_reproducible_by_slice():
    full = I.make_sequence(3, 2, 5200, 16, 4, "bf16", stream=("context",))
    part = I.make_sequence(3, 2, 1200, 16, 4, "bf16", stream=("context",), t0=3900, channels=[1, 7])
    assert np.array_equal(full["x"][:, 3900:5100, [1, 7]], part["x"])
    assert np.array_equal(full["B"][:, 3900:5100], part["B"])
    other = I.make_sequence(3, 2, 100, 16, 4, "bf16", stream=("noisy", 0, 1))
    assert not np.array_equal(other["x"], full["x"][:, :100])


def test_input_distributions():
    s = I.make_sequence(1, 1, 8192, 64, 16, "f32")
    p = I.make_params(1, 64, 16)
    assert abs(s["x"].mean()) < 0.02 and abs(s["x"].std() - 1) < 0.02
    assert abs(s["dt"].mean() + 2) < 0.02 and abs(s["dt"].std() - 0.5) < 0.02
    assert abs(s["B"].std() - 0.25) < 0.01
    assert p["A"].max() <= -1.0 and p["A"].min() >= -16.0
