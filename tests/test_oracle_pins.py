"""The CPU oracle, pinned to facts other than itself (runs without a GPU)."""
import numpy as np
import pytest

import oracle
from oracle_pins import ALL_PINS, _rand_inputs, _rel


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(pin):
    ok, detail = pin()
    assert ok, f"{pin.__name__}: {detail}"


MUTATIONS = {
    1: "decay sign flipped",
    2: "D skip dropped",
    3: "B and C swapped",
    4: "Δ bias ignored",
    5: "softplus skipped",
    6: "readout before update",
    7: "gate σ(z) instead of z·σ(z)",
    8: "Δ missing from input term",
    9: "A transposed",
}


@pytest.mark.parametrize("m", sorted(MUTATIONS), ids=[MUTATIONS[m] for m in sorted(MUTATIONS)])
def test_planted_mistake_is_caught(m):
    """Plant one deliberate mistake in the oracle; at least one pin must fail."""
    oracle.set_mutation(m)
    try:
        failed = [p.__name__ for p in ALL_PINS if not p()[0]]
    finally:
        oracle.set_mutation(0)
    assert oracle.get_mutation() == 0
    assert failed, f"mutation {m} ({MUTATIONS[m]}) passed every pin"


def test_f32_oracle_close_to_f64():
    """The fp32-state oracle stays within the fp32 parity bound of the fp64 one
    on a tiny-config-sized input (bounds the graded oracle's own error)."""
    rng = np.random.default_rng(5)
    x = _rand_inputs(rng, 1, 64, 32, 16, structured=True)
    y64, s64 = oracle.fwd(**x, precision="f64")
    y32, s32 = oracle.fwd(**x, precision="f32")
    assert _rel(y32, y64) < 1e-5
    assert _rel(s32, s64) < 1e-5


def test_softplus_identity_branch_is_continuous():
    """Δ_raw just below and above the identity threshold give outputs that
    differ only by the tiny change in Δ (no jump at the branch)."""
    rng = np.random.default_rng(6)
    x = _rand_inputs(rng, 1, 1, 3, 4)
    x["delta_bias"] = None
    x["delta"] = np.full_like(x["delta"], 20.0 - 1e-9)
    y1, _ = oracle.fwd(**x)
    x["delta"] = np.full_like(x["delta"], 20.0 + 1e-9)
    y2, _ = oracle.fwd(**x)
    assert _rel(y2, y1) < 1e-8


def test_rejects_bad_sizes():
    with pytest.raises(ValueError):
        oracle.fwd(np.zeros((1, 2, 3)), np.zeros((1, 2, 3)), np.zeros((3, 300)),
                   np.zeros((1, 2, 300)), np.zeros((1, 2, 300)))


def test_empty_sequence():
    y, s = oracle.fwd(np.zeros((2, 0, 3)), np.zeros((2, 0, 3)), -np.ones((3, 4)),
                      np.zeros((2, 0, 4)), np.zeros((2, 0, 4)))
    assert y.shape == (2, 0, 3)
    assert np.array_equal(s, np.zeros((2, 3, 4)))
