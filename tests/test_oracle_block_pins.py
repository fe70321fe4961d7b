"""Pins of the Mamba block oracle (oracle.block.block_fwd) that do not
restate its composition.

- A worked example derived on paper (tests/golden/block_hand_example.txt):
  L = 2, d_model = d_inner = 2, d_state = 1, every value exact in ln 2 and
  ln 3.  It fixes which projection feeds x, z, Δ, B and C, the conv's tap
  orientation, where dt_bias enters, the D skip, the gate's input and the
  output projection's orientation.
- The gate pin: with W_inz = 0 every gate z σ(z) is 0, so the output is 0
  for any hidden state and any other weights (the README's block multiplies
  the scan output by silu(z) before out_proj).
- The L = 1 reduction: with identity in_proj_x, a current-tap-only conv and
  no Δ projection, one token reduces the scan to its closed form
  y = (Δ u Σ_n C_n B_n + D u) silu(z) ("Understanding Mamba and Selective
  State Space Models (SSMs)" §2.2 first cut from h = 0, §3.1 readout).
Planted mistakes (oracle.block.set_mutation, test-only) are each caught.
"""
import math
import os

import numpy as np
import pytest

from oracle import block as ob

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "block_hand_example.txt")


def load_golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split("=", 1)
            vals[k.strip()] = np.array([eval(e, {"__builtins__": {}}, {"log": math.log})
                                        for e in v.split(";")], dtype=np.float64)
    return vals


def golden_case():
    g = load_golden()
    w = {
        "in_proj_x": g["in_proj_x"].reshape(2, 2), "in_proj_z": g["in_proj_z"].reshape(2, 2),
        "conv_w": g["conv_w"].reshape(2, 4), "conv_b": g["conv_b"],
        "x_proj_dt": g["x_proj_dt"].reshape(1, 2), "dt_proj": g["dt_proj"].reshape(2, 1),
        "dt_bias": g["dt_bias"], "x_proj_B": g["x_proj_B"].reshape(1, 2),
        "x_proj_C": g["x_proj_C"].reshape(1, 2), "A": g["A"].reshape(2, 1), "D": g["D"],
        "out_proj": g["out_proj"].reshape(2, 2),
    }
    return g["hidden"].reshape(1, 2, 2), w, g["out"].reshape(1, 2, 2)


def rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def pin_golden():
    h, w, ref = golden_case()
    e = rel(ob.block_fwd(h, w, store_bf16=False), ref)
    return e <= 1e-12, e


def random_weights(rng, d_model=6, d_inner=10, N=16, rank=2):
    return {
        "in_proj_x": rng.normal(size=(d_inner, d_model)) * 0.4,
        "in_proj_z": rng.normal(size=(d_inner, d_model)) * 0.4,
        "conv_w": rng.normal(size=(d_inner, 4)) * 0.7,
        "conv_b": rng.normal(size=d_inner) * 0.2,
        "x_proj_dt": rng.normal(size=(rank, d_inner)) * 0.3,
        "x_proj_B": rng.normal(size=(N, d_inner)) * 0.3,
        "x_proj_C": rng.normal(size=(N, d_inner)) * 0.3,
        "dt_proj": rng.normal(size=(d_inner, rank)) * 0.3,
        "dt_bias": rng.normal(size=d_inner) * 0.3 - 1.0,
        "A": -np.tile(np.arange(1, N + 1, dtype=np.float64), (d_inner, 1)),
        "D": rng.normal(size=d_inner),
        "out_proj": rng.normal(size=(d_model, d_inner)) * 0.3,
    }


def pin_zero_gate():
    rng = np.random.default_rng(11)
    w = random_weights(rng)
    w["in_proj_z"] = np.zeros_like(w["in_proj_z"])
    out = ob.block_fwd(rng.normal(size=(2, 7, 6)), w, store_bf16=False)
    m = float(np.max(np.abs(out)))
    return m == 0.0, m


def silu(v):
    return v / (1.0 + np.exp(-v))


def pin_single_token():
    rng = np.random.default_rng(12)
    d, N = 5, 16
    w = random_weights(rng, d_model=d, d_inner=d, N=N)
    w["in_proj_x"] = np.eye(d)
    w["conv_w"] = np.zeros((d, 4))
    w["conv_w"][:, 3] = 1.0
    w["conv_b"] = np.zeros(d)
    w["x_proj_dt"] = np.zeros_like(w["x_proj_dt"])
    w["A"] = -np.exp(rng.normal(size=(d, N)) * 0.5)
    h = rng.normal(size=(1, 1, d))
    u = silu(h[0, 0])                                  # current tap only, x = h
    z = w["in_proj_z"] @ h[0, 0]
    Bv = w["x_proj_B"] @ u
    Cv = w["x_proj_C"] @ u
    delta = np.log1p(np.exp(w["dt_bias"]))             # Δraw = 0: Δ = softplus(dt_bias)
    y = (delta * u * float(Cv @ Bv) + w["D"] * u) * silu(z)
    e = rel(ob.block_fwd(h, w, store_bf16=False)[0, 0], w["out_proj"] @ y)
    return e <= 1e-12, e


PINS = [pin_golden, pin_zero_gate, pin_single_token]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_block_pin(pin):
    ok, detail = pin()
    assert ok, detail


@pytest.mark.parametrize("mutation", ob.MUTATIONS)
def test_planted_block_mistake_is_caught(mutation):
    def holds(pin):
        try:
            return pin()[0]
        except ValueError:   # a shape mismatch fails as loudly as a wrong value
            return False

    ob.set_mutation(mutation)
    try:
        caught = [p.__name__ for p in PINS if not holds(p)]
    finally:
        ob.set_mutation(None)
    assert caught, f"no pin catches {mutation}"
