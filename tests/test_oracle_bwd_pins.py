"""Pins of the backward oracle (oracle.bwd) to things other than itself.

The adjoint is checked against central finite differences of the forward
oracle, which is itself pinned by closed forms and invariants
(test_oracle_pins.py).  J = Σ dy·y + Σ dlast·last_state is smooth in every
input (softplus, exp and the sigmoid gate), so in fp64 a central difference
with step 1e-6 agrees with the exact derivative to ~1e-9 relative; the bound
used is 1e-6.  Planted mistakes in the adjoint must break that agreement.
"""
import numpy as np
import pytest

import oracle

FD_EPS = 1e-6
FD_TOL = 1e-6


def problem(seed, b=2, L=6, d=3, N=4, gate=True, with_D=True, with_bias=True, dlast=True,
            delta_scale=0.5):
    rng = np.random.default_rng(seed)
    p = {
        "u": rng.normal(size=(b, L, d)),
        "delta": rng.normal(size=(b, L, d)) * delta_scale,
        "A": -np.tile(np.arange(1, N + 1, dtype=np.float64), (d, 1)) * rng.uniform(0.5, 1.5, size=(d, 1)),
        "B": rng.normal(size=(b, L, N)),
        "C": rng.normal(size=(b, L, N)),
        "D": rng.normal(size=d) if with_D else None,
        "z": rng.normal(size=(b, L, d)) if gate else None,
        "delta_bias": rng.normal(size=d) * 0.3 if with_bias else None,
    }
    dy = rng.normal(size=(b, L, d))
    dl = rng.normal(size=(b, d, N)) if dlast else None
    return p, dy, dl


def objective(p, dy, dl, softplus):
    y, st = oracle.fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                       delta_bias=p["delta_bias"], softplus=softplus)
    j = float((y * dy).sum())
    if dl is not None:
        j += float((st * dl).sum())
    return j


GRAD_OF = {"u": "du", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC", "D": "dD",
           "z": "dz", "delta_bias": "dbias"}


def fd_gradient(p, dy, dl, softplus, name):
    base = p[name]
    out = np.zeros_like(base)
    for idx in np.ndindex(base.shape):
        q = dict(p)
        plus = base.copy()
        plus[idx] += FD_EPS
        minus = base.copy()
        minus[idx] -= FD_EPS
        q[name] = plus
        jp = objective(q, dy, dl, softplus)
        q[name] = minus
        jm = objective(q, dy, dl, softplus)
        out[idx] = (jp - jm) / (2 * FD_EPS)
    return out


def bwd_of(p, dy, dl, softplus):
    return oracle.bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"], z=p["z"],
                      delta_bias=p["delta_bias"], dlast=dl, softplus=softplus)


def worst_rel(p, dy, dl, softplus):
    g = bwd_of(p, dy, dl, softplus)
    worst = 0.0
    for name, key in GRAD_OF.items():
        if p[name] is None:
            assert key not in g
            continue
        fd = fd_gradient(p, dy, dl, softplus, name)
        scale = max(np.max(np.abs(fd)), 1e-12)
        worst = max(worst, float(np.max(np.abs(fd - g[key])) / scale))
    return worst


@pytest.mark.parametrize("case", [
    dict(),
    dict(gate=False),
    dict(with_D=False, with_bias=False),
    dict(dlast=False),
    dict(b=1, L=9, d=2, N=16),
], ids=["full", "no_gate", "no_D_no_bias", "no_dlast", "N16"])
def test_adjoint_matches_finite_differences(case):
    p, dy, dl = problem(11, **case)
    assert worst_rel(p, dy, dl, True) <= FD_TOL


def test_adjoint_without_softplus():
    p, dy, dl = problem(12)
    p["delta"] = np.abs(p["delta"]) * 0.2 + 0.05        # Δ used as given, kept positive
    p["delta_bias"] = np.abs(p["delta_bias"]) * 0.1
    assert worst_rel(p, dy, dl, False) <= FD_TOL


def test_adjoint_on_softplus_branches():
    """Δ_raw far below zero (tiny Δ) and above the identity threshold."""
    p, dy, dl = problem(13, L=5)
    p["delta"][0, :2, :] = -30.0
    p["delta"][1, 2:4, :] = 25.0
    assert worst_rel(p, dy, dl, True) <= FD_TOL


@pytest.mark.parametrize("mutation", [10, 11, 12])
def test_planted_adjoint_mistakes_are_caught(mutation):
    p, dy, dl = problem(14)
    oracle.set_mutation(mutation)
    try:
        bad = worst_rel(p, dy, dl, True)
    finally:
        oracle.set_mutation(0)
    assert bad > 1e-3, f"mutation {mutation} not caught ({bad:.3g})"


def test_gradients_are_linear_in_upstream():
    p, dy1, dl1 = problem(15)
    _, dy2, dl2 = problem(16)
    g1 = bwd_of(p, dy1, dl1, True)
    g2 = bwd_of(p, dy2, dl2, True)
    g12 = bwd_of(p, 2.0 * dy1 - 0.5 * dy2, 2.0 * dl1 - 0.5 * dl2, True)
    for k in g1:
        np.testing.assert_allclose(g12[k], 2.0 * g1[k] - 0.5 * g2[k], rtol=1e-12, atol=1e-12)


def test_shared_gradients_sum_over_channels_and_batch():
    """dB, dC sum per-channel contributions; dA, dD, dbias sum per-batch ones."""
    p, dy, dl = problem(17, b=2, d=3)
    full = bwd_of(p, dy, dl, True)
    d = p["u"].shape[2]
    acc_B = np.zeros_like(full["dB"])
    acc_C = np.zeros_like(full["dC"])
    for ch in range(d):
        q = {k: v for k, v in p.items()}
        for k in ("u", "delta", "z"):
            q[k] = p[k][:, :, ch:ch + 1]
        q["A"] = p["A"][ch:ch + 1]
        q["D"] = p["D"][ch:ch + 1]
        q["delta_bias"] = p["delta_bias"][ch:ch + 1]
        g = bwd_of(q, dy[:, :, ch:ch + 1], dl[:, ch:ch + 1], True)
        acc_B += g["dB"]
        acc_C += g["dC"]
        np.testing.assert_allclose(g["dA"][0], full["dA"][ch], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(g["du"][:, :, 0], full["du"][:, :, ch], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(acc_B, full["dB"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(acc_C, full["dC"], rtol=1e-12, atol=1e-13)
    per_b = [bwd_of({**p, **{k: p[k][i:i + 1] for k in ("u", "delta", "z", "B", "C")}},
                    dy[i:i + 1], dl[i:i + 1], True) for i in range(2)]
    for k in ("dA", "dD", "dbias"):
        np.testing.assert_allclose(per_b[0][k] + per_b[1][k], full[k], rtol=1e-12, atol=1e-13)
