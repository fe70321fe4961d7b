"""Pins of the multi-head scalar-decay scan oracle (oracle.ssd).

1. It is the Mamba-1 selective scan (independently pinned in
   test_oracle_pins.py) with every channel of a head sharing the head's Δ and
   a decay constant over the state index: oracle.fwd on H·P channels with
   A[ch, n] = A_h, Δraw[ch] = dt_h, bias[ch] = dt_bias_h, D[ch] = D_h.
2. A chunked matrix form -- within a chunk y = (L ∘ C Bᵀ) (Δ x) with
   L[t, s] = exp(Σ_{s<r<=t} Δ_r A) for s <= t, states passed between chunks
   as H_end = exp(ΣΔA) H_start + Σ_s exp(Σ_{s<r} Δ_r A) Δ_s x_s B_sᵀ -- written
   here in numpy, equals the recurrence for several chunk lengths.
3. Closed forms: one step, and a decay of zero (A -> -inf).
"""
import numpy as np
import pytest

import oracle


def problem(seed, b=2, L=11, H=3, P=4, N=5):
    rng = np.random.default_rng(seed)
    return dict(x=rng.normal(size=(b, L, H, P)), dt=rng.normal(size=(b, L, H)) * 0.5,
                A=-rng.uniform(0.5, 2.0, size=H), B=rng.normal(size=(b, L, N)), C=rng.normal(size=(b, L, N)),
                D=rng.normal(size=H), dt_bias=rng.normal(size=H) * 0.3)


def softplus(v):
    return np.where(v > 20, v, np.log1p(np.exp(np.minimum(v, 20))))


def test_equals_mamba1_scan_with_shared_delta_and_scalar_decay():
    p = problem(1)
    b, L, H, P = p["x"].shape
    N = p["B"].shape[-1]
    y, st = oracle.ssd(p["x"], p["dt"], p["A"], p["B"], p["C"], D=p["D"], dt_bias=p["dt_bias"])
    u = p["x"].reshape(b, L, H * P)
    delta = np.repeat(p["dt"], P, axis=2)
    A1 = np.repeat(p["A"], P)[:, None] * np.ones((1, N))
    y1, st1 = oracle.fwd(u, delta, A1, p["B"], p["C"], D=np.repeat(p["D"], P),
                         delta_bias=np.repeat(p["dt_bias"], P))
    np.testing.assert_allclose(y.reshape(b, L, H * P), y1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(st.reshape(b, H * P, N), st1, rtol=1e-12, atol=1e-12)


def chunked(p, Q):
    """The chunked matrix form in float64 (no D term)."""
    x, B, C = p["x"], p["B"], p["C"]
    b, L, H, P = x.shape
    N = B.shape[-1]
    delta = softplus(p["dt"] + p["dt_bias"])          # [b, L, H]
    y = np.zeros_like(x)
    state = np.zeros((b, H, P, N))
    for c0 in range(0, L, Q):
        c1 = min(L, c0 + Q)
        a = delta[:, c0:c1] * p["A"]                    # [b, q, H] log-decays
        cum = np.cumsum(a, axis=1)
        S = np.einsum("btn,bsn->bts", C[:, c0:c1], B[:, c0:c1])
        q = c1 - c0
        mask = np.tril(np.ones((q, q)))
        Lm = np.exp(np.clip(cum[:, :, None, :] - cum[:, None, :, :], None, 0.0)) * mask[None, :, :, None]
        xd = delta[:, c0:c1, :, None] * x[:, c0:c1]     # Δ x  [b, q, H, P]
        y[:, c0:c1] = np.einsum("bts,btsh,bshp->bthp", S, Lm, xd)
        y[:, c0:c1] += np.exp(cum)[..., None] * np.einsum("btn,bhpn->bthp", C[:, c0:c1], state)
        w = np.exp(cum[:, -1:, :] - cum)                # decay from s to the chunk end
        state = np.exp(cum[:, -1])[:, :, None, None] * state + np.einsum("bsh,bshp,bsn->bhpn", w, xd, B[:, c0:c1])
    return y, state


@pytest.mark.parametrize("Q", [1, 3, 8, 11])
def test_chunked_matrix_form_equals_recurrence(Q):
    p = problem(2)
    y, st = oracle.ssd(p["x"], p["dt"], p["A"], p["B"], p["C"], dt_bias=p["dt_bias"])
    yc, stc = chunked(p, Q)
    np.testing.assert_allclose(yc, y, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(stc, st, rtol=1e-11, atol=1e-12)


def test_single_step_closed_form():
    p = problem(3, L=1)
    y, st = oracle.ssd(p["x"], p["dt"], p["A"], p["B"], p["C"], D=p["D"], dt_bias=p["dt_bias"])
    delta = softplus(p["dt"] + p["dt_bias"])[:, 0]     # [b, H]
    bc = np.einsum("bn,bn->b", p["B"][:, 0], p["C"][:, 0])
    ref = (delta * bc[:, None])[..., None] * p["x"][:, 0] + p["D"][None, :, None] * p["x"][:, 0]
    np.testing.assert_allclose(y[:, 0], ref, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(st, delta[:, :, None, None] * p["x"][:, 0, :, :, None] * p["B"][:, 0, None, None, :],
                               rtol=1e-13, atol=1e-13)


def test_zero_decay_forgets_the_past():
    p = problem(4)
    p["A"] = np.full_like(p["A"], -1e6)
    y, _ = oracle.ssd(p["x"], p["dt"], p["A"], p["B"], p["C"], dt_bias=p["dt_bias"])
    delta = softplus(p["dt"] + p["dt_bias"])
    bc = np.einsum("btn,btn->bt", p["B"], p["C"])
    np.testing.assert_allclose(y, (delta * bc[..., None])[..., None] * p["x"], rtol=1e-12, atol=1e-12)
