"""Pins of the CPU oracle against facts the pages and the mathematics fix.

Each pin returns (ok, detail).  The pins are written from the equations of
"Understanding Mamba and Selective State Space Models (SSMs)" (§2.1 classic
SSM and its convolutional form, §2.2 first/second cut, §3.1 readout, §4.3
negative diagonal A) and from properties any correct implementation has.
None of them re-runs the oracle's own loop: they use a closed form, a library
convolution, a worked example derived by hand, or an invariant that relates
two different oracle calls.
"""
import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _silu(z):
    return z / (1.0 + np.exp(-z))


def _softplus(x):
    return np.where(x > 20.0, x, np.log1p(np.exp(np.minimum(x, 20.0))))


def _rand_inputs(rng, batch, L, d, N, gate=True, structured=False):
    u = rng.standard_normal((batch, L, d))
    delta = 0.5 * rng.standard_normal((batch, L, d))
    z = rng.standard_normal((batch, L, d)) if gate else None
    B = rng.standard_normal((batch, L, N))
    C = rng.standard_normal((batch, L, N))
    if structured:
        A = -np.tile(np.arange(1, N + 1, dtype=np.float64), (d, 1))
    else:
        A = -np.exp(rng.standard_normal((d, N)) * 0.7)
    D = rng.standard_normal(d)
    bias = np.log(np.expm1(np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), d))))
    return dict(u=u, delta=delta, z=z, B=B, C=C, A=A, D=D, delta_bias=bias)


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / den) if a.size else 0.0


# ----------------------------------------------------------------------------
def load_hand_example():
    vals = {}
    with open(os.path.join(GOLDEN, "hand_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split("=", 1)
            vals[k.strip()] = [eval(e, {"__builtins__": {}}, {"log": math.log})
                               for e in v.split(";")]
    return vals


def pin_hand_example():
    """Worked example derived on paper (tests/golden/hand_example.txt)."""
    g = load_hand_example()
    L, N = 3, 2
    A = np.array(g["A"]).reshape(1, N)
    D = np.array(g["D"])
    bias = np.array(g["bias"])
    u = np.array(g["u"]).reshape(1, L, 1)
    dr = np.array(g["delta_raw"]).reshape(1, L, 1)
    B = np.array(g["B"]).reshape(1, L, N)
    C = np.array(g["C"]).reshape(1, L, N)
    z = np.array(g["z"]).reshape(1, L, 1)
    errs = []
    for prec, tol in (("f64", 1e-15), ("f32", 2e-7)):
        y, st = oracle.fwd(u, dr, A, B, C, D=D, z=None, delta_bias=bias, precision=prec)
        errs.append(_rel(y.ravel(), g["y_nogate"]) / tol)
        errs.append(_rel(st.ravel(), g["last_state"]) / tol)
        yg, _ = oracle.fwd(u, dr, A, B, C, D=D, z=z, delta_bias=bias, precision=prec)
        errs.append(_rel(yg.ravel(), g["y_gate"]) / tol)
        s1, y1 = oracle.step(np.array(g["step_state_in"]).reshape(1, 1, N), u[:, 0, :],
                             dr[:, 0, :], A, B[:, 0, :], C[:, 0, :], D=D, z=None,
                             delta_bias=bias, precision=prec)
        errs.append(_rel(s1.ravel(), g["step_state_out"]) / tol)
        errs.append(_rel(y1.ravel(), g["step_y_nogate"]) / tol)
    worst = max(errs)
    return worst <= 1.0, f"worst error / tolerance = {worst:.3g}"


def pin_closed_form_L1(seed=11):
    """L = 1 from a zero state: h = Δ B u, y = (Δ u Σ_n C_n B_n + D u)·silu(z)."""
    rng = np.random.default_rng(seed)
    x = _rand_inputs(rng, 3, 1, 7, 5)
    dt = _softplus(x["delta"] + x["delta_bias"][None, None, :])          # [b,1,d]
    cb = np.sum(x["C"] * x["B"], axis=-1)[:, :, None]                     # [b,1,1]
    y_ref = (dt * x["u"] * cb + x["D"][None, None, :] * x["u"]) * _silu(x["z"])
    st_ref = dt[:, 0, :, None] * x["B"][:, 0, None, :] * x["u"][:, 0, :, None]
    worst = 0.0
    for prec, tol in (("f64", 1e-13), ("f32", 5e-6)):
        y, st = oracle.fwd(**x, precision=prec)
        worst = max(worst, _rel(y, y_ref) / tol, _rel(st, st_ref) / tol)
    return worst <= 1.0, f"worst error / tolerance = {worst:.3g}"


def pin_lti_convolution(seed=12, L=48, d=6, N=5):
    """§2.1: with Δ, B, C fixed over time the SSM is time invariant and equals a
    causal convolution y = K * u + D u with K_k = Σ_n C_n exp(Δ A_n)^k Δ B_n.
    Checked against numpy.convolve with K built from powers."""
    rng = np.random.default_rng(seed)
    batch = 2
    x = _rand_inputs(rng, batch, L, d, N, gate=False)
    x["delta"] = np.repeat(x["delta"][:, :1, :], L, axis=1)
    x["B"] = np.repeat(x["B"][:, :1, :], L, axis=1)
    x["C"] = np.repeat(x["C"][:, :1, :], L, axis=1)
    y, _ = oracle.fwd(**x, precision="f64")
    y_ref = np.empty_like(y)
    k = np.arange(L, dtype=np.float64)
    for b in range(batch):
        for ch in range(d):
            dt = float(_softplus(x["delta"][b, 0, ch] + x["delta_bias"][ch]))
            Ab = np.exp(dt * x["A"][ch])                                   # [N]
            K = np.sum(x["C"][b, 0][:, None] * np.power(Ab[:, None], k[None, :])
                       * dt * x["B"][b, 0][:, None], axis=0)               # [L]
            y_ref[b, :, ch] = np.convolve(x["u"][b, :, ch], K)[:L] + x["D"][ch] * x["u"][b, :, ch]
    err = _rel(y, y_ref)
    return err <= 1e-12, f"relative error {err:.3g}"


def pin_linearity(seed=13):
    """With Δ, B, C, z fixed, y and the final state are linear in u."""
    rng = np.random.default_rng(seed)
    x = _rand_inputs(rng, 2, 40, 5, 4)
    u1 = x.pop("u")
    u2 = rng.standard_normal(u1.shape)
    a, b = 0.7, -1.9
    y1, s1 = oracle.fwd(u=u1, **x)
    y2, s2 = oracle.fwd(u=u2, **x)
    y3, s3 = oracle.fwd(u=a * u1 + b * u2, **x)
    err = max(_rel(y3, a * y1 + b * y2), _rel(s3, a * s1 + b * s2))
    return err <= 1e-12, f"relative error {err:.3g}"


def pin_chunked_equals_sequential(seed=14, L=37):
    """Re-associating time into chunks with the (P, h) combine gives the same
    outputs as the sequential loop, for every chunk length."""
    rng = np.random.default_rng(seed)
    x = _rand_inputs(rng, 2, L, 4, 6)
    y, s = oracle.fwd(**x)
    worst = 0.0
    for chunk in (1, 2, 3, 7, 16, L, L + 5):
        yc, sc = oracle.fwd_chunked(**x, chunk=chunk)
        worst = max(worst, _rel(yc, y), _rel(sc, s))
    return worst <= 1e-12, f"worst relative error {worst:.3g}"


def pin_causality(seed=15, L=30, tp=17):
    """Changing u at time t' leaves every y_t with t < t' unchanged (bitwise)."""
    rng = np.random.default_rng(seed)
    x = _rand_inputs(rng, 1, L, 3, 4)
    y, _ = oracle.fwd(**x)
    x["u"] = x["u"].copy()
    x["u"][:, tp, :] += 3.0
    y2, _ = oracle.fwd(**x)
    ok = np.array_equal(y[:, :tp], y2[:, :tp]) and not np.array_equal(y[:, tp], y2[:, tp])
    return ok, "prefix unchanged and y_t' changed" if ok else "causality violated"


def pin_channel_batch_independence(seed=16):
    """Permuting channels (with their A, D, bias rows) permutes the outputs;
    each batch entry computed alone equals the batched result."""
    rng = np.random.default_rng(seed)
    x = _rand_inputs(rng, 3, 20, 6, 4)
    y, s = oracle.fwd(**x)
    perm = rng.permutation(6)
    xp = dict(x)
    for k in ("u", "delta", "z"):
        xp[k] = x[k][:, :, perm]
    xp["A"] = x["A"][perm]
    xp["D"] = x["D"][perm]
    xp["delta_bias"] = x["delta_bias"][perm]
    yp, sp = oracle.fwd(**xp)
    err = max(_rel(yp, y[:, :, perm]), _rel(sp, s[:, perm]))
    for b in range(3):
        xb = {k: (v[b:b + 1] if (v is not None and k in ("u", "delta", "z", "B", "C")) else v)
              for k, v in x.items()}
        yb, sb = oracle.fwd(**xb)
        err = max(err, _rel(yb, y[b:b + 1]), _rel(sb, s[b:b + 1]))
    return err <= 1e-15, f"relative error {err:.3g}"


def pin_delta_to_zero(seed=17):
    """Δ -> 0+ (Δ_raw = -40, no bias): the state stays ~0 and y = D u silu(z)."""
    rng = np.random.default_rng(seed)
    x = _rand_inputs(rng, 2, 25, 4, 4)
    x["delta"] = np.full_like(x["delta"], -40.0)
    x["delta_bias"] = None
    y, s = oracle.fwd(**x)
    y_ref = x["D"][None, None, :] * x["u"] * _silu(x["z"])
    err = _rel(y, y_ref)
    return err <= 1e-14 and np.max(np.abs(s)) < 1e-14, f"relative error {err:.3g}"


def pin_A_to_minus_infinity(seed=18):
    """A -> -inf: the decay vanishes, so every step restarts from zero:
    y_t = (Δ_t u_t Σ_n C_t,n B_t,n + D u_t)·silu(z_t)."""
    rng = np.random.default_rng(seed)
    x = _rand_inputs(rng, 2, 25, 4, 4)
    x["A"] = np.full_like(x["A"], -1e30)
    y, _ = oracle.fwd(**x)
    dt = _softplus(x["delta"] + x["delta_bias"][None, None, :])
    cb = np.sum(x["C"] * x["B"], axis=-1)[:, :, None]
    y_ref = (dt * x["u"] * cb + x["D"][None, None, :] * x["u"]) * _silu(x["z"])
    err = _rel(y, y_ref)
    return err <= 1e-13, f"relative error {err:.3g}"


def pin_decode_equivalence(seed=19, L=23):
    """L single-token steps from a zero state reproduce the forward scan:
    the same y at every step and the same final state (exact, both precisions)."""
    rng = np.random.default_rng(seed)
    x = _rand_inputs(rng, 2, L, 5, 4)
    ok = True
    for prec in ("f64", "f32"):
        y, s = oracle.fwd(**x, precision=prec)
        st = np.zeros_like(s)
        ys = np.empty_like(y)
        for t in range(L):
            st, ys[:, t, :] = oracle.step(st, x["u"][:, t], x["delta"][:, t], x["A"],
                                          x["B"][:, t], x["C"][:, t], D=x["D"],
                                          z=x["z"][:, t], delta_bias=x["delta_bias"],
                                          precision=prec)
        ok = ok and np.array_equal(ys, y) and np.array_equal(st, s)
    return ok, "bitwise equal" if ok else "step loop differs from the scan"


def pin_B_scaling(seed=20, s_=-2.5):
    """Scaling B by s scales the state, and the non-skip part of y, by s."""
    rng = np.random.default_rng(seed)
    x = _rand_inputs(rng, 2, 30, 4, 4)
    y1, s1 = oracle.fwd(**x)
    x2 = dict(x)
    x2["B"] = s_ * x["B"]
    y2, s2 = oracle.fwd(**x2)
    g = _silu(x["z"])
    skip = x["D"][None, None, :] * x["u"]
    err = max(_rel(y2 / g - skip, s_ * (y1 / g - skip)), _rel(s2, s_ * s1))
    return err <= 1e-10, f"relative error {err:.3g}"


ALL_PINS = [pin_hand_example, pin_closed_form_L1, pin_lti_convolution, pin_linearity,
            pin_chunked_equals_sequential, pin_causality, pin_channel_batch_independence,
            pin_delta_to_zero, pin_A_to_minus_infinity, pin_decode_equivalence,
            pin_B_scaling]
