"""Oracle of the Mamba block's inner forward path -- TEST INFRASTRUCTURE ONLY.

Composes plain steps, in order, in float64 (numpy matmul as the library
primitive for the projections; the pinned conv and scan oracles for the rest):

  x = hidden · W_inxᵀ,  z = hidden · W_inzᵀ          (in_proj, no bias)
  u = silu(conv_b + causal_conv4(x))                 (deep-dive §3.3)
  dt_low = u · W_dtlowᵀ,  B = u · W_Bᵀ,  C = u · W_Cᵀ (the selection projections:
                                                      Δ, B, C as functions of the token)
  Δraw = dt_low · W_dtᵀ                               (Δ's low-rank projection; its bias
                                                      dt_bias enters the softplus --
                                                      README "Initialization")
  y = scan(u, Δraw, A, B, C, D, z, dt_bias)          (the selective scan, softplus on)
  out = y · W_outᵀ                                    (out_proj, no bias)

The pages give the block's interface (d_model, d_state = 16, d_conv = 4,
expand = 2, out.shape == hidden.shape, "roughly 3 · expand · d_model^2
parameters" -- the README's Usage > Mamba) and that Δ has a linear projection
with a bias (README, Initialization).  Where they are silent the readings
are: no biases on in_proj / x_proj / out_proj; Δ's projection is low rank,
dt_rank = ceil(d_model / 16), so that the block's parameters stay close to
3 · expand · d_model^2.

`store_bf16=True` rounds every intermediate the GPU layer stores in bf16 (x,
z, u, dt_low, B, C, Δraw, y, out) to bf16 (round to nearest even) at the same
points, so the comparison measures arithmetic differences only.
"""
import numpy as np

from . import conv_silu, fwd

# Test-only switch: plants one named mistake in block_fwd so that the tests
# can check that the pins catch it.  None (the default) runs the block as
# written above.
MUTATIONS = ("swap_xz", "gate_from_x", "conv_reversed", "dt_bias_ignored", "swap_BC", "no_D",
             "out_proj_T", "select_from_x", "no_softplus")
_mutation = None


def set_mutation(name):
    """Plant mistake `name` (one of MUTATIONS) in block_fwd; None clears it."""
    global _mutation
    if name is not None and name not in MUTATIONS:
        raise ValueError(name)
    _mutation = name


def round_bf16(a):
    """float64 -> nearest bf16 value (ties to even), returned as float64."""
    f = np.asarray(a, dtype=np.float64).astype(np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    out = rounded.astype(np.uint32).view(np.float32).astype(np.float64)
    nan = np.isnan(f)
    if nan.any():
        out[nan] = np.nan
    return out


def block_fwd(hidden, w, store_bf16=True, precision="f64"):
    """hidden [b, L, d_model]; w a dict of float arrays (names as in the layer
    weights: in_proj_x, in_proj_z [d_inner, d_model], conv_w [d_inner, 4],
    conv_b [d_inner], x_proj_dt [dt_rank, d_inner], x_proj_B, x_proj_C
    [d_state, d_inner], dt_proj [d_inner, dt_rank], dt_bias [d_inner], A
    [d_inner, d_state], D [d_inner], out_proj [d_model, d_inner]).  Returns
    out [b, L, d_model] in float64."""
    r = round_bf16 if store_bf16 else (lambda a: a)
    mut = _mutation
    h = np.asarray(hidden, dtype=np.float64)
    g = {k: (None if v is None else np.asarray(v, dtype=np.float64)) for k, v in w.items()}
    if mut == "swap_xz":
        g["in_proj_x"], g["in_proj_z"] = g["in_proj_z"], g["in_proj_x"]
    if mut == "conv_reversed":
        g["conv_w"] = g["conv_w"][:, ::-1]
    if mut == "swap_BC":
        g["x_proj_B"], g["x_proj_C"] = g["x_proj_C"], g["x_proj_B"]
    if mut == "out_proj_T":
        g["out_proj"] = g["out_proj"].T
    x = r(h @ g["in_proj_x"].T)
    z = r(h @ g["in_proj_z"].T)
    u = r(conv_silu(x, g["conv_w"], g["conv_b"]))
    src = x if mut == "select_from_x" else u
    dt_low = r(src @ g["x_proj_dt"].T)
    B = r(src @ g["x_proj_B"].T)
    C = r(src @ g["x_proj_C"].T)
    delta = r(dt_low @ g["dt_proj"].T)
    y, _ = fwd(u, delta, g["A"], B, C, D=None if mut == "no_D" else g["D"],
               z=x if mut == "gate_from_x" else z,
               delta_bias=None if mut == "dt_bias_ignored" else g["dt_bias"],
               softplus=mut != "no_softplus", precision=precision)
    y = r(y)
    return r(y @ g["out_proj"].T)
