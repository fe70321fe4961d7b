"""GPU parity of ss_step (single-token decode) against the CPU oracle, and
decode/scan equivalence on the GPU, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_37_b200 as ss
from gpu_util import rel_max_err, tol_for
from ss_inputs import CONFIGS, fwd_inputs, sample_channels, step_inputs, step_sequence_inputs, to_f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def oracle_step(inp, state, precision):
    return oracle.step(state, to_f64(inp["u"]), to_f64(inp["delta"]), to_f64(inp["A"]),
                       to_f64(inp["B"]), to_f64(inp["C"]), D=to_f64(inp["D"]), z=to_f64(inp["z"]),
                       delta_bias=to_f64(inp["delta_bias"]), precision=precision)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("shape", [(3, 64), (2, 100), (5, 1000)])
@pytest.mark.parametrize("A_kind", ["structured", "general"])
def test_step_small(dtype, shape, A_kind):
    b, d = shape
    inp = step_inputs(b, d, 16, dtype, 10 + b + d, DEV, gate=(d != 100), A_kind=A_kind)
    st0 = to_f64(inp["state"])
    y = ss.ss_step(inp["state"], inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                   z=inp["z"], delta_bias=inp["delta_bias"], sync_check=True)
    tol = tol_for(inp["u"].dtype)
    for prec in ("f32", "f64"):
        sr, yr = oracle_step(inp, st0, prec)
        assert rel_max_err(to_f64(y), yr) <= tol
        assert rel_max_err(to_f64(inp["state"]), sr) <= tol


# Options and shapes of the bf16 step: one batch row, many rows, a few
# channels, d_inner not a multiple of the 64-channel block, gate / softplus /
# D / bias on and off.
OPTS = [(1, 8, True, True, True), (37, 4096, True, True, True), (300, 24, False, True, False), (512, 4096, True, True, True),
        (4, 136, True, False, True), (2, 2048, False, False, False)]


@pytest.mark.parametrize("b,d,gate,softplus,opts", OPTS,
                         ids=[f"b{b}_d{d}_g{int(g)}_sp{int(s)}_o{int(o)}" for b, d, g, s, o in OPTS])
def test_step_options(b, d, gate, softplus, opts):
    inp = step_inputs(b, d, 16, "bf16", 70 + b + d, DEV, gate=gate, bias=opts)
    if not opts:
        inp["D"] = None
    if not softplus:   # Δ is used as given: keep it positive (and without the negative bias)
        inp["delta"] = (inp["delta"].float().abs() * 0.1 + 0.01).to(torch.bfloat16)
        inp["delta_bias"] = None
    st0 = to_f64(inp["state"])
    y = ss.ss_step(inp["state"], inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                   z=inp["z"], delta_bias=inp["delta_bias"], softplus=softplus, sync_check=True)
    sr, yr = oracle.step(st0, to_f64(inp["u"]), to_f64(inp["delta"]), to_f64(inp["A"]), to_f64(inp["B"]),
                         to_f64(inp["C"]), D=to_f64(inp["D"]), z=to_f64(inp["z"]),
                         delta_bias=to_f64(inp["delta_bias"]), softplus=softplus, precision="f32")
    tol = tol_for(inp["u"].dtype)
    assert rel_max_err(to_f64(y), yr) <= tol
    assert rel_max_err(to_f64(inp["state"]), sr) <= tol


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_step_loop_equals_scan(dtype):
    """L decode steps from a zero state reproduce ss_fwd (y at every step and
    the final state), both on the GPU."""
    b, L, d = 2, 80, 192
    inp = fwd_inputs(b, L, d, 16, dtype, 21, DEV, gate=True, D_kind="normal")
    y_scan, s_scan = ss.ss_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                               z=inp["z"], delta_bias=inp["delta_bias"], chunk_len=32,
                               sync_check=True)
    state = torch.zeros(b, d, 16, device=DEV)
    ys = torch.empty_like(y_scan)
    for t in range(L):
        ys[:, t] = ss.ss_step(state, inp["u"][:, t].contiguous(), inp["delta"][:, t].contiguous(),
                              inp["A"], inp["B"][:, t].contiguous(), inp["C"][:, t].contiguous(),
                              D=inp["D"], z=inp["z"][:, t].contiguous(),
                              delta_bias=inp["delta_bias"])
    torch.cuda.synchronize()
    tol = tol_for(inp["u"].dtype)
    assert rel_max_err(to_f64(ys), to_f64(y_scan)) <= tol
    assert rel_max_err(to_f64(state), to_f64(s_scan)) <= tol


def test_config_decode_1000_steps():
    """The decode workload: batch 256, d_inner 5120, fp32 state ~ N(0,1),
    1000 successive steps with fresh bf16 inputs; sampled channels against the
    oracle stepping the same 1000 tokens."""
    c = CONFIGS["decode"]
    base = step_inputs(c.batch, c.d_inner, c.d_state, c.dtype, c.seed, DEV, gate=c.gate)
    seq = step_sequence_inputs(c.steps, c.batch, c.d_inner, c.d_state, c.dtype, c.seed + 1, DEV,
                               gate=c.gate)
    samples = sample_channels(c.batch, c.d_inner, 64, c.seed)
    bidx = sorted(set(b for b, _ in samples))
    state0 = base["state"].clone()
    y_hist = {}
    state = base["state"]
    for t in range(c.steps):
        y = ss.ss_step(state, seq["u"][t], seq["delta"][t], base["A"], seq["B"][t], seq["C"][t],
                       D=base["D"], z=seq["z"][t], delta_bias=base["delta_bias"])
        y_hist[t] = y[bidx].clone()
    torch.cuda.synchronize()
    # oracle on the sampled channels, grouped by batch entry
    for prec in ("f32", "f64"):
        errs_y, errs_s = [], []
        for b in bidx:
            chs = [ch for bb, ch in samples if bb == b]
            idx = torch.tensor(chs, device=DEV)
            st = to_f64(state0[b].index_select(0, idx))[None]
            A = to_f64(base["A"].index_select(0, idx))
            D = to_f64(base["D"].index_select(0, idx))
            bias = to_f64(base["delta_bias"].index_select(0, idx))
            u = to_f64(seq["u"][:, b].index_select(1, idx))
            dl = to_f64(seq["delta"][:, b].index_select(1, idx))
            z = to_f64(seq["z"][:, b].index_select(1, idx))
            Bm = to_f64(seq["B"][:, b])
            Cm = to_f64(seq["C"][:, b])
            ys_ref = np.empty((c.steps, len(chs)))
            for t in range(c.steps):
                st, yr = oracle.step(st, u[t][None], dl[t][None], A, Bm[t][None], Cm[t][None],
                                     D=D, z=z[t][None], delta_bias=bias, precision=prec)
                ys_ref[t] = yr[0]
            row = bidx.index(b)
            ys_gpu = np.stack([to_f64(y_hist[t][row].index_select(0, idx)) for t in range(c.steps)])
            errs_y.append((ys_gpu, ys_ref))
            errs_s.append((to_f64(state[b].index_select(0, idx)), st[0]))
        ey = rel_max_err(np.concatenate([g.ravel() for g, _ in errs_y]),
                         np.concatenate([r.ravel() for _, r in errs_y]))
        es = rel_max_err(np.concatenate([g.ravel() for g, _ in errs_s]),
                         np.concatenate([r.ravel() for _, r in errs_s]))
        assert ey <= 2e-2, f"y vs {prec}: {ey:.3g}"
        assert es <= 2e-2, f"state vs {prec}: {es:.3g}"
