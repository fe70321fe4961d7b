"""Helpers for the GPU parity tests: run the CPU oracle on the exact inputs the
GPU consumed (whole problems, or a sample of channels over the full length)
and compare with the bound max|y - y_ref| <= tol * max|y_ref|."""
import numpy as np
import torch

import oracle
from ss_inputs import to_f64

TOL_FP32 = 1e-5   # fp32 inputs, state kept in fp32
TOL_BF16 = 2e-2   # bf16 inputs, state kept in fp32


def tol_for(dtype):
    return TOL_FP32 if dtype == torch.float32 else TOL_BF16


def rel_max_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    return err / den if den > 0 else err


def oracle_full(inp, precision="f32", softplus=True):
    """Oracle over the whole problem. Returns (y [b,L,d], last_state [b,d,N]) float64."""
    return oracle.fwd(to_f64(inp["u"]), to_f64(inp["delta"]), to_f64(inp["A"]), to_f64(inp["B"]),
                      to_f64(inp["C"]), D=to_f64(inp.get("D")), z=to_f64(inp.get("z")),
                      delta_bias=to_f64(inp.get("delta_bias")), softplus=softplus,
                      precision=precision)


def oracle_samples(inp, samples, precision="f32", softplus=True):
    """Oracle on a list of (b, ch) channels over the full length.
    Returns {(b, ch): (y [L], state [N])} in float64."""
    out = {}
    by_b = {}
    for b, ch in samples:
        by_b.setdefault(b, []).append(ch)
    for b, chs in by_b.items():
        idx = torch.tensor(chs, dtype=torch.long, device=inp["u"].device)

        def cols(t):
            return None if t is None else to_f64(t[b].index_select(1, idx))[None]

        def vec(t):
            return None if t is None else to_f64(t.index_select(0, idx))

        y, st = oracle.fwd(cols(inp["u"]), cols(inp["delta"]), vec(inp["A"]),
                           to_f64(inp["B"][b])[None], to_f64(inp["C"][b])[None],
                           D=vec(inp.get("D")), z=cols(inp.get("z")),
                           delta_bias=vec(inp.get("delta_bias")), softplus=softplus,
                           precision=precision)
        for k, ch in enumerate(chs):
            out[(b, ch)] = (y[0, :, k], st[0, k])
    return out


def gpu_samples(y, last_state, samples):
    out = {}
    by_b = {}
    for b, ch in samples:
        by_b.setdefault(b, []).append(ch)
    for b, chs in by_b.items():
        idx = torch.tensor(chs, dtype=torch.long, device=y.device)
        ys = to_f64(y[b].index_select(1, idx))
        ss = to_f64(last_state[b].index_select(0, idx)) if last_state is not None else None
        for k, ch in enumerate(chs):
            out[(b, ch)] = (ys[:, k], None if ss is None else ss[k])
    return out


def compare_samples(gpu, ref, tol):
    """Relative max error over all sampled channels, for y and for the state."""
    gy = np.concatenate([gpu[k][0] for k in ref])
    ry = np.concatenate([ref[k][0] for k in ref])
    ey = rel_max_err(gy, ry)
    es = 0.0
    if all(gpu[k][1] is not None for k in ref):
        gs = np.concatenate([gpu[k][1] for k in ref])
        rs = np.concatenate([ref[k][1] for k in ref])
        es = rel_max_err(gs, rs)
    return ey, es
