"""GPU parity of the fused conv1d + SiLU prologue (ss_fwd_conv, ss_step_conv)
against the CPU oracle: oracle.conv_silu (pinned against torch's conv1d) then
the scan oracle, on the same inputs.  Bounds as for ss_fwd: 1e-5 · max|y_ref|
with fp32 inputs, 2e-2 · max|y_ref| with bf16 inputs (state fp32)."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_37_b200 as ss
from gpu_util import rel_max_err, tol_for
from ss_inputs import conv_params, fwd_inputs, step_inputs, to_f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def oracle_conv_fwd(inp, w, b, precision="f32"):
    u = oracle.conv_silu(to_f64(inp["u"]), to_f64(w), to_f64(b))
    return oracle.fwd(u, to_f64(inp["delta"]), to_f64(inp["A"]), to_f64(inp["B"]), to_f64(inp["C"]),
                      D=to_f64(inp["D"]), z=to_f64(inp["z"]), delta_bias=to_f64(inp["delta_bias"]),
                      precision=precision)


def run(inp, w, b, **kw):
    return ss.ss_fwd_conv(inp["u"], w, inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                          delta_bias=inp["delta_bias"], conv_b=b, sync_check=True, **kw)


def check(inp, w, b, y, st, precisions=("f32",)):
    tol = tol_for(inp["u"].dtype)
    for prec in precisions:
        yr, sr = oracle_conv_fwd(inp, w, b, prec)
        assert rel_max_err(to_f64(y), yr) <= tol
        assert rel_max_err(to_f64(st), sr) <= tol


SHAPES = [(2, 200, 200), (1, 97, 256), (2, 33, 40), (38, 100, 512)]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"b{b}_L{l}_d{d}" for b, l, d in SHAPES])
@pytest.mark.parametrize("chunk", [0, 32, 96])
def test_fwd_conv_bf16(shape, chunk):
    b, L, d = shape
    seed = 500 + b + L + d + chunk
    inp = fwd_inputs(b, L, d, 16, "bf16", seed, DEV, gate=True, D_kind="normal")
    w, cb = conv_params(d, seed, DEV, bias="normal" if chunk else "zero")
    y, st = run(inp, w, cb, chunk_len=chunk)
    check(inp, w, cb, y, st)


@pytest.mark.parametrize("shape", [(38, 100, 512), (2, 200, 200)], ids=["wide", "narrow"])
def test_fwd_conv_bf16_no_gate(shape):
    """Without the gate the prologue runs in the kernel that is not
    specialised for softplus and gate both on."""
    b, L, d = shape
    inp = fwd_inputs(b, L, d, 16, "bf16", 640 + d, DEV, gate=False, D_kind="normal")
    w, cb = conv_params(d, 640 + d, DEV, bias="normal")
    for chunk in (0, 64):
        y, st = run(inp, w, cb, chunk_len=chunk)
        check(inp, w, cb, y, st)


@pytest.mark.parametrize("chunk", [0, 64])
def test_fwd_conv_fp32(chunk):
    inp = fwd_inputs(2, 130, 64, 16, "fp32", 71, DEV, gate=True, D_kind="normal")
    w, cb = conv_params(64, 71, DEV, bias="normal")
    y, st = run(inp, w, cb, chunk_len=chunk)
    check(inp, w, cb, y, st, precisions=("f32", "f64"))


def test_conv_state_is_the_last_three_inputs():
    for L in (1, 2, 5, 64):
        inp = fwd_inputs(2, L, 96, 16, "bf16", 80 + L, DEV)
        w, cb = conv_params(96, 80, DEV)
        cs = torch.full((2, 96, 3), 7.0, device=DEV)
        run(inp, w, cb, conv_state=cs)
        ref = torch.zeros(2, 96, 3, device=DEV)
        k = min(L, 3)
        ref[:, :, 3 - k:] = inp["u"][:, L - k:, :].float().permute(0, 2, 1)
        assert torch.equal(cs, ref), L


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_step_conv_sequence_matches_fwd_conv(dtype):
    b, L, d = 3, 40, 128
    inp = fwd_inputs(b, L, d, 16, dtype, 90, DEV, gate=True, D_kind="normal")
    w, cb = conv_params(d, 90, DEV, bias="normal")
    y_f, st_f = run(inp, w, cb)
    state = torch.zeros(b, d, 16, device=DEV)
    cstate = torch.zeros(b, d, 3, device=DEV)
    ys = []
    for t in range(L):
        ys.append(ss.ss_step_conv(state, cstate, inp["u"][:, t].contiguous(), w, inp["delta"][:, t].contiguous(),
                                  inp["A"], inp["B"][:, t].contiguous(), inp["C"][:, t].contiguous(), D=inp["D"],
                                  z=inp["z"][:, t].contiguous(), delta_bias=inp["delta_bias"], conv_b=cb,
                                  sync_check=True))
    y_s = torch.stack(ys, dim=1)
    tol = tol_for(inp["u"].dtype)
    yr, sr = oracle_conv_fwd(inp, w, cb)
    assert rel_max_err(to_f64(y_s), yr) <= tol
    assert rel_max_err(to_f64(state), sr) <= tol
    assert rel_max_err(to_f64(y_s), to_f64(y_f)) <= tol
    ref_cs = inp["u"][:, L - 3:, :].float().permute(0, 2, 1)
    assert torch.equal(cstate, ref_cs)


def test_fwd_conv_rejects_missing_weights():
    inp = fwd_inputs(1, 16, 64, 16, "bf16", 3, DEV)
    dims = ss.ss_dims(1, 16, 64, 16)
    launch = ss.ss_launch(torch.cuda.current_stream().cuda_stream, None, 0, 0, 0)
    y = torch.empty_like(inp["u"])
    p = lambda t: None if t is None else t.data_ptr()
    rc = ss.lib().ss_fwd_conv(p(inp["u"]), None, None, p(inp["delta"]), None, p(inp["A"]), p(inp["B"]),
                              p(inp["C"]), None, None, p(y), None, None, ss.SS_BF16, dims, launch)
    assert rc == ss.SS_ERR_INVALID_ARG
