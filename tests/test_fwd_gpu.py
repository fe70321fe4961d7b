"""GPU parity of ss_fwd against the CPU oracle, through the C ABI.

Bound (stated for the path): max|y - y_ref| <= 1e-5 * max|y_ref| for fp32
inputs and <= 2e-2 * max|y_ref| for bf16 inputs, with the state kept in fp32
on both sides; the same bound applies to the final state.  Small problems are
compared element by element; the full-size workloads (run in the launch
configuration the benchmark times) on a seeded sample of channels over the
whole sequence.
"""
import numpy as np
import pytest
import torch

import selective_state_space_37_b200 as ss
from gpu_util import (compare_samples, gpu_samples, oracle_full, oracle_samples, rel_max_err,
                      tol_for)
from ss_inputs import CONFIGS, fwd_inputs, sample_channels, to_f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def run(inp, **kw):
    return ss.ss_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                     z=inp["z"], delta_bias=inp["delta_bias"], **kw)


def check_full(inp, y, st, precisions=("f32", "f64"), softplus=True):
    tol = tol_for(inp["u"].dtype)
    for prec in precisions:
        yr, sr = oracle_full(inp, precision=prec, softplus=softplus)
        ey = rel_max_err(to_f64(y), yr)
        es = rel_max_err(to_f64(st), sr)
        assert ey <= tol, f"y vs {prec} oracle: {ey:.3g} > {tol}"
        assert es <= tol, f"last_state vs {prec} oracle: {es:.3g} > {tol}"


def cfg_inputs(name, device=DEV):
    c = CONFIGS[name]
    return c, fwd_inputs(c.batch, c.seqlen, c.d_inner, c.d_state, c.dtype, c.seed, device,
                         gate=c.gate, D_kind=c.D_kind)


# --------------------------------------------------------------- tiny fp32
@pytest.mark.parametrize("chunk", [0, 32])
def test_tiny_fp32_config(chunk):
    _, inp = cfg_inputs("tiny_fp32")
    y, st = run(inp, chunk_len=chunk, sync_check=True)
    check_full(inp, y, st)


# ------------------------------------------------ small problems, all paths
SHAPES = [(2, 200, 200), (1, 97, 256), (3, 64, 128), (1, 1, 128), (2, 33, 40), (1, 300, 520)]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"b{b}_L{l}_d{d}" for b, l, d in SHAPES])
@pytest.mark.parametrize("A_kind", ["structured", "general"])
@pytest.mark.parametrize("chunk", [0, 32, 96])
def test_small_bf16(shape, A_kind, chunk):
    b, L, d = shape
    seed = 100 + b * 7 + L + d + (1 if A_kind == "general" else 0) + chunk
    gate = (L + chunk) % 2 == 0
    inp = fwd_inputs(b, L, d, 16, "bf16", seed, DEV, gate=gate,
                     D_kind="normal" if d % 3 else "none", bias=(d % 5 != 0), A_kind=A_kind)
    y, st = run(inp, chunk_len=chunk, sync_check=True)
    check_full(inp, y, st, precisions=("f32",))


@pytest.mark.parametrize("shape", [(38, 100, 512), (20, 600, 512), (19, 333, 1000)],
                         ids=["wide_many_blocks", "wide_two_chunks", "wide_ragged"])
def test_wide_variant_shapes(shape):
    """Problems with at least half an SM's worth of channel blocks per SM run
    the one-CTA-per-SM variant (the small tests above run the two-CTA one)."""
    b, L, d = shape
    inp = fwd_inputs(b, L, d, 16, "bf16", 40 + b + L + d, DEV, gate=True, D_kind="normal")
    for chunk in (0, 96):
        y, st = run(inp, chunk_len=chunk, sync_check=True)
        check_full(inp, y, st, precisions=("f32",))


@pytest.mark.parametrize("gate,softplus", [(False, True), (True, False), (False, False)],
                         ids=["no_gate", "no_softplus", "neither"])
def test_wide_variant_options(gate, softplus):
    """The one-CTA-per-SM variant with the gate or the softplus off: the
    kernel instantiated for both on is not the one that runs here."""
    inp = fwd_inputs(38, 100, 512, 16, "bf16", 61, DEV, gate=gate, D_kind="normal", bias=softplus)
    if not softplus:
        inp["delta"] = (inp["delta"].float().abs() * 0.1).to(torch.bfloat16)
    for chunk in (0, 64):
        y, st = run(inp, chunk_len=chunk, softplus=softplus, sync_check=True)
        check_full(inp, y, st, precisions=("f32",), softplus=softplus)


@pytest.mark.parametrize("shape", [(2, 130, 64), (1, 70, 96), (2, 200, 30)])
@pytest.mark.parametrize("chunk", [0, 64])
def test_small_fp32(shape, chunk):
    b, L, d = shape
    inp = fwd_inputs(b, L, d, 16, "fp32", 7 + L + d, DEV, gate=True, D_kind="normal",
                     A_kind="general" if d % 2 else "structured")
    y, st = run(inp, chunk_len=chunk, sync_check=True)
    check_full(inp, y, st)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("d", [100, 36])
def test_unaligned_row_stride_plain_path(dtype, d):
    """Rows whose byte length is not a multiple of 16 take the non-TMA path."""
    inp = fwd_inputs(2, 150, d, 16, dtype, 31 + d, DEV, gate=True, D_kind="ones")
    for chunk in (0, 64):
        y, st = run(inp, chunk_len=chunk, sync_check=True)
        check_full(inp, y, st, precisions=("f32",))


def test_softplus_off():
    inp = fwd_inputs(2, 120, 128, 16, "bf16", 55, DEV, gate=True, D_kind="ones", bias=False)
    inp["delta"] = (inp["delta"].float().abs() * 0.1).to(torch.bfloat16)
    y, st = run(inp, softplus=False, chunk_len=64, sync_check=True)
    check_full(inp, y, st, precisions=("f32",), softplus=False)


def test_force_general_matches_structured():
    inp = fwd_inputs(2, 256, 256, 16, "bf16", 77, DEV, gate=True, D_kind="ones")
    y1, s1 = run(inp, chunk_len=64, sync_check=True)
    y2, s2 = run(inp, chunk_len=64, force_general_A=True, sync_check=True)
    assert rel_max_err(to_f64(y1), to_f64(y2)) <= 2e-2
    assert rel_max_err(to_f64(s1), to_f64(s2)) <= 2e-2


def test_chunk_lengths_agree():
    inp = fwd_inputs(1, 1000, 384, 16, "bf16", 78, DEV, gate=True, D_kind="normal")
    yr, sr = oracle_full(inp, precision="f32")
    for chunk in (32, 64, 160, 512, 992, 4096):
        y, st = run(inp, chunk_len=chunk, sync_check=True)
        assert rel_max_err(to_f64(y), yr) <= 2e-2, chunk
        assert rel_max_err(to_f64(st), sr) <= 2e-2, chunk


# ------------------------------------------------------------ edge cases
def test_zero_length_writes_zero_state():
    inp = fwd_inputs(2, 0, 64, 16, "bf16", 1, DEV)
    st = torch.full((2, 64, 16), 7.0, device=DEV)
    y, st = run(inp, last_state=st, sync_check=True)
    assert y.shape == (2, 0, 64)
    assert torch.count_nonzero(st).item() == 0


def test_empty_batch_is_noop():
    inp = fwd_inputs(0, 16, 64, 16, "bf16", 1, DEV)
    y, st = run(inp, sync_check=True)
    assert y.numel() == 0 and st.numel() == 0


def test_no_last_state():
    inp = fwd_inputs(1, 64, 128, 16, "bf16", 2, DEV)
    y, st = run(inp, return_last_state=False, chunk_len=32, sync_check=True)
    assert st is None
    yr, _ = oracle_full(inp)
    assert rel_max_err(to_f64(y), yr) <= 2e-2


def test_misaligned_pointer_is_rejected():
    inp = fwd_inputs(1, 32, 64, 16, "bf16", 3, DEV)
    raw = torch.empty(32 * 64 + 1, dtype=torch.bfloat16, device=DEV)
    u_off = raw[1:].view(1, 32, 64)
    u_off.copy_(inp["u"])
    with pytest.raises(ss.SelscanError) as e:
        ss.ss_fwd(u_off, inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"])
    assert e.value.status == ss.SS_ERR_INVALID_ARG


def test_workspace_too_small_is_rejected():
    inp = fwd_inputs(1, 256, 128, 16, "bf16", 4, DEV)
    ws = torch.empty(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(ss.SelscanError) as e:
        run(inp, chunk_len=32, workspace=ws)
    assert e.value.status == ss.SS_ERR_WORKSPACE


def test_bounded_wait_reports_timeout_and_context_survives():
    """A carry that is never published makes its successor's bounded wait run
    out: the call reports SS_ERR_TIMEOUT (no hang, no trap), and the next call
    on the same context is correct."""
    inp = fwd_inputs(1, 128, 128, 16, "bf16", 5, DEV)
    nbytes = ss.fwd_workspace_bytes(1, 128, 128, True, 32)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    run(inp, chunk_len=32, workspace=ws, timeout_iters=2000, extra_flags=ss.SS_TEST_DROP_CARRY)
    assert ss.ss_check(ws) == ss.SS_ERR_TIMEOUT
    y, st = run(inp, chunk_len=32, workspace=ws, sync_check=True)
    assert ss.ss_check(ws) == ss.SS_OK
    check_full(inp, y, st, precisions=("f32",))


# ------------------------------------------------------ full-size workloads
def test_config_mamba130m_full():
    c, inp = cfg_inputs("mamba130m")
    y, st = run(inp, sync_check=True)
    check_full(inp, y, st, precisions=("f32",))
    samples = sample_channels(c.batch, c.d_inner, 16, c.seed)
    ref = oracle_samples(inp, samples, precision="f64")
    ey, es = compare_samples(gpu_samples(y, st, samples), ref, 2e-2)
    assert ey <= 2e-2 and es <= 2e-2


@pytest.mark.parametrize("name,count", [("mamba2p8b", 64), ("million", 64)])
def test_config_sampled(name, count):
    c, inp = cfg_inputs(name)
    y, st = run(inp, sync_check=True)
    samples = sample_channels(c.batch, c.d_inner, count, c.seed)
    got = gpu_samples(y, st, samples)
    for prec in ("f32", "f64"):
        ref = oracle_samples(inp, samples, precision=prec)
        ey, es = compare_samples(got, ref, 2e-2)
        assert ey <= 2e-2, f"{name} y vs {prec}: {ey:.3g}"
        assert es <= 2e-2, f"{name} state vs {prec}: {es:.3g}"
    del inp, y, st
    torch.cuda.empty_cache()


# ------------------------------------------------- entering state (continuation)
CONT = [((2, 400, 256), 150, 0, 0), ((2, 400, 256), 256, 64, 64), ((1, 700, 128), 333, 0, 96),
        ((3, 130, 70), 64, 32, 32)]


@pytest.mark.parametrize("shape,split,c1,c2", CONT,
                         ids=[f"b{b}_L{l}_d{d}_at{s}_c{c1}_{c2}" for (b, l, d), s, c1, c2 in CONT])
def test_continuation_from_last_state(shape, split, c1, c2):
    """ss_fwd over [0, T) then ss_fwd_with_state over [T, L) from its last
    state reproduces the whole-sequence oracle (every output of both parts
    and the final state), with and without time chunks in either part."""
    b, L, d = shape
    inp = fwd_inputs(b, L, d, 16, "bf16", 55 + L + split, DEV, gate=True, D_kind="normal")
    part = lambda sl: {k: (v[:, sl].contiguous() if k in ("u", "delta", "z", "B", "C") and v is not None else v)
                       for k, v in inp.items()}
    p1, p2 = part(slice(0, split)), part(slice(split, L))
    y1, s1 = run(p1, chunk_len=c1, sync_check=True)
    y2, s2 = run(p2, chunk_len=c2, initial_state=s1, sync_check=True)
    yr, sr = oracle_full(inp, precision="f64")
    tol = tol_for(torch.bfloat16)
    assert rel_max_err(to_f64(torch.cat([y1, y2], dim=1)), yr) <= tol
    assert rel_max_err(to_f64(s2), sr) <= tol


def test_with_state_zero_length_and_zero_state():
    inp = fwd_inputs(2, 0, 64, 16, "bf16", 3, DEV)
    h0 = torch.randn(2, 64, 16, device=DEV)
    _, st = run(inp, initial_state=h0, sync_check=True)
    assert torch.equal(st, h0)
    inp = fwd_inputs(2, 100, 64, 16, "bf16", 4, DEV, gate=True)
    ya, sa = run(inp, sync_check=True)
    yb, sb = run(inp, initial_state=torch.zeros(2, 64, 16, device=DEV), sync_check=True)
    assert torch.equal(ya, yb) and torch.equal(sa, sb)
