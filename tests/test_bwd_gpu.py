"""GPU parity of ss_bwd against the fp64 backward oracle, through the C ABI.

Bounds, each relative to max|ref| of the output compared:
  - fp32 inputs: 1e-4 for every gradient.  The kernel works in fp32 with the
    CUDA math library; the largest error comes from sums over up to batch·L
    (dA, dD, dbias) or d (dB, dC) terms rounded in fp32 (~1e-6 here), so the
    bound keeps a wide margin while failing on any dropped or wrong term.
  - bf16 inputs: du, ddelta, dz are rounded to bf16 on output (2^-9 relative
    per element): 1e-2.  dA, dB, dC, dD, dbias stay fp32, computed with the
    hardware approximate exp2 / log2 / reciprocal (relative error ~1e-6): 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_37_b200 as ss
from gpu_util import rel_max_err
from ss_inputs import CONFIGS, bwd_upstream, fwd_inputs, to_f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")

IO_GRADS = ("du", "ddelta", "dz")
ORACLE_KEY = {"du": "du", "ddelta": "ddelta", "dz": "dz", "dA": "dA", "dB": "dB", "dC": "dC",
              "dD": "dD", "ddelta_bias": "dbias"}


def tols(dtype):
    if dtype == torch.float32:
        return 1e-4, 1e-4
    return 1e-2, 2e-3


def run_both(inp, dy, dl, softplus=True, chunk_len=0):
    got = ss.ss_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy, D=inp["D"], z=inp["z"],
                    delta_bias=inp["delta_bias"], dlast_state=dl, softplus=softplus, chunk_len=chunk_len,
                    sync_check=True)
    ref = oracle.bwd(to_f64(inp["u"]), to_f64(inp["delta"]), to_f64(inp["A"]), to_f64(inp["B"]),
                     to_f64(inp["C"]), to_f64(dy), D=to_f64(inp["D"]), z=to_f64(inp["z"]),
                     delta_bias=to_f64(inp["delta_bias"]), dlast=to_f64(dl), softplus=softplus)
    return got, ref


def check(got, ref, dtype):
    tol_io, tol_acc = tols(dtype)
    assert set(got) == {k for k, v in ORACLE_KEY.items() if v in ref}
    for k, t in got.items():
        e = rel_max_err(to_f64(t), ref[ORACLE_KEY[k]])
        bound = tol_io if k in IO_GRADS else tol_acc
        assert e <= bound, f"{k}: {e:.3g} > {bound}"


SHAPES = [(2, 200, 130), (1, 64, 64), (3, 1, 10), (2, 129, 70), (1, 300, 256)]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"b{b}_L{l}_d{d}" for b, l, d in SHAPES])
def test_bwd_bf16(shape):
    b, L, d = shape
    seed = 300 + b + L + d
    inp = fwd_inputs(b, L, d, 16, "bf16", seed, DEV, gate=True, D_kind="normal")
    dy, dl = bwd_upstream(b, L, d, 16, "bf16", seed, DEV)
    got, ref = run_both(inp, dy, dl)
    check(got, ref, torch.bfloat16)


@pytest.mark.parametrize("shape", [(2, 150, 70), (1, 70, 33)])
def test_bwd_fp32(shape):
    b, L, d = shape
    inp = fwd_inputs(b, L, d, 16, "fp32", 7 + L + d, DEV, gate=True, D_kind="normal",
                     A_kind="general" if d % 2 else "structured")
    dy, dl = bwd_upstream(b, L, d, 16, "fp32", 7 + L + d, DEV)
    got, ref = run_both(inp, dy, dl)
    check(got, ref, torch.float32)


# Forced time chunks: the chunk length is rounded up to whole 32-step
# segments, so these give 2 .. 10 chunks with a ragged last chunk and a
# ragged last segment; the chunks' carried state and adjoint must be exact.
CHUNKED = [((2, 300, 96), 64), ((1, 333, 64), 32), ((3, 200, 130), 96), ((1, 1000, 64), 100)]


@pytest.mark.parametrize("shape,chunk", CHUNKED, ids=[f"b{b}_L{l}_d{d}_c{c}" for (b, l, d), c in CHUNKED])
def test_bwd_time_chunks_bf16(shape, chunk):
    b, L, d = shape
    seed = 900 + L + chunk
    inp = fwd_inputs(b, L, d, 16, "bf16", seed, DEV, gate=True, D_kind="normal")
    dy, dl = bwd_upstream(b, L, d, 16, "bf16", seed, DEV)
    got, ref = run_both(inp, dy, dl, chunk_len=chunk)
    check(got, ref, torch.bfloat16)


def test_bwd_time_chunks_fp32_general_A():
    inp = fwd_inputs(2, 260, 70, 16, "fp32", 77, DEV, gate=True, D_kind="normal", A_kind="general")
    dy, dl = bwd_upstream(2, 260, 70, 16, "fp32", 77, DEV)
    got, ref = run_both(inp, dy, dl, chunk_len=64)
    check(got, ref, torch.float32)


def test_bwd_time_chunks_fp32_aligned_rows():
    """fp32 rows a multiple of 16 bytes: the chunk pass stages them with
    16-byte asynchronous copies (4 channels each)."""
    inp = fwd_inputs(2, 230, 64, 16, "fp32", 78, DEV, gate=True, D_kind="normal")
    dy, dl = bwd_upstream(2, 230, 64, 16, "fp32", 78, DEV)
    got, ref = run_both(inp, dy, dl, chunk_len=64)
    check(got, ref, torch.float32)


def test_bwd_chunked_matches_unchunked():
    """Chunking re-associates exact linear recurrences: the chunked and the
    one-chunk gradients agree to fp32 rounding."""
    inp = fwd_inputs(2, 640, 128, 16, "bf16", 81, DEV, gate=True, D_kind="normal")
    dy, dl = bwd_upstream(2, 640, 128, 16, "bf16", 81, DEV)
    one = ss.ss_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy, D=inp["D"], z=inp["z"],
                    delta_bias=inp["delta_bias"], dlast_state=dl, chunk_len=640, sync_check=True)
    many = ss.ss_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy, D=inp["D"], z=inp["z"],
                     delta_bias=inp["delta_bias"], dlast_state=dl, chunk_len=32, sync_check=True)
    for k in one:
        e = rel_max_err(to_f64(many[k]), to_f64(one[k]))
        assert e <= (1e-2 if k in IO_GRADS else 1e-4), f"{k}: {e:.3g}"


def test_bwd_general_A_bf16():
    inp = fwd_inputs(2, 160, 96, 16, "bf16", 41, DEV, gate=True, D_kind="ones", A_kind="general")
    dy, dl = bwd_upstream(2, 160, 96, 16, "bf16", 41, DEV)
    got, ref = run_both(inp, dy, dl)
    check(got, ref, torch.bfloat16)


@pytest.mark.parametrize("variant", ["no_gate", "no_D_no_bias", "no_dlast"])
def test_bwd_optional_inputs(variant):
    b, L, d = 2, 100, 80
    inp = fwd_inputs(b, L, d, 16, "bf16", 51, DEV, gate=(variant != "no_gate"),
                     D_kind="none" if variant == "no_D_no_bias" else "normal",
                     bias=(variant != "no_D_no_bias"))
    dy, dl = bwd_upstream(b, L, d, 16, "bf16", 51, DEV, dlast=(variant != "no_dlast"))
    got, ref = run_both(inp, dy, dl)
    check(got, ref, torch.bfloat16)


def test_bwd_softplus_off():
    inp = fwd_inputs(2, 90, 64, 16, "bf16", 61, DEV, gate=True, D_kind="ones", bias=False)
    inp["delta"] = (inp["delta"].float().abs() * 0.1 + 0.01).to(torch.bfloat16)
    dy, dl = bwd_upstream(2, 90, 64, 16, "bf16", 61, DEV)
    got, ref = run_both(inp, dy, dl, softplus=False)
    check(got, ref, torch.bfloat16)


def test_bwd_zero_length():
    inp = fwd_inputs(2, 0, 64, 16, "bf16", 1, DEV)
    dy, dl = bwd_upstream(2, 0, 64, 16, "bf16", 1, DEV)
    got = ss.ss_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy, D=inp["D"], z=inp["z"],
                    delta_bias=inp["delta_bias"], dlast_state=dl, sync_check=True)
    for k in ("dA", "dD", "ddelta_bias"):
        assert torch.count_nonzero(got[k]).item() == 0


def test_bwd_rejects_bad_arguments():
    inp = fwd_inputs(1, 32, 64, 16, "bf16", 2, DEV)
    dy, dl = bwd_upstream(1, 32, 64, 16, "bf16", 2, DEV)
    dims = ss.ss_dims(1, 32, 64, 16)
    flags = ss.SS_BF16 | ss.SS_DELTA_SOFTPLUS
    need = int(ss.lib().ss_bwd_workspace_bytes(dims, flags))
    # one 32-step segment, one chunk: checkpoints 64 x 16 fp32, their Σ Δ (64
    # floats -> 256 B), h_loc and g_loc records 64 x 16 each, Σ Δ record 256 B
    assert need == 4096 + 256 + 4096 + 4096 + 256
    g = {k: torch.empty_like(inp["u"]) for k in ("du", "ddelta", "dz")}
    f = {k: torch.empty(s, device=DEV) for k, s in (("dA", (64, 16)), ("dB", (1, 32, 16)), ("dC", (1, 32, 16)))}
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    small = torch.empty(16, dtype=torch.uint8, device=DEV)

    def call(z, dz, workspace):
        launch = ss.ss_launch(torch.cuda.current_stream().cuda_stream, workspace.data_ptr(),
                              workspace.numel(), 0, 0)
        p = lambda t: None if t is None else t.data_ptr()
        return ss.lib().ss_bwd(p(inp["u"]), p(inp["delta"]), p(inp["delta_bias"]), p(inp["A"]), p(inp["B"]),
                               p(inp["C"]), p(inp["D"]), p(z), p(dy), p(dl), p(g["du"]), p(g["ddelta"]),
                               p(f["dA"]), p(f["dB"]), p(f["dC"]), None, p(dz), None,
                               flags | ss.SS_SYNC_CHECK, dims, launch)

    assert call(inp["z"], None, ws) == ss.SS_ERR_INVALID_ARG      # dz missing while z given
    assert call(None, g["dz"], ws) == ss.SS_ERR_INVALID_ARG       # dz given without z
    assert call(inp["z"], g["dz"], small) == ss.SS_ERR_WORKSPACE
    assert call(inp["z"], g["dz"], ws) == ss.SS_OK


def test_bwd_config_mamba130m_full():
    """The 130M-shaped layer at full size, every gradient compared."""
    c = CONFIGS["mamba130m"]
    inp = fwd_inputs(c.batch, c.seqlen, c.d_inner, c.d_state, c.dtype, c.seed, DEV, gate=c.gate,
                     D_kind=c.D_kind)
    dy, dl = bwd_upstream(c.batch, c.seqlen, c.d_inner, c.d_state, c.dtype, c.seed, DEV)
    got, ref = run_both(inp, dy, dl)
    check(got, ref, torch.bfloat16)
    del inp, dy, dl, got
    torch.cuda.empty_cache()


def test_bwd_config_mamba2p8b_sampled():
    """The 2.8B-shaped layer (batch 4, L 8192, d_inner 5120) in the bench's
    launch configuration (4 time chunks).  du, dΔraw, dz, dB and dC of batch
    entry 0 against the oracle run on that entry (all channels, full L; dB and
    dC sum over its channels); dA, dD and dbias (sums over batch and time) on
    48 sampled channels against the oracle run on those channels of every
    entry."""
    c = CONFIGS["mamba2p8b"]
    inp = fwd_inputs(c.batch, c.seqlen, c.d_inner, c.d_state, c.dtype, c.seed, DEV, gate=c.gate,
                     D_kind=c.D_kind)
    dy, dl = bwd_upstream(c.batch, c.seqlen, c.d_inner, c.d_state, c.dtype, c.seed, DEV)
    got = ss.ss_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy, D=inp["D"], z=inp["z"],
                    delta_bias=inp["delta_bias"], dlast_state=dl, sync_check=True)
    tol_io, tol_acc = tols(torch.bfloat16)
    one = slice(0, 1)
    ref = oracle.bwd(to_f64(inp["u"][one]), to_f64(inp["delta"][one]), to_f64(inp["A"]), to_f64(inp["B"][one]),
                     to_f64(inp["C"][one]), to_f64(dy[one]), D=to_f64(inp["D"]), z=to_f64(inp["z"][one]),
                     delta_bias=to_f64(inp["delta_bias"]), dlast=to_f64(dl[one]))
    for k in ("du", "ddelta", "dz", "dB", "dC"):
        e = rel_max_err(to_f64(got[k][one]), ref[k])
        assert e <= (tol_io if k in IO_GRADS else tol_acc), f"{k}: {e:.3g}"
    chs = torch.from_numpy(np.sort(np.random.default_rng(11).choice(c.d_inner, size=48, replace=False))).to(DEV)
    pick = lambda t: t.index_select(-1, chs)
    ref = oracle.bwd(to_f64(pick(inp["u"])), to_f64(pick(inp["delta"])), to_f64(inp["A"][chs]), to_f64(inp["B"]),
                     to_f64(inp["C"]), to_f64(pick(dy)), D=to_f64(inp["D"][chs]), z=to_f64(pick(inp["z"])),
                     delta_bias=to_f64(inp["delta_bias"][chs]), dlast=to_f64(dl[:, chs]))
    for k, rk in (("dA", "dA"), ("dD", "dD"), ("ddelta_bias", "dbias")):
        e = rel_max_err(to_f64(got[k][chs]), ref[rk])
        assert e <= tol_acc, f"{k}: {e:.3g}"
    del inp, dy, dl, got
    torch.cuda.empty_cache()
