"""GPU parity of ss_ssd_fwd (multi-head scalar-decay scan, tensor cores)
against oracle.ssd (fp64 recurrence, pinned in test_oracle_ssd_pins.py).
Bound: max|y - y_ref| <= 2e-2 · max|y_ref| and the same for the final state
-- the products' operands are bf16 (the masked C Bᵀ, X̃ and the carried
state's hi/lo pair round to 2^-9 relative each), accumulation fp32.  Both
d_state 64 (padded) and 128 run the tcgen05 kernel."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import selective_state_space_37_b200 as ss
from gpu_util import rel_max_err
from ss_inputs import ssd_inputs, to_f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
TOL = 2e-2


def run_and_ref(inp, softplus=True, chunk_len=0, split=True):
    y, st = ss.ss_ssd_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"], dt_bias=inp["dt_bias"],
                          softplus=softplus, chunk_len=chunk_len, split=split, sync_check=True)
    yr, sr = oracle.ssd(to_f64(inp["x"]), to_f64(inp["dt"]), to_f64(inp["A"]), to_f64(inp["B"]),
                        to_f64(inp["C"]), D=to_f64(inp["D"]), dt_bias=to_f64(inp["dt_bias"]), softplus=softplus)
    return y, st, yr, sr


SHAPES = [(2, 100, 3, 64), (1, 64, 2, 128), (2, 257, 4, 128), (1, 1, 2, 64), (3, 130, 1, 128)]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"b{b}_L{l}_H{h}_N{n}" for b, l, h, n in SHAPES])
def test_ssd_matches_oracle(shape):
    b, L, H, N = shape
    inp = ssd_inputs(b, L, H, N, seed=600 + L + H + N, device=DEV)
    y, st, yr, sr = run_and_ref(inp)
    assert rel_max_err(to_f64(y), yr) <= TOL
    assert rel_max_err(to_f64(st), sr) <= TOL


def test_ssd_softplus_off_and_no_skip():
    inp = ssd_inputs(2, 150, 2, 64, seed=7, device=DEV)
    inp["dt"] = (inp["dt"].float().abs() * 0.05 + 0.01).to(torch.bfloat16)
    inp["D"] = None
    inp["dt_bias"] = None
    y, st, yr, sr = run_and_ref(inp, softplus=False)
    assert rel_max_err(to_f64(y), yr) <= TOL
    assert rel_max_err(to_f64(st), sr) <= TOL


def test_ssd_zero_length_and_bad_sizes():
    inp = ssd_inputs(2, 0, 3, 64, seed=1, device=DEV)
    y, st = ss.ss_ssd_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], sync_check=True)
    assert torch.count_nonzero(st).item() == 0
    dims = ss.ss_ssd_dims(1, 8, 2, 32, 64)        # headdim 32: unsupported
    launch = ss.ss_launch(torch.cuda.current_stream().cuda_stream, None, 0, 0, 0)
    rc = ss.lib().ss_ssd_fwd(None, None, None, inp["A"].data_ptr(), None, None, None, None, None, 0, dims,
                             ctypes.byref(launch))
    assert rc == ss.SS_ERR_UNSUPPORTED


def test_ssd_full_size_sampled_heads():
    """The Mamba-2-2.7B-shaped layer (batch 4, L 8192, 80 heads, d_state 128)
    in the bench's launch configuration; the oracle recomputes a sample of
    (batch, head) pairs alone (heads are independent), every step and every
    channel of each."""
    b, L, H, N = 4, 8192, 80, 128
    inp = ssd_inputs(b, L, H, N, seed=3, device=DEV)
    y, st = ss.ss_ssd_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"], dt_bias=inp["dt_bias"],
                          sync_check=True)
    rng = np.random.default_rng(5)
    picks = [(int(rng.integers(b)), int(h)) for h in rng.choice(H, size=6, replace=False)]
    picks.append((b - 1, H - 1))   # the last sequence: on 148 SMs it is among those cut into segments
    for bi, h in picks:
        yr, sr = oracle.ssd(to_f64(inp["x"][bi:bi + 1, :, h:h + 1]), to_f64(inp["dt"][bi:bi + 1, :, h:h + 1]),
                            to_f64(inp["A"][h:h + 1]), to_f64(inp["B"][bi:bi + 1]), to_f64(inp["C"][bi:bi + 1]),
                            D=to_f64(inp["D"][h:h + 1]), dt_bias=to_f64(inp["dt_bias"][h:h + 1]))
        assert rel_max_err(to_f64(y[bi:bi + 1, :, h:h + 1]), yr) <= TOL, (bi, h)
        assert rel_max_err(to_f64(st[bi:bi + 1, h:h + 1]), sr) <= TOL, (bi, h)
    del inp, y, st
    torch.cuda.empty_cache()


# Forced time segments (the segment length rounds up to whole 128-step
# chunks): 2 .. 8 segments, ragged last chunk and segment, both state widths;
# the state pass, the fold and the main pass must carry the state exactly.
SEGS = [((2, 1000, 3, 128), 128), ((1, 333, 2, 64), 64), ((3, 700, 2, 128), 200), ((1, 4096, 1, 64), 512)]


@pytest.mark.parametrize("shape,seg", SEGS, ids=[f"b{b}_L{l}_H{h}_N{n}_s{s}" for (b, l, h, n), s in SEGS])
def test_ssd_time_segments(shape, seg):
    b, L, H, N = shape
    inp = ssd_inputs(b, L, H, N, seed=700 + L + seg, device=DEV)
    y, st, yr, sr = run_and_ref(inp, chunk_len=seg)
    assert rel_max_err(to_f64(y), yr) <= TOL
    assert rel_max_err(to_f64(st), sr) <= TOL


# Chunk boundaries of the 128-step chunks: one step short, exact, one over,
# two chunks, three chunks and one step; both state widths (64 is padded).
EDGES = [(L, N) for L in (127, 128, 129, 256, 385) for N in (64, 128)]


@pytest.mark.parametrize("L,N", EDGES, ids=[f"L{l}_N{n}" for l, n in EDGES])
def test_ssd_chunk_boundaries(L, N):
    inp = ssd_inputs(1, L, 2, N, seed=900 + L + N, device=DEV)
    y, st, yr, sr = run_and_ref(inp)
    assert rel_max_err(to_f64(y), yr) <= TOL
    assert rel_max_err(to_f64(st), sr) <= TOL


def test_ssd_extreme_decays():
    """Three heads: a fast decay with large steps (A = -30, Δ around 5, so
    e^{cum} underflows within a few steps and the mask's factored decays
    underflow with it), a near-zero decay rate and no decay at all (A = 0: the
    state sums every input of the sequence)."""
    inp = ssd_inputs(2, 300, 3, 128, seed=41, device=DEV)
    inp["A"] = torch.tensor([-30.0, -1e-3, 0.0], dtype=torch.float32, device=DEV)
    inp["dt_bias"] = torch.tensor([5.0, -2.0, -3.0], dtype=torch.float32, device=DEV)
    y, st, yr, sr = run_and_ref(inp)
    for h in range(3):
        assert rel_max_err(to_f64(y[:, :, h]), yr[:, :, h]) <= TOL, h
        assert rel_max_err(to_f64(st[:, h]), sr[:, h]) <= TOL, h


def test_ssd_full_size_sampled_heads_dstate64():
    """The padded d_state 64 path at the 2.7B layer's size (batch 4, L 8192,
    80 heads), sampled (batch, head) pairs against the oracle."""
    b, L, H, N = 4, 8192, 80, 64
    inp = ssd_inputs(b, L, H, N, seed=13, device=DEV)
    y, st = ss.ss_ssd_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"], dt_bias=inp["dt_bias"],
                          sync_check=True)
    rng = np.random.default_rng(9)
    picks = [(int(rng.integers(b)), int(h)) for h in rng.choice(H, size=4, replace=False)]
    for bi, h in picks:
        yr, sr = oracle.ssd(to_f64(inp["x"][bi:bi + 1, :, h:h + 1]), to_f64(inp["dt"][bi:bi + 1, :, h:h + 1]),
                            to_f64(inp["A"][h:h + 1]), to_f64(inp["B"][bi:bi + 1]), to_f64(inp["C"][bi:bi + 1]),
                            D=to_f64(inp["D"][h:h + 1]), dt_bias=to_f64(inp["dt_bias"][h:h + 1]))
        assert rel_max_err(to_f64(y[bi:bi + 1, :, h:h + 1]), yr) <= TOL, (bi, h)
        assert rel_max_err(to_f64(st[bi:bi + 1, h:h + 1]), sr) <= TOL, (bi, h)
    del inp, y, st
    torch.cuda.empty_cache()


def test_ssd_split_matches_whole():
    """Segments re-associate an exact linear recurrence: split and whole
    results agree far inside the bf16 bound."""
    inp = ssd_inputs(2, 2048, 4, 128, seed=17, device=DEV)
    y1, s1 = ss.ss_ssd_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"], dt_bias=inp["dt_bias"],
                           split=False, sync_check=True)
    y2, s2 = ss.ss_ssd_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"], dt_bias=inp["dt_bias"],
                           chunk_len=256, sync_check=True)
    assert rel_max_err(to_f64(y2), to_f64(y1)) <= 1e-2
    assert rel_max_err(to_f64(s2), to_f64(s1)) <= 1e-2


def test_ssd_mamba2_130m_full():
    """The Mamba-2-130M-shaped layer (batch 8, L 2048, 24 heads, d_state 128)
    with the library's own segment choice, every output against the oracle."""
    inp = ssd_inputs(8, 2048, 24, 128, seed=3, device=DEV)
    y, st, yr, sr = run_and_ref(inp)
    assert rel_max_err(to_f64(y), yr) <= TOL
    assert rel_max_err(to_f64(st), sr) <= TOL


def test_ssd_bounded_wait_reports_timeout_and_context_survives():
    """d_state 128: a hand-over that is never signalled (SS_TEST_DROP_CARRY:
    the first CTA's first C Bᵀ completion) makes the compute warps' bounded
    wait run out, and with it the producer's wait for their mask.  The call
    reports SS_ERR_TIMEOUT through the workspace's status word (no hang, no
    trap: copies in flight are drained, MMAs completed and TMEM released
    before the CTA ends), and the next call on the same context is correct."""
    inp = ssd_inputs(2, 300, 3, 128, seed=77, device=DEV)
    dims = ss.ss_ssd_dims(2, 300, 3, 64, 128)
    nb = int(ss.lib().ss_ssd_fwd_workspace_bytes(ctypes.byref(dims), 0))
    ws = torch.zeros(nb, dtype=torch.uint8, device=DEV)
    args = (inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"])
    kw = dict(D=inp["D"], dt_bias=inp["dt_bias"], workspace=ws)
    ss.ss_ssd_fwd(*args, **kw, timeout_iters=200, extra_flags=ss.SS_TEST_DROP_CARRY)
    assert ss.ss_check(ws) == ss.SS_ERR_TIMEOUT
    y, st = ss.ss_ssd_fwd(*args, **kw, sync_check=True)
    assert ss.ss_check(ws) == ss.SS_OK
    yr, sr = oracle.ssd(to_f64(inp["x"]), to_f64(inp["dt"]), to_f64(inp["A"]), to_f64(inp["B"]),
                        to_f64(inp["C"]), D=to_f64(inp["D"]), dt_bias=to_f64(inp["dt_bias"]), softplus=True)
    assert rel_max_err(to_f64(y), yr) <= TOL
    assert rel_max_err(to_f64(st), sr) <= TOL
