"""ss_fwd_noalloc: the forward scan for callers that cannot allocate device
memory (fixed-memory runtimes, plugin interfaces with no allocator, paths
that cannot afford cudaMalloc's synchronization).  It runs on a scratch array
the library reserves when loaded, instead of a caller workspace.

Checked through the C ABI against ss_fwd (the entry point with a caller
workspace) on the same inputs, within the bf16 parity bound the other tests
use, on two calls in a row (the shared array keeps the previous call's
contents, so the second call also checks that what must start at zero is
reset), and against the CPU oracle as well.  This file is collected last; it passes alone in a fresh process and
after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import selective_state_space_37_b200 as ss
from selective_state_space_37_b200 import _binding as bd
from ss_inputs import fwd_inputs, to_f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
TOL = 2e-2   # bf16 inputs, fp32 state: max|y - y_ref| <= TOL * max|y_ref|


def _rel(a, b):
    a, b = to_f64(a), to_f64(b)
    return float(np.max(np.abs(a - b)) / np.max(np.abs(b)))


def _noalloc(inp, y, st, flags, dims, stream):
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return ss.lib().ss_fwd_noalloc(p(inp["u"]), p(inp["delta"]), p(inp["delta_bias"]), p(inp["A"]),
                                   p(inp["B"]), p(inp["C"]), p(inp["D"]), p(inp["z"]), p(y), p(st),
                                   flags, ctypes.byref(dims), ctypes.c_void_p(stream))


def test_noalloc_matches_workspace_entry_point_twice():
    # Time-chunked problem, so the carry records in the scratch array are used.
    batch, L, d = 2, 1000, 384
    assert ss.fwd_chunk_len(batch, L, d) > 0
    inp = fwd_inputs(batch, L, d, 16, "bf16", 2024, DEV, gate=True, D_kind="normal")
    y_ref, st_ref = ss.ss_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                              z=inp["z"], delta_bias=inp["delta_bias"], sync_check=True)
    dims = bd.ss_dims(batch, L, d, 16)
    flags = bd.SS_BF16 | bd.SS_DELTA_SOFTPLUS | bd.SS_SYNC_CHECK
    stream = torch.cuda.current_stream(DEV).cuda_stream
    yo, so = oracle.fwd(to_f64(inp["u"]), to_f64(inp["delta"]), to_f64(inp["A"]), to_f64(inp["B"]),
                        to_f64(inp["C"]), D=to_f64(inp["D"]), z=to_f64(inp["z"]),
                        delta_bias=to_f64(inp["delta_bias"]), precision="f32")
    for _ in range(2):
        y = torch.full_like(y_ref, float("nan"))
        st = torch.full_like(st_ref, float("nan"))
        rc = _noalloc(inp, y, st, flags, dims, stream)
        assert rc == ss.SS_OK, ss.status_string(rc)
        assert _rel(y, y_ref) <= TOL
        assert _rel(st, st_ref) <= TOL
        assert float(np.max(np.abs(to_f64(y) - yo)) / np.max(np.abs(yo))) <= TOL
        assert float(np.max(np.abs(to_f64(st) - so)) / np.max(np.abs(so))) <= TOL


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # Many channels and enough time chunks need more carry records than the
    # array holds: rejected before any launch, so placeholder pointers are
    # never touched.
    batch, L, d = 1, 1 << 20, 1 << 16
    need = ss.fwd_workspace_bytes(batch, L, d, True, 0)
    assert need > (32 << 20)
    dims = bd.ss_dims(batch, L, d, 16)
    fake = ctypes.c_void_p(256)
    rc = ss.lib().ss_fwd_noalloc(fake, fake, None, fake, fake, fake, None, None, fake, None,
                                 bd.SS_BF16 | bd.SS_DELTA_SOFTPLUS, ctypes.byref(dims), None)
    assert rc == ss.SS_ERR_WORKSPACE
