"""ss_fwd_host (activations in host memory, batch slices uploaded, scanned and
downloaded with the three overlapped) against ss_fwd on the same slices on
the device, and against the CPU oracle, through the C ABI."""
import ctypes

import pytest
import torch

import oracle
import selective_state_space_37_b200 as ss
from gpu_util import rel_max_err, tol_for
from ss_inputs import fwd_inputs, to_f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
ACT = ("u", "delta", "z", "B", "C")


def host_copy(inp, pin=True):
    return {k: (None if inp[k] is None else (inp[k].cpu().pin_memory() if pin else inp[k].cpu().clone()))
            for k in ACT}


def device_slices(inp, rows):
    """ss_fwd applied to each batch slice on the device: what ss_fwd_host
    must reproduce bit for bit (same kernels, same per-slice plan)."""
    b = inp["u"].shape[0]
    ys, sts = [], []
    for r0 in range(0, b, rows):
        sl = {k: (None if inp[k] is None else inp[k][r0:r0 + rows].contiguous()) for k in ACT}
        y, st = ss.ss_fwd(sl["u"], sl["delta"], inp["A"], sl["B"], sl["C"], D=inp["D"], z=sl["z"],
                          delta_bias=inp["delta_bias"], sync_check=True)
        ys.append(y)
        sts.append(st)
    return torch.cat(ys).cpu(), torch.cat(sts).cpu()


@pytest.mark.parametrize("rows", [1, 2, 3, 5])
def test_host_equals_device_slices(rows):
    inp = fwd_inputs(5, 300, 96, 16, "bf16", 41 + rows, DEV, gate=True, D_kind="normal")
    h = host_copy(inp)
    y, st = ss.ss_fwd_host(h["u"], h["delta"], inp["A"], h["B"], h["C"], D=inp["D"], z=h["z"],
                           delta_bias=inp["delta_bias"], rows_per_slice=rows, sync_check=True)
    assert y.device.type == "cpu" and st.device.type == "cpu"
    y_ref, st_ref = device_slices(inp, rows)
    assert torch.equal(y, y_ref)
    assert torch.equal(st, st_ref)


def test_host_against_oracle_and_pageable():
    inp = fwd_inputs(3, 200, 64, 16, "bf16", 7, DEV, gate=True, D_kind="normal")
    h = host_copy(inp, pin=False)
    y, st = ss.ss_fwd_host(h["u"], h["delta"], inp["A"], h["B"], h["C"], D=inp["D"], z=h["z"],
                           delta_bias=inp["delta_bias"], rows_per_slice=2, sync_check=True)
    yr, sr = oracle.fwd(to_f64(inp["u"]), to_f64(inp["delta"]), to_f64(inp["A"]), to_f64(inp["B"]),
                        to_f64(inp["C"]), D=to_f64(inp["D"]), z=to_f64(inp["z"]),
                        delta_bias=to_f64(inp["delta_bias"]))
    tol = tol_for(torch.bfloat16)
    assert rel_max_err(to_f64(y), yr) <= tol
    assert rel_max_err(to_f64(st), sr) <= tol


def test_host_fp32_no_gate_no_state():
    inp = fwd_inputs(2, 70, 32, 16, "fp32", 9, DEV, gate=False)
    h = host_copy(inp)
    y, st = ss.ss_fwd_host(h["u"], h["delta"], inp["A"], h["B"], h["C"], D=inp["D"], z=None,
                           delta_bias=inp["delta_bias"], return_last_state=False, sync_check=True)
    assert st is None
    y_ref, _ = device_slices(inp, 1)
    assert torch.equal(y, y_ref)


def test_host_zero_length_and_bad_workspace():
    inp = fwd_inputs(2, 0, 64, 16, "bf16", 3, DEV)
    h = host_copy(inp)
    y, st = ss.ss_fwd_host(h["u"], h["delta"], inp["A"], h["B"], h["C"], D=inp["D"], z=h["z"],
                           delta_bias=inp["delta_bias"], sync_check=True)
    assert y.numel() == 0 and torch.count_nonzero(st).item() == 0
    inp = fwd_inputs(2, 64, 64, 16, "bf16", 4, DEV)
    h = host_copy(inp)
    dims = ss.ss_dims(2, 64, 64, 16)
    need = int(ss.lib().ss_fwd_host_workspace_bytes(ctypes.byref(dims), ss.SS_BF16, 1))
    small = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    y = torch.empty_like(h["u"])
    launch = ss.ss_launch(torch.cuda.current_stream().cuda_stream, small.data_ptr(), small.numel(), 0, 0)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    rc = ss.lib().ss_fwd_host(p(h["u"]), p(h["delta"]), p(inp["delta_bias"]), p(inp["A"]), p(h["B"]), p(h["C"]),
                              p(inp["D"]), p(h["z"]), p(y), None, ss.SS_BF16 | ss.SS_DELTA_SOFTPLUS,
                              ctypes.byref(dims), ctypes.byref(launch), 1)
    assert rc == ss.SS_ERR_WORKSPACE


def test_host_failure_in_first_slice_stays_reported():
    """A device-side failure in one slice stays in the call's status word: the
    first slice's dropped carry (test-only flag, batch entry 0) makes its
    bounded wait run out, the later slices scan normally without clearing the
    word, and both SS_SYNC_CHECK and ss_check on the same launch report
    SS_ERR_TIMEOUT; the next call on the same context is correct."""
    b, L, d = 3, 512, 128
    inp = fwd_inputs(b, L, d, 16, "bf16", 12, DEV, gate=True)
    h = host_copy(inp)
    dims = ss.ss_dims(b, L, d, 16)
    flags = ss.SS_BF16 | ss.SS_DELTA_SOFTPLUS | ss.SS_SYNC_CHECK
    assert int(ss.lib().ss_fwd_chunk_len(ctypes.byref(ss.ss_dims(1, L, d, 16)), ss.SS_BF16)) > 0  # slices are chunked
    need = int(ss.lib().ss_fwd_host_workspace_bytes(ctypes.byref(dims), flags, 1))
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    y = torch.empty_like(h["u"]).pin_memory()
    stream = torch.cuda.current_stream().cuda_stream
    launch = ss.ss_launch(stream, ws.data_ptr(), need, 2000, 0)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    rc = ss.lib().ss_fwd_host(p(h["u"]), p(h["delta"]), p(inp["delta_bias"]), p(inp["A"]), p(h["B"]), p(h["C"]),
                              p(inp["D"]), p(h["z"]), p(y), None, flags | ss.SS_TEST_DROP_CARRY,
                              ctypes.byref(dims), ctypes.byref(launch), 1)
    assert rc == ss.SS_ERR_TIMEOUT
    assert ss.lib().ss_check(ctypes.byref(launch)) == ss.SS_ERR_TIMEOUT
    rc = ss.lib().ss_fwd_host(p(h["u"]), p(h["delta"]), p(inp["delta_bias"]), p(inp["A"]), p(h["B"]), p(h["C"]),
                              p(inp["D"]), p(h["z"]), p(y), None, flags, ctypes.byref(dims), ctypes.byref(launch), 1)
    assert rc == ss.SS_OK
    y_ref, _ = device_slices(inp, 1)
    assert torch.equal(y, y_ref)
