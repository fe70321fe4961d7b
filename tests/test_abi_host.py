"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, and rejects bad arguments before touching a GPU (runs without one)."""
import ctypes
import os
import re

import pytest

import selective_state_space_37_b200 as ss
from selective_state_space_37_b200 import _binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "selscan.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(ss_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def L():
    return ss.lib()


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert set(names) == set(bd.EXPORTED), names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version(L):
    assert ss.status_string(ss.SS_OK) == "SS_OK"
    assert ss.status_string(ss.SS_ERR_TIMEOUT) == "SS_ERR_TIMEOUT"
    assert ss.status_string(12345) == "SS_ERR_UNKNOWN"
    assert L.ss_version() == 10000


def _fake(addr):
    return ctypes.c_void_p(addr)


def _call_fwd(L, dims, launch, u=0x10000, dl=0x20000, A=0x30000, B=0x40000, C=0x50000,
              y=0x60000, D=None, z=None, bias=None, st=None, flags=ss.SS_BF16):
    p = lambda a: None if a is None else _fake(a)
    return L.ss_fwd(p(u), p(dl), p(bias), p(A), p(B), p(C), p(D), p(z), p(y), p(st), flags,
                    None if dims is None else ctypes.byref(dims),
                    None if launch is None else ctypes.byref(launch))


def test_fwd_rejects_bad_arguments(L):
    ok_dims = ss.ss_dims(2, 64, 128, 16)
    launch = ss.ss_launch(None, None, 0, 0, 0)
    assert _call_fwd(L, None, launch) == ss.SS_ERR_INVALID_ARG
    assert _call_fwd(L, ok_dims, None) == ss.SS_ERR_INVALID_ARG
    assert _call_fwd(L, ss.ss_dims(-1, 64, 128, 16), launch) == ss.SS_ERR_INVALID_ARG
    assert _call_fwd(L, ss.ss_dims(2, -5, 128, 16), launch) == ss.SS_ERR_INVALID_ARG
    assert _call_fwd(L, ss.ss_dims(2, 64, 128, 0), launch) == ss.SS_ERR_INVALID_ARG
    assert _call_fwd(L, ss.ss_dims(2, 64, 128, 32), launch) == ss.SS_ERR_UNSUPPORTED
    assert _call_fwd(L, ss.ss_dims(2, 64, 128, 64), launch) == ss.SS_ERR_UNSUPPORTED
    assert _call_fwd(L, ss.ss_dims(1 << 31, 64, 128, 16), launch) == ss.SS_ERR_INVALID_ARG
    assert _call_fwd(L, ss.ss_dims(1 << 20, 1 << 30, 1 << 20, 16), launch) == ss.SS_ERR_INVALID_ARG
    # required pointers
    assert _call_fwd(L, ok_dims, launch, u=None) == ss.SS_ERR_INVALID_ARG
    assert _call_fwd(L, ok_dims, launch, C=None) == ss.SS_ERR_INVALID_ARG
    assert _call_fwd(L, ok_dims, launch, y=None) == ss.SS_ERR_INVALID_ARG
    # misalignment of a required or an optional pointer
    assert _call_fwd(L, ok_dims, launch, u=0x10002) == ss.SS_ERR_INVALID_ARG
    assert _call_fwd(L, ok_dims, launch, D=0x70004) == ss.SS_ERR_INVALID_ARG
    # unknown flag bits
    assert _call_fwd(L, ok_dims, launch, flags=1 << 12) == ss.SS_ERR_INVALID_ARG
    # missing or too small workspace
    assert _call_fwd(L, ok_dims, launch) == ss.SS_ERR_WORKSPACE
    small = ss.ss_launch(None, _fake(0x80000), 16, 0, 0)
    assert _call_fwd(L, ok_dims, small) == ss.SS_ERR_WORKSPACE
    mis = ss.ss_launch(None, _fake(0x80008), 1 << 20, 0, 0)
    assert _call_fwd(L, ok_dims, mis) == ss.SS_ERR_WORKSPACE
    # empty problems are no-ops and touch nothing
    assert _call_fwd(L, ss.ss_dims(0, 64, 128, 16), launch) == ss.SS_OK
    assert _call_fwd(L, ss.ss_dims(2, 64, 0, 16), launch) == ss.SS_OK


def test_step_rejects_bad_arguments(L):
    launch = ss.ss_launch(None, None, 0, 0, 0)
    f = lambda a: None if a is None else _fake(a)

    def call(dims, state=0x1000, u=0x2000, y=0x3000, flags=0):
        return L.ss_step(f(state), f(u), _fake(0x4000), _fake(0x5000), _fake(0x6000),
                         _fake(0x7000), None, None, f(y), None, flags,
                         None if dims is None else ctypes.byref(dims), ctypes.byref(launch))

    assert call(None) == ss.SS_ERR_INVALID_ARG
    assert call(ss.ss_dims(4, 0, 64, 8)) == ss.SS_ERR_UNSUPPORTED
    assert call(ss.ss_dims(4, 0, -1, 16)) == ss.SS_ERR_INVALID_ARG
    assert call(ss.ss_dims(4, 0, 64, 16), state=None) == ss.SS_ERR_INVALID_ARG
    assert call(ss.ss_dims(4, 0, 64, 16), y=0x3004) == ss.SS_ERR_INVALID_ARG
    assert call(ss.ss_dims(4, 0, 64, 16), flags=1 << 13) == ss.SS_ERR_INVALID_ARG
    assert call(ss.ss_dims(0, 0, 64, 16)) == ss.SS_OK


def test_workspace_layout(L):
    dims = ss.ss_dims(1, 1024, 256, 16)
    # 4 chunks of 256, 2 channel blocks: 256 B header, 32 B of status words
    # (rounded to 256), then 4 * 256 records of 48 floats.
    assert L.ss_fwd_workspace_bytes(ctypes.byref(dims), ss.SS_BF16, 256) == 512 + 4 * 256 * 48 * 4
    # a chunk length is rounded up to the 32-step tile
    assert (L.ss_fwd_workspace_bytes(ctypes.byref(dims), ss.SS_BF16, 250)
            == L.ss_fwd_workspace_bytes(ctypes.byref(dims), ss.SS_BF16, 256))
    # no chunking: the 256-byte header only
    assert L.ss_fwd_workspace_bytes(ctypes.byref(dims), ss.SS_BF16, 4096) == 256
    assert L.ss_fwd_workspace_bytes(ctypes.byref(ss.ss_dims(1, 0, 256, 16)), ss.SS_BF16, 0) == 256
    assert L.ss_fwd_workspace_bytes(ctypes.byref(ss.ss_dims(1, 8, 256, 32)), ss.SS_BF16, 0) == 0


def test_bwd_workspace_layout(L):
    """Checkpoints [b][nseg][d][16] and their Σ Δ [b][nseg][d], then records
    for min(16, nseg) time chunks (h_loc, g_loc [b][k][d][16], Σ Δ [b][k][d]),
    each region rounded up to 256 bytes."""
    al = lambda x: (x + 255) // 256 * 256

    def expect(b, L_, d):
        nseg = max(1, -(-L_ // 32))
        k = min(16, nseg)
        return (al(b * nseg * d * 64) + al(b * nseg * d * 4) + 2 * al(b * k * d * 64) + al(b * k * d * 4))

    for b, L_, d in ((1, 32, 64), (2, 1000, 130), (4, 8192, 5120), (3, 1, 10), (1, 0, 64)):
        got = L.ss_bwd_workspace_bytes(ctypes.byref(ss.ss_dims(b, L_, d, 16)), ss.SS_BF16)
        assert got == expect(b, L_, d), (b, L_, d)
    assert L.ss_bwd_workspace_bytes(ctypes.byref(ss.ss_dims(1, 8, 64, 32)), ss.SS_BF16) == 0


def test_auto_chunking_is_a_tile_multiple(L):
    for (b, l, d) in ((4, 8192, 5120), (8, 2048, 1536), (1, 1 << 20, 1536), (1, 64, 32)):
        dims = ss.ss_dims(b, l, d, 16)
        c = L.ss_fwd_chunk_len(ctypes.byref(dims), ss.SS_BF16)
        assert c == 0 or (c % 32 == 0 and 0 < c < l)
        assert L.ss_fwd_workspace_bytes(ctypes.byref(dims), ss.SS_BF16, 0) >= 256


def test_python_binding_checks_arguments():
    import torch
    u = torch.zeros(1, 4, 8)
    with pytest.raises(ValueError):
        ss.ss_fwd(u, u, torch.zeros(8, 16), torch.zeros(1, 4, 16), torch.zeros(1, 4, 16))
    with pytest.raises(ValueError):
        ss.ss_step(torch.zeros(1, 8, 16), torch.zeros(1, 8), torch.zeros(1, 8), torch.zeros(8, 16),
                   torch.zeros(1, 16), torch.zeros(1, 16))


def test_python_binding_checks_new_entry_points():
    """The host-buffer forward wants its parameters on a CUDA device; the
    backward, SSD and entering-state forward refuse CPU tensors before any
    library call (no GPU needed to check)."""
    import torch
    u = torch.zeros(1, 4, 8)
    A = torch.zeros(8, 16)
    B = torch.zeros(1, 4, 16)
    with pytest.raises(ValueError):
        ss.ss_fwd_host(u, u, A, B, B)                  # A on the CPU
    with pytest.raises(ValueError):
        ss.ss_bwd(u, u, A, B, B, u)                    # CPU tensors
    with pytest.raises(ValueError):
        ss.ss_fwd(u, u, A, B, B, initial_state=torch.zeros(1, 8, 16))
    with pytest.raises(ValueError):
        ss.ss_fwd_host(torch.zeros(1, 4), u, A, B, B)  # u not [batch, L, d_inner]


def test_host_and_ssd_workspace_sizes(L):
    """ss_fwd_host's staging is two slots of one slice's activations and
    states plus one slice's forward workspace; ss_ssd_fwd's workspace is a
    256-byte status header then segment records for min(8, chunks) segments."""
    al = lambda x: (x + 255) // 256 * 256
    dims = ss.ss_dims(3, 100, 64, 16)
    for rows in (1, 2, 3, 5):
        r = min(rows, 3)
        slot = 4 * al(r * 100 * 64 * 2) + 2 * al(r * 100 * 16 * 2) + al(r * 64 * 16 * 4)
        fwd = al(L.ss_fwd_workspace_bytes(ctypes.byref(ss.ss_dims(r, 100, 64, 16)), ss.SS_BF16, 0))
        assert L.ss_fwd_host_workspace_bytes(ctypes.byref(dims), ss.SS_BF16, rows) == 2 * slot + fwd
    assert L.ss_fwd_host_workspace_bytes(ctypes.byref(ss.ss_dims(0, 100, 64, 16)), ss.SS_BF16, 1) == 0
    for b, Lq, H, N in ((2, 1000, 3, 128), (1, 64, 2, 64), (4, 8192, 80, 128)):
        chunks = max(1, -(-Lq // 64))
        k = min(8, chunks)
        want = 256 + al(b * H * (k - 1) * 64 * N * 4) + al(b * H * k * 4)
        got = L.ss_ssd_fwd_workspace_bytes(ctypes.byref(ss.ss_ssd_dims(b, Lq, H, 64, N)), 0)
        assert got == want, (b, Lq, H, N)
    assert L.ss_ssd_fwd_workspace_bytes(ctypes.byref(ss.ss_ssd_dims(1, 64, 2, 32, 64)), 0) == 0


def test_missing_library_fails_loudly():
    """With the native library absent, the binding raises instead of falling
    back to any other implementation (checked in a fresh interpreter)."""
    import subprocess
    import sys
    code = ("import selective_state_space_37_b200 as ss\n"
            "try:\n"
            "    ss.lib()\n"
            "except RuntimeError as e:\n"
            "    print('raised', 'not found' in str(e))\n"
            "else:\n"
            "    print('loaded')\n")
    env = dict(os.environ, SELSCAN_LIB="/nonexistent/libselscan.so")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env,
                         cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))), timeout=300)
    assert out.stdout.strip() == "raised True", out.stdout + out.stderr
