"""GPU parity of ss_block_fwd (the Mamba block's inner forward path) against
oracle.block_fwd, which composes fp64 matmuls with the pinned conv and scan
oracles and rounds to bf16 at the points where the layer stores bf16.  Bound:
max|out - out_ref| <= 2e-2 · max|out_ref| (the scan's bf16 bound; the
projections accumulate in fp32, so their own error is far smaller)."""
import numpy as np
import pytest
import torch

import selective_state_space_37_b200 as ss
from gpu_util import rel_max_err
from oracle.block import block_fwd
from ss_inputs import block_inputs, to_f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def np_weights(w):
    return {k: (None if v is None else to_f64(v)) for k, v in w.items()}


@pytest.mark.parametrize("shape", [(2, 64, 64), (2, 300, 256), (1, 97, 128)])
def test_block_matches_oracle(shape):
    b, L, dm = shape
    hidden, w = block_inputs(b, L, dm, seed=400 + L + dm, device=DEV)
    out = ss.ss_block_fwd(hidden, w)
    torch.cuda.synchronize()
    ref = block_fwd(to_f64(hidden), np_weights(w), store_bf16=True)
    assert out.shape == hidden.shape
    assert rel_max_err(to_f64(out), ref) <= 2e-2


def test_block_rejects_bad_sizes():
    hidden, w = block_inputs(1, 16, 64, seed=1, device=DEV)
    w2 = dict(w)
    w2["in_proj_x"] = torch.empty((130, 64), dtype=torch.bfloat16, device=DEV)   # d_inner mismatch
    with pytest.raises(ValueError):
        ss.ss_block_fwd(hidden, w2)
    st = ss._binding._block_struct(w, DEV)
    st.d_inner = 100                                                          # not a multiple of 8
    assert int(ss.lib().ss_block_scratch_bytes(st, 1, 16)) == 0


def test_block_full_size_prefix():
    """The Mamba-2.8B-shaped block (batch 4, L 8192, d_model 2560) on the whole
    input, as the bench times it; the block is causal, so the oracle on the
    first 256 tokens of two batch rows gives those rows' exact outputs."""
    b, L, dm = 4, 8192, 2560
    hidden, w = block_inputs(b, L, dm, seed=9, device=DEV)
    out = ss.ss_block_fwd(hidden, w)
    torch.cuda.synchronize()
    wn = np_weights(w)
    T = 256
    for bi in (0, 3):
        ref = block_fwd(to_f64(hidden[bi:bi + 1, :T]), wn, store_bf16=True)
        assert rel_max_err(to_f64(out[bi:bi + 1, :T]), ref) <= 2e-2, bi
    del hidden, w, out
    torch.cuda.empty_cache()
