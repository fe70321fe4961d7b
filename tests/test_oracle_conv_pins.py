"""Pins of the conv1d + SiLU prologue oracle (oracle.conv_silu).

The causal depthwise convolution of width 4 ("Understanding Mamba and
Selective State Space Models (SSMs)" §3.3) is checked against the library
routine torch.nn.functional.conv1d (fp64, groups = channels, left padding
W - 1, then the first L outputs), which fixes the weight orientation (w[:, W-1]
multiplies the current token) and the causal zero padding; SiLU against
torch.nn.functional.silu.  Special cases pin the index direction by hand.
"""
import numpy as np
import pytest
import torch

import oracle


def library_conv_silu(x, w, bias):
    xt = torch.from_numpy(x).permute(0, 2, 1)              # [b, d, L]
    d, W = w.shape
    out = torch.nn.functional.conv1d(xt, torch.from_numpy(w)[:, None, :],
                                     torch.from_numpy(bias) if bias is not None else None,
                                     padding=W - 1, groups=d)[..., : x.shape[1]]
    return torch.nn.functional.silu(out).permute(0, 2, 1).numpy()


@pytest.mark.parametrize("shape,W", [((2, 37, 5), 4), ((1, 3, 4), 4), ((3, 16, 7), 2), ((1, 9, 3), 1)])
def test_matches_library_conv(shape, W):
    rng = np.random.default_rng(sum(shape) + W)
    x = rng.normal(size=shape)
    w = rng.normal(size=(shape[2], W))
    bias = rng.normal(size=shape[2])
    for b in (bias, None):
        got = oracle.conv_silu(x, w, b)
        np.testing.assert_allclose(got, library_conv_silu(x, w, b), rtol=1e-12, atol=1e-13)


def silu(v):
    return v / (1.0 + np.exp(-v))


def test_current_token_only_is_silu_of_x():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(2, 10, 3))
    w = np.zeros((3, 4))
    w[:, 3] = 1.0
    np.testing.assert_allclose(oracle.conv_silu(x, w), silu(x), rtol=1e-14, atol=0)


def test_oldest_tap_is_a_causal_shift_by_three():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(1, 12, 2))
    w = np.zeros((2, 4))
    w[:, 0] = 1.0
    u = oracle.conv_silu(x, w)
    np.testing.assert_allclose(u[:, 3:], silu(x[:, :-3]), rtol=1e-14, atol=0)
    np.testing.assert_array_equal(u[:, :3], 0.0)          # silu(0) on the zero padding


def test_causality():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(1, 20, 4))
    w = rng.normal(size=(4, 4))
    u0 = oracle.conv_silu(x, w)
    x2 = x.copy()
    x2[:, 11] += 1.0
    u1 = oracle.conv_silu(x2, w)
    np.testing.assert_array_equal(u0[:, :11], u1[:, :11])
    assert np.all(np.abs(u0[:, 11:15] - u1[:, 11:15]) > 0)
    np.testing.assert_array_equal(u0[:, 15:], u1[:, 15:])


# --------------------------------------------------------- block composition
from oracle.block import block_fwd, round_bf16  # noqa: E402


def block_weights(rng, d_model=12, d_inner=24, N=16, rank=3):
    return {
        "in_proj_x": rng.normal(size=(d_inner, d_model)) * 0.3,
        "in_proj_z": rng.normal(size=(d_inner, d_model)) * 0.3,
        "conv_w": rng.normal(size=(d_inner, 4)) * 0.7,
        "conv_b": np.zeros(d_inner),
        "x_proj_dt": rng.normal(size=(rank, d_inner)) * 0.2,
        "x_proj_B": rng.normal(size=(N, d_inner)) * 0.2,
        "x_proj_C": rng.normal(size=(N, d_inner)) * 0.2,
        "dt_proj": rng.normal(size=(d_inner, rank)) * 0.3,
        "dt_bias": rng.normal(size=d_inner) * 0.3 - 2.0,
        "A": -np.tile(np.arange(1, N + 1, dtype=np.float64), (d_inner, 1)),
        "D": rng.normal(size=d_inner),
        "out_proj": rng.normal(size=(d_model, d_inner)) * 0.2,
    }


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(5)
    a = rng.normal(size=4096) * 10.0 ** rng.integers(-6, 6, size=4096)
    ref = torch.from_numpy(a).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(round_bf16(a), ref)


def test_block_zero_input_gives_zero_output():
    """With zero conv bias, zero hidden makes x = u = 0, so every SSM input
    term vanishes and out = 0 exactly."""
    rng = np.random.default_rng(6)
    w = block_weights(rng)
    out = block_fwd(np.zeros((2, 9, 12)), w, store_bf16=False)
    np.testing.assert_array_equal(out, 0.0)


def test_block_is_linear_in_out_proj_and_shape_preserving():
    rng = np.random.default_rng(7)
    w = block_weights(rng)
    h = rng.normal(size=(2, 10, 12))
    o1 = block_fwd(h, w, store_bf16=False)
    assert o1.shape == h.shape                       # README: y.shape == x.shape
    w2 = dict(w)
    w2["out_proj"] = 2.5 * w["out_proj"]
    np.testing.assert_allclose(block_fwd(h, w2, store_bf16=False), 2.5 * o1, rtol=1e-12, atol=1e-14)
