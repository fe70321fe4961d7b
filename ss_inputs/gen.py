"""Seeded random draws for the selective-scan workloads (torch generators).

Every tensor is drawn from a torch.Generator seeded from (seed, tensor tag),
so the same call on the same device type gives the same values.  Large
workloads are drawn directly on the GPU in slices (no host staging); the CPU
oracle then receives the exact values of a sample of channels copied back.
"""
import math

import numpy as np
import torch

_TAGS = {"u": 1, "delta": 2, "z": 3, "B": 4, "C": 5, "bias": 6, "D": 7, "A": 8, "state": 9,
         "dy": 10, "dlast": 11, "conv_w": 12, "conv_b": 13, "hidden": 14, "w_in_x": 15,
         "w_in_z": 16, "w_x_dt": 17, "w_x_B": 18, "w_x_C": 19, "w_dt": 20, "w_out": 21,
         "ssd_x": 22, "ssd_dt": 23, "ssd_B": 24, "ssd_C": 25, "ssd_A": 26}
_SLICE = 1 << 26  # elements drawn per slice when filling a large tensor


def _gen(device, seed, tag):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000003 + _TAGS[tag])
    return g


def _normal(shape, std, dtype, device, seed, tag):
    """N(0, std^2) rounded once to dtype, drawn in fp32 slices."""
    g = _gen(device, seed, tag)
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, _SLICE):
        e = min(n, s + _SLICE)
        tmp = torch.randn(e - s, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            tmp.mul_(std)
        flat[s:e].copy_(tmp)
    return out


def _torch_dtype(name):
    return {"fp32": torch.float32, "bf16": torch.bfloat16}[name]


def delta_bias_init(d, seed, device="cpu", lo=1e-3, hi=1e-1):
    """bias = softplus^-1(Δ0) with Δ0 log-uniform in [lo, hi]; fp32 [d]."""
    g = _gen(device, seed, "bias")
    r = torch.rand(d, generator=g, device=device, dtype=torch.float64)
    d0 = torch.exp(math.log(lo) + r * (math.log(hi) - math.log(lo)))
    return torch.log(torch.expm1(d0)).to(torch.float32)


def structured_A(d, N, device="cpu"):
    """A[d, n] = -(n + 1), fp32 [d, N]."""
    return (-(torch.arange(N, dtype=torch.float32, device=device) + 1.0)).repeat(d, 1).contiguous()


def general_A(d, N, seed, device="cpu"):
    """A[d, n] = -(n + 1) * (1 + 0.25 * U[0,1)): negative, but off the
    a_d * (n + 1) ladder, so the general-A code path is exercised."""
    g = _gen(device, seed, "A")
    r = torch.rand(d, N, generator=g, device=device, dtype=torch.float32)
    return (structured_A(d, N, device) * (1.0 + 0.25 * r)).contiguous()


def fwd_inputs(batch, seqlen, d_inner, d_state=16, dtype="bf16", seed=0, device="cpu",
               gate=True, D_kind="ones", bias=True, A_kind="structured", delta_std=0.5):
    """Inputs of one ss_fwd call as a dict of torch tensors on `device`.

    u, delta, z : [batch, seqlen, d_inner] in `dtype`
    B, C        : [batch, seqlen, d_state] in `dtype`
    A           : [d_inner, d_state] fp32; D, delta_bias : [d_inner] fp32
    """
    dt = _torch_dtype(dtype)
    shp = (batch, seqlen, d_inner)
    out = {
        "u": _normal(shp, 1.0, dt, device, seed, "u"),
        "delta": _normal(shp, delta_std, dt, device, seed, "delta"),
        "z": _normal(shp, 1.0, dt, device, seed, "z") if gate else None,
        "B": _normal((batch, seqlen, d_state), 1.0, dt, device, seed, "B"),
        "C": _normal((batch, seqlen, d_state), 1.0, dt, device, seed, "C"),
    }
    out["A"] = (structured_A(d_inner, d_state, device) if A_kind == "structured"
                else general_A(d_inner, d_state, seed, device))
    if D_kind == "ones":
        out["D"] = torch.ones(d_inner, dtype=torch.float32, device=device)
    elif D_kind == "normal":
        out["D"] = _normal((d_inner,), 1.0, torch.float32, device, seed, "D")
    else:
        out["D"] = None
    out["delta_bias"] = delta_bias_init(d_inner, seed, "cpu").to(device) if bias else None
    return out


def bwd_upstream(batch, seqlen, d_inner, d_state=16, dtype="bf16", seed=0, device="cpu",
                 dlast=True):
    """Upstream gradients of one backward call: dy [batch, seqlen, d_inner] in
    `dtype` and dlast_state [batch, d_inner, d_state] fp32 (or None), N(0, 1)."""
    dy = _normal((batch, seqlen, d_inner), 1.0, _torch_dtype(dtype), device, seed, "dy")
    dl = _normal((batch, d_inner, d_state), 1.0, torch.float32, device, seed, "dlast") if dlast else None
    return dy, dl


def conv_params(d_inner, seed=0, device="cpu", bias="zero", width=4):
    """Weights of the causal conv1d prologue: conv_w [d_inner, width] fp32 drawn
    Kaiming-normal for a depthwise kernel (std sqrt(2 / width)), conv_b zero
    (the deep-dive's initialisation, §3.3) or N(0, 0.1^2) with bias="normal"."""
    w = _normal((d_inner, width), math.sqrt(2.0 / width), torch.float32, device, seed, "conv_w")
    if bias == "zero":
        b = torch.zeros(d_inner, dtype=torch.float32, device=device)
    elif bias == "normal":
        b = _normal((d_inner,), 0.1, torch.float32, device, seed, "conv_b")
    else:
        b = None
    return w, b


def block_inputs(batch, seqlen, d_model, d_state=16, seed=0, device="cpu", expand=2):
    """One Mamba block's input and random-init weights (the block's interface:
    d_inner = expand · d_model, d_conv = 4; dt_rank = ceil(d_model / 16)).
    hidden ~ N(0, 1) bf16; projection matrices N(0, 1/fan_in) bf16; conv taps
    Kaiming-normal, conv bias 0; dt_bias as delta_bias_init; A = -(n+1); D = 1.
    Returns (hidden, weights dict named as ss_block_weights' fields)."""
    d_inner = expand * d_model
    rank = -(-d_model // 16)
    bf = torch.bfloat16

    def mat(tag, rows, cols):
        return _normal((rows, cols), 1.0 / math.sqrt(cols), bf, device, seed, tag)

    w = {
        "in_proj_x": mat("w_in_x", d_inner, d_model),
        "in_proj_z": mat("w_in_z", d_inner, d_model),
        "x_proj_dt": mat("w_x_dt", rank, d_inner),
        "x_proj_B": mat("w_x_B", d_state, d_inner),
        "x_proj_C": mat("w_x_C", d_state, d_inner),
        "dt_proj": mat("w_dt", d_inner, rank),
        "out_proj": mat("w_out", d_model, d_inner),
        "dt_bias": delta_bias_init(d_inner, seed, "cpu").to(device),
        "A": structured_A(d_inner, d_state, device),
        "D": torch.ones(d_inner, dtype=torch.float32, device=device),
    }
    w["conv_w"], w["conv_b"] = conv_params(d_inner, seed, device)
    hidden = _normal((batch, seqlen, d_model), 1.0, bf, device, seed, "hidden")
    return hidden, w


def ssd_inputs(batch, seqlen, nheads, d_state=128, headdim=64, seed=0, device="cpu"):
    """Inputs of the multi-head scalar-decay scan (Mamba-2 SSD model): x ~ N(0,1)
    [batch, L, nheads, headdim] bf16; dt ~ N(0, 0.5^2) [batch, L, nheads] bf16;
    B, C ~ N(0,1) [batch, L, d_state] bf16 (one group); A_h = -U[1, 16] (one
    negative decay rate per head); dt_bias as delta_bias_init; D = 1."""
    bf = torch.bfloat16
    g = _gen("cpu", seed, "ssd_A")
    A = -(1.0 + 15.0 * torch.rand(nheads, generator=g, dtype=torch.float32)).to(device)
    return {
        "x": _normal((batch, seqlen, nheads, headdim), 1.0, bf, device, seed, "ssd_x"),
        "dt": _normal((batch, seqlen, nheads), 0.5, bf, device, seed, "ssd_dt"),
        "B": _normal((batch, seqlen, d_state), 1.0, bf, device, seed, "ssd_B"),
        "C": _normal((batch, seqlen, d_state), 1.0, bf, device, seed, "ssd_C"),
        "A": A,
        "dt_bias": delta_bias_init(nheads, seed, "cpu").to(device),
        "D": torch.ones(nheads, dtype=torch.float32, device=device),
    }


def step_inputs(batch, d_inner, d_state=16, dtype="bf16", seed=0, device="cpu", gate=True,
                bias=True, A_kind="structured"):
    """One decode step's inputs: u, delta, z [batch, d_inner]; B, C [batch, d_state];
    A, D, delta_bias as in fwd_inputs; state [batch, d_inner, d_state] fp32 ~ N(0, 1)."""
    dt = _torch_dtype(dtype)
    out = {
        "u": _normal((batch, d_inner), 1.0, dt, device, seed, "u"),
        "delta": _normal((batch, d_inner), 0.5, dt, device, seed, "delta"),
        "z": _normal((batch, d_inner), 1.0, dt, device, seed, "z") if gate else None,
        "B": _normal((batch, d_state), 1.0, dt, device, seed, "B"),
        "C": _normal((batch, d_state), 1.0, dt, device, seed, "C"),
        "state": _normal((batch, d_inner, d_state), 1.0, torch.float32, device, seed, "state"),
    }
    out["A"] = (structured_A(d_inner, d_state, device) if A_kind == "structured"
                else general_A(d_inner, d_state, seed, device))
    out["D"] = torch.ones(d_inner, dtype=torch.float32, device=device)
    out["delta_bias"] = delta_bias_init(d_inner, seed, "cpu").to(device) if bias else None
    return out


def step_sequence_inputs(steps, batch, d_inner, d_state=16, dtype="bf16", seed=0,
                         device="cpu", gate=True):
    """Per-step inputs for `steps` successive decode steps, stacked on a leading
    axis: u, delta, z [steps, batch, d_inner]; B, C [steps, batch, d_state]."""
    dt = _torch_dtype(dtype)
    return {
        "u": _normal((steps, batch, d_inner), 1.0, dt, device, seed, "u"),
        "delta": _normal((steps, batch, d_inner), 0.5, dt, device, seed, "delta"),
        "z": _normal((steps, batch, d_inner), 1.0, dt, device, seed, "z") if gate else None,
        "B": _normal((steps, batch, d_state), 1.0, dt, device, seed, "B"),
        "C": _normal((steps, batch, d_state), 1.0, dt, device, seed, "C"),
    }


def to_f64(t):
    """Exact float64 numpy copy of a tensor (None passes through)."""
    if t is None:
        return None
    return t.detach().to("cpu").to(torch.float64).numpy()


def sample_channels(batch, d_inner, count, seed):
    """A seeded sample of distinct (b, channel) pairs, always including the
    first and last channel of the first and last batch entry."""
    rng = np.random.default_rng(seed + 777)
    total = batch * d_inner
    count = min(count, total)
    picks = set([0, total - 1, d_inner - 1, (batch - 1) * d_inner])
    picks = set(p for p in picks if 0 <= p < total)
    while len(picks) < count:
        picks.add(int(rng.integers(0, total)))
    flat = sorted(picks)[:max(count, len(picks))]
    return [(p // d_inner, p % d_inner) for p in flat]
