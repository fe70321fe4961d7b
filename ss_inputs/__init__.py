"""Seeded synthetic inputs for the selective scan (shared by tests, bench, oracle checks).

This module holds the workload recipes and random draws only -- none of the
scan's arithmetic.  Both the CUDA path and the CPU oracle consume what it
produces; the oracle receives the exact values (bf16 widened to float64).

Recipe (the Mamba-shaped workloads of the pages: d_inner = 2 * d_model of the
130M and 2.8B checkpoints listed in the mamba README's "Pretrained Models"
table, d_state = 16 as in the README usage example and the deep-dive article
§2.2 third cut):
  u, z, B, C    ~ N(0, 1)
  delta_raw     ~ N(0, 0.5^2)                   (standard deviation 0.5)
  delta_bias[d] = softplus^-1(exp(U[ln 1e-3, ln 1e-1]))  (the "targeted range
                  of Δ set through the bias" of the README's Initialization
                  note; the range itself is the workload's)
  A[d, n]       = -(n + 1)                      (real, negative, diagonal:
                  A = -exp(A_log) of the deep-dive §4.3, S4D-real values)
  D             = 1, or N(0, 1) for the 2.8B-shaped layer
  B, C          : [batch, L, N], one group shared by all channels
  I/O dtype     : fp32 for the tiny case, bf16 otherwise; A, D, bias fp32.
  Backward upstream gradients: dy ~ N(0, 1) in the I/O dtype and
  dlast_state ~ N(0, 1) fp32.
  Conv prologue (deep-dive §3.3): conv_w [d, 4] Kaiming-normal, std sqrt(2/4);
  conv_b = 0 (or N(0, 0.1^2) where a test covers the bias); x takes u's recipe.
  Mamba block (README Usage > Mamba: expand 2, d_conv 4): hidden ~ N(0, 1) bf16,
  projection matrices N(0, 1/fan_in) bf16, dt_rank = ceil(d_model / 16).
  Mamba-2 SSD scan (model-architecture page: headdim 64, d_state 128, one
  group): x, B, C ~ N(0, 1) bf16, dt ~ N(0, 0.5^2), A_h = -U[1, 16], D = 1.
"""
from .configs import CONFIGS, FwdConfig, StepConfig, get_config
from .gen import (block_inputs, ssd_inputs, bwd_upstream, conv_params, fwd_inputs, step_inputs, step_sequence_inputs, general_A,
                  to_f64, sample_channels)

__all__ = ["CONFIGS", "FwdConfig", "StepConfig", "get_config", "fwd_inputs", "bwd_upstream", "conv_params",
           "block_inputs", "ssd_inputs",
           "step_inputs", "step_sequence_inputs", "general_A", "to_f64",
           "sample_channels"]
