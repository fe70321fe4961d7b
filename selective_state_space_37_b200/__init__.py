"""selective_state_space_37_b200 -- B200-native Mamba selective scan.

Python binding of libselscan (C ABI in include/selscan.h, CUDA kernels for
sm_100a in csrc/).  Three operations:

  ss_fwd   forward selective scan over a sequence, with optional final state;
  ss_step  one decode step on a carried fp32 state;
  ss_bwd   gradients of ss_fwd's inputs from the gradients of its outputs;
  ss_fwd_conv / ss_step_conv  the same with the causal conv1d + SiLU
           prologue fused in;
  ss_block_fwd  the Mamba block's inner forward path around the scan;
  ss_ssd_fwd    the multi-head scalar-decay scan (Mamba-2's SSD model);
  ss_fwd_host   ss_fwd on activations in host memory, batch slices'
                uploads, scans and downloads overlapped.

Build the library with ``python -m selective_state_space_37_b200.csrc.build``
(``__graft_entry__.build()`` does the same).
"""
from ._binding import (D_STATE, EXPORTED, LIB_PATH, SS_BF16, SS_DELTA_SOFTPLUS,
                       SS_ERR_CUDA, SS_ERR_INVALID_ARG, SS_ERR_TIMEOUT, SS_ERR_UNSUPPORTED,
                       SS_ERR_WORKSPACE, SS_FORCE_GENERAL_A, SS_OK, SS_SYNC_CHECK,
                       SS_TEST_DROP_CARRY, SelscanError, block_scratch_bytes, bwd_workspace_bytes,
                       fwd_chunk_len, ss_block_fwd, ss_block_weights, ss_ssd_dims, ss_ssd_fwd,
                       fwd_workspace_bytes, lib, ss_bwd, ss_check, ss_dims, ss_fwd, ss_fwd_conv,
                       ss_launch, ss_step, ss_step_conv, status_string, workspace_for,
                       ss_fwd_host, fwd_host_workspace_bytes, clear_workspaces)

__all__ = ["ss_fwd", "ss_fwd_host", "fwd_host_workspace_bytes", "ss_step", "ss_bwd", "ss_fwd_conv", "ss_step_conv", "ss_block_fwd", "ss_ssd_fwd",
           "block_scratch_bytes", "ss_block_weights", "ss_ssd_dims", "ss_check", "fwd_workspace_bytes", "fwd_chunk_len",
           "bwd_workspace_bytes",
           "status_string", "lib", "SelscanError", "ss_dims", "ss_launch", "workspace_for", "clear_workspaces",
           "D_STATE", "EXPORTED", "LIB_PATH", "SS_OK", "SS_ERR_INVALID_ARG",
           "SS_ERR_UNSUPPORTED", "SS_ERR_CUDA", "SS_ERR_TIMEOUT", "SS_ERR_WORKSPACE",
           "SS_BF16", "SS_DELTA_SOFTPLUS", "SS_SYNC_CHECK", "SS_FORCE_GENERAL_A",
           "SS_TEST_DROP_CARRY"]
