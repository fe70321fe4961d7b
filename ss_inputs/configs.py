"""The five workloads the scan is checked and measured on (shapes and recipes only)."""
from dataclasses import dataclass


@dataclass(frozen=True)
class FwdConfig:
    name: str
    batch: int
    seqlen: int
    d_inner: int
    d_state: int
    dtype: str          # "fp32" or "bf16" for u, delta, z, B, C, y
    D_kind: str         # "ones" or "normal"
    gate: bool
    seed: int
    description: str

    @property
    def ch_ts(self) -> int:
        """Channel-timesteps: one (batch, t, channel) element of u."""
        return self.batch * self.seqlen * self.d_inner

    def compulsory_bytes(self, conv=False) -> int:
        """Bytes every forward pass must move at least once: u (or, with the
        conv prologue, x), delta_raw, z read and y written (one element each
        per channel-timestep), B and C read, A/D/bias (and conv weights) read
        and the final state written."""
        e = 4 if self.dtype == "fp32" else 2
        per_chts = (4 if self.gate else 3) * e
        bc = 2 * self.batch * self.seqlen * self.d_state * e
        params = self.d_inner * (self.d_state * 4 + 8 + (20 if conv else 0))
        state = self.batch * self.d_inner * self.d_state * 4
        return self.ch_ts * per_chts + bc + params + state

    def bwd_compulsory_bytes(self) -> int:
        """Bytes every backward pass must move at least once: u, delta_raw, z and
        dy read, du, ddelta and dz written (one element each per
        channel-timestep); B and C read and dB, dC written in fp32; A/D/bias
        read, dA/dD/dbias written; dlast_state read."""
        e = 4 if self.dtype == "fp32" else 2
        per_chts = (7 if self.gate else 5) * e
        bc = self.batch * self.seqlen * self.d_state * (2 * e + 2 * 4)
        params = 2 * self.d_inner * (self.d_state * 4 + 8)
        state = self.batch * self.d_inner * self.d_state * 4
        return self.ch_ts * per_chts + bc + params + state


@dataclass(frozen=True)
class StepConfig:
    name: str
    batch: int
    d_inner: int
    d_state: int
    steps: int
    dtype: str
    gate: bool
    seed: int
    description: str

    def compulsory_bytes_per_step(self) -> int:
        """State read + written in fp32, u/delta/z read and y written, B/C read,
        parameters read."""
        e = 4 if self.dtype == "fp32" else 2
        state = 2 * self.batch * self.d_inner * self.d_state * 4
        io = (4 if self.gate else 3) * self.batch * self.d_inner * e
        bc = 2 * self.batch * self.d_state * e
        params = self.d_inner * (self.d_state * 4 + 8)
        return state + io + bc + params


CONFIGS = {
    "tiny_fp32": FwdConfig("tiny_fp32", 1, 64, 32, 16, "fp32", "ones", True, 0,
                           "tiny fp32 scan: batch 1, L 64, d_inner 32, N 16"),
    "mamba130m": FwdConfig("mamba130m", 8, 2048, 1536, 16, "bf16", "ones", True, 1,
                           "Mamba-130M-shaped layer: batch 8, L 2048, d_inner 1536, N 16"),
    "mamba2p8b": FwdConfig("mamba2p8b", 4, 8192, 5120, 16, "bf16", "normal", True, 2,
                           "Mamba-2.8B-shaped layer: batch 4, L 8192, d_inner 5120, N 16"),
    "million": FwdConfig("million", 1, 1 << 20, 1536, 16, "bf16", "ones", True, 3,
                         "million-token scan: batch 1, L 1048576, d_inner 1536, N 16"),
    "million_profile": FwdConfig("million_profile", 1, 1 << 17, 1536, 16, "bf16", "ones", True, 3,
                                 "reduced million-token scan for profiling: batch 1, L 131072, "
                                 "d_inner 1536, N 16"),
    "decode": StepConfig("decode", 256, 5120, 16, 1000, "bf16", True, 4,
                         "decode step: batch 256, d_inner 5120, N 16, 1000 steps"),
}


def get_config(name: str):
    return CONFIGS[name]
