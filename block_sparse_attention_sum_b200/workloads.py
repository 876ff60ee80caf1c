"""Named synthetic workloads (shapes, seeds, tau, sink) for tests and the bench.

Each workload is the operator call the Sol-Attn pages measure, with seeded synthetic inputs in
place of model activations:

* ``tiny``      B=1, H=2,  N=1024, i.i.d. N(0,1), tau = 1.0, no sink.
* ``wan``       B=1, H=12, N=14040 = 9x30x52 latent grid (Wan 2.1 1.3B, 832x480x33 frames, the
                stable-diffusion.cpp Sol-Attn validation run), last 64-token block partial, tau = 1.0.
* ``s32k_*``    B=1, H=32, N=32768 = 16x32x64, tau tuned to 80 / 85 / 90 % non-exact
                (query-block, key-block) pairs, with a 512-token exact text-prefix sink
                (Sol-Attn README, "Exact KV sink"; Sol-Attn2 draft, "FP8 Kernel Performance").
* ``s64k``      B=1, H=32, N=65536 = 16x64x64, tau tuned to 90 %.
* ``s128k``     B=1, H=32, N=131072 = 32x64x64, tau tuned to 90 %.
* ``sol2_64k``  the ``s64k`` inputs through the Sol-Attn2 complementary-tail entry point.

Tau values for the tuned workloads are read from ``tuned_tau.json`` beside this file; that file is
written by the oracle's tau tuner and holds only input settings, not expected outputs.
"""
from __future__ import annotations

import json
import os
from dataclasses import dataclass

from .inputs import GridSpec, grf_qkv, iid_qkv

_HERE = os.path.dirname(os.path.abspath(__file__))
TUNED_TAU_PATH = os.path.join(_HERE, "tuned_tau.json")


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    kind: str                 # "iid" or "grf"
    seed: int
    grid: GridSpec | None
    tau: float | None         # None: read the tuned value
    target_sparsity: float | None
    sink_start: int = -1      # < 0 with sink_tokens > 0 means a suffix sink
    sink_tokens: int = 0      # <= 0 means no sink
    entry: str = "sol_attn"   # "sol_attn" or "sol_attn2"

    def resolved_tau(self) -> float:
        if self.tau is not None:
            return self.tau
        tuned = load_tuned_tau()
        key = self.input_key()
        if key not in tuned:
            raise KeyError(f"no tuned tau for workload {self.name!r} (key {key!r}); run oracle/tune_tau.py")
        return float(tuned[key]["tau"])

    def input_key(self) -> str:
        """Workloads that share inputs and target share one tuned tau (s64k and sol2_64k)."""
        t = "" if self.target_sparsity is None else f"@{self.target_sparsity:.2f}"
        sink = f"+sink{self.sink_start}:{self.sink_tokens}" if self.sink_tokens > 0 else ""
        return f"{self.kind}{self.B}x{self.N}x{self.H}s{self.seed}{sink}{t}"

    def make_inputs(self, device="cpu"):
        if self.kind == "iid":
            return iid_qkv(self.B, self.N, self.H, seed=self.seed, device=device)
        return grf_qkv(self.B, self.H, self.grid, seed_base=self.seed, device=device)


def load_tuned_tau() -> dict:
    if not os.path.exists(TUNED_TAU_PATH):
        return {}
    with open(TUNED_TAU_PATH) as f:
        return json.load(f)


_G32 = GridSpec(16, 32, 64)
_G64 = GridSpec(16, 64, 64)
_G128 = GridSpec(32, 64, 64)

WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 1, 2, 1024, "iid", 0, None, 1.0, None),
        Workload("wan", 1, 12, 14040, "grf", 1003, GridSpec(9, 30, 52), 1.0, None),
        Workload("s32k_80", 1, 32, 32768, "grf", 1006, _G32, None, 0.80, 0, 512),
        Workload("s32k_85", 1, 32, 32768, "grf", 1006, _G32, None, 0.85, 0, 512),
        Workload("s32k_90", 1, 32, 32768, "grf", 1006, _G32, None, 0.90, 0, 512),
        Workload("s64k", 1, 32, 65536, "grf", 1009, _G64, None, 0.90),
        Workload("s128k", 1, 32, 131072, "grf", 1012, _G128, None, 0.90),
        Workload("sol2_64k", 1, 32, 65536, "grf", 1009, _G64, None, 0.90, entry="sol_attn2"),
    ]
}
