"""Named decode workloads (shapes, window, state format, input recipe knobs)."""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    B: int                 # sequences
    H: int                 # heads per sequence
    D: int                 # d_k = d_v
    T: int                 # decode steps
    W: int                 # window length (tokens per low-bit freeze)
    r: int = 0             # compensator pairs per head
    gate: str = "scalar"   # "scalar" (GDN) or "diag" (KDA, per key channel)
    fmt: str = "int8"      # "int8" (row scales) or "int4_g32" (group-32 scales)
    act: str = "bf16"      # dtype of q, k, v, o
    buf: str = "bf16"      # dtype of buffered write vectors u
    outliers: bool = True  # 2% of key and value channels scaled x20
    warmup: int = 512      # fp32 recurrence tokens that make the initial state (0: zero state)
    seed: int = 0
    smooth: bool = False   # residual smoothing at every quantization
    comp_rule: str = "columns"  # compensator tokens: "columns" or "power"

    @property
    def heads(self) -> int:
        return self.B * self.H

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # tiny parity case: zero initial state, fp32 activations, no outliers
    "gdn-tiny": Workload("gdn-tiny", B=1, H=2, D=16, T=64, W=8, act="f32", buf="f32",
                         outliers=False, warmup=0, seed=1001),
    # mid batch, L2-resident
    "gdn-mid": Workload("gdn-mid", B=64, H=16, D=128, T=1024, W=64, seed=1002),
    # KDA: per-key-channel gate, 4 compensator pairs
    "kda": Workload("kda", B=256, H=32, D=128, T=512, W=64, r=4, gate="diag", seed=1003),
    # long decode over a packed int4 state
    "gdn-long-int4": Workload("gdn-long-int4", B=8, H=16, D=128, T=8192, W=128, fmt="int4_g32",
                              seed=1004),
    # serving-scale batch (the throughput workload)
    "gdn-serving": Workload("gdn-serving", B=1024, H=32, D=128, T=256, W=64, seed=1005),
    # prompt prefill before decode: T = prompt length L, one chunkwise launch over all of it
    "gdn-prefill": Workload("gdn-prefill", B=8, H=32, D=128, T=4096, W=64, warmup=0,
                            seed=1006),
    # the same prompt batch with the per-key-channel gate
    "kda-prefill": Workload("kda-prefill", B=8, H=32, D=128, T=4096, W=64, gate="diag",
                            warmup=0, seed=1007),
}


def get(name: str) -> Workload:
    try:
        return WORKLOADS[name]
    except KeyError:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(WORKLOADS)}") from None
