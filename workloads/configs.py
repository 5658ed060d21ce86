"""The five synthetic workloads of the hot path, with their sizes.

Each workload stands in for one operating point the KV-cache compression pages
describe:

* ``tiny``     - a small fp32 case the oracle finishes in well under a second.
* ``llama8b``  - one LLaMA-3-8B attention layer (32 query / 8 KV heads, d=128),
                 batch 4, 8K context, per-head top-1024 eviction (the SnapKV /
                 H2O family the ZigZagKV page builds on, its Section 4.1).
* ``zigzag``   - 32 layers of that shape at 32K context with ZigZagKV's
                 per-layer budgets (LMBA at 90 % mass, Eq. 3-6 of the ZigZagKV
                 page): average budget 20 % of context, floor 2 %.
* ``fastgen``  - batch 8 at 16K context with FastGen's three head policies
                 (local window / special tokens / full cache).
* ``chunk``    - 128K context with ChunkLLM-style chunk selection (chunk key =
                 key of the chunk's last token, keep top chunks totalling 48 %).
* ``chunk_icac`` - the same with ChunkLLM's decode-time re-selection: whenever a
                 generated token closes a chunk, the chunks are re-scored against
                 that step's query and re-selected (16 most recent chunks always
                 kept, as in ChunkLLM's long-generation setting). Not one of the
                 five benchmark workloads.
* ``fastgen_sliding`` - fastgen whose local heads also evict while decoding: each keeps
                 exactly its most recent 256 tokens. Not one of the five benchmark workloads.

Nothing here computes any part of the method; this module only holds sizes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    batch: int
    hq: int
    hkv: int
    d: int
    L: int
    dtype: str                 # "fp32" or "bf16": the type Q/K/V are stored and read in
    w: int                     # observation window (0: no scoring in this workload)
    policy: str                # "topb" | "zigzag" | "fastgen" | "chunk"
    steps: int                 # decode steps (tokens appended per sequence)
    seed: int
    top_b: int = 0             # per-KV-head budget for "topb"
    n_sinks: int = 0           # tiny: keys 0..n_sinks-1 become attention sinks
    key_temp: tuple = ()       # (lo, hi) of U[lo, hi] key temperature
    key_temp_per: str = ""     # "kv_head" or "layer"
    mass: float = 0.9          # LMBA attention-mass fraction
    avg_frac: float = 0.20     # zigzag: average budget as a fraction of L
    floor_frac: float = 0.02   # zigzag: per-layer floor as a fraction of L
    local_window: int = 256    # fastgen local policy window
    special_frac: float = 0.04 # fastgen special-token set size as a fraction of L
    chunk_mean: float = 24.0   # chunk: mean of the Geometric chunk length
    keep_frac: float = 0.48    # chunk: fraction of tokens the kept chunks must reach
    icac: bool = False         # chunk: re-select chunks at every generated chunk boundary (ChunkLLM ICAC)
    n_local: int = 0           # chunk: most recent chunks always kept (ChunkLLM local chunks)
    local_sliding: bool = False  # fastgen: local heads keep only their last local_window tokens while decoding

    # ---- derived sizes -------------------------------------------------
    @property
    def G(self) -> int:
        return self.hq // self.hkv

    @property
    def n_slots(self) -> int:
        """A slot is one (layer, batch row, KV head); slots are row-major in that order."""
        return self.n_layers * self.batch * self.hkv

    @property
    def slots_per_layer(self) -> int:
        return self.batch * self.hkv

    @property
    def avg_budget(self) -> int:
        return int(round(self.avg_frac * self.L))

    @property
    def floor_budget(self) -> int:
        return int(round(self.floor_frac * self.L))

    @property
    def n_special(self) -> int:
        return int(round(self.special_frac * self.L))

    @property
    def chunk_target(self) -> int:
        return int(math.ceil(self.keep_frac * self.L))

    @property
    def reserve(self) -> int:
        """Rows kept free per slot for the tokens appended while decoding."""
        return self.steps

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload(
        name="tiny", n_layers=1, batch=1, hq=4, hkv=2, d=64, L=512, dtype="fp32",
        w=16, policy="topb", top_b=64, steps=4, seed=1, n_sinks=4),
    "llama8b": Workload(
        name="llama8b", n_layers=1, batch=4, hq=32, hkv=8, d=128, L=8192, dtype="bf16",
        w=32, policy="topb", top_b=1024, steps=64, seed=2,
        key_temp=(0.5, 2.0), key_temp_per="kv_head"),
    "zigzag": Workload(
        name="zigzag", n_layers=32, batch=1, hq=32, hkv=8, d=128, L=32768, dtype="bf16",
        w=32, policy="zigzag", steps=32, seed=3,
        key_temp=(0.3, 3.0), key_temp_per="layer"),
    "fastgen": Workload(
        name="fastgen", n_layers=1, batch=8, hq=32, hkv=8, d=128, L=16384, dtype="bf16",
        w=0, policy="fastgen", steps=128, seed=4),
    "chunk": Workload(
        name="chunk", n_layers=1, batch=1, hq=32, hkv=8, d=128, L=131072, dtype="bf16",
        w=32, policy="chunk", steps=256, seed=5),
    "fastgen_sliding": Workload(
        name="fastgen_sliding", n_layers=1, batch=8, hq=32, hkv=8, d=128, L=16384, dtype="bf16",
        w=0, policy="fastgen", steps=512, seed=4, local_sliding=True),
    "chunk_icac": Workload(
        name="chunk_icac", n_layers=1, batch=1, hq=32, hkv=8, d=128, L=131072, dtype="bf16",
        w=32, policy="chunk", steps=256, seed=5, icac=True, n_local=16),
}

ORDER = ["tiny", "llama8b", "zigzag", "fastgen", "chunk"]


def get(name: str) -> Workload:
    return WORKLOADS[name]
