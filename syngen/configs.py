"""The synthetic workloads: shapes, value recipes and step counts.

Shapes stand in for a Llama-3.1-8B / LLaMA-3-8B attention layer (32 query heads,
8 KV heads, head dim 128) at the context lengths the pages measure (32K, 128K,
256K), as named in "SALSA: Training-Consistent Sparse Caching with Sink
Preservation for Linearized LLMs" (abstract: Llama-3.1-8B, 32K) and "SLAKE:
Softmax-Approximated Training-Free Linear Attention with KV-Cache Eviction for
Long-Sequence LLMs" (abstract: LLaMA-3 8B, 128K).  No dataset and no trained
weight is used: every value is drawn from the seeded generator.
"""

from __future__ import annotations

import dataclasses
import math


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    T0: int            # prefilled history length at decode step 0
    block_size: int
    n_sink: int
    window: int
    top_k: int
    steps: int         # decode (+ append) steps the workload runs
    n_planted: int = 0         # planted blocks per (layer, b, kv head)
    planted_amp: float = 3.0   # planted key = amp * q_hat + planted_std * N(0,1)
    planted_std: float = 0.1
    head_scale: bool = False   # per-(layer, kv head) scale U(0.5, 2) on K and V
    block_offset_std: float = 0.0  # per-block key offset N(0, std^2), positions >= n_sink
    seed: int = 0
    appends_after_decode: int = 0  # extra appends after the decode steps (parity only)
    # per-layer (top_k, window), cycled over the layers; empty: every layer has
    # top_k and window above
    layer_budgets: tuple = ()
    # per-KV-head (top_k, window), cycled over the KV heads; empty: every head
    # has the layer's budget
    head_budgets: tuple = ()

    def for_layer(self, layer: int) -> "Workload":
        """The workload as layer `layer` sees it: its own top-k and window when
        the budgets vary by layer (the generators draw the same values for the
        same positions either way)."""
        if not self.layer_budgets:
            return self
        k, win = self.layer_budgets[layer % len(self.layer_budgets)]
        return dataclasses.replace(self, top_k=k, window=win, layer_budgets=())

    def for_head(self, h: int) -> "Workload":
        """The workload as KV head `h` sees it: its own top-k and window when the
        budgets vary by head."""
        if not self.head_budgets:
            return self
        k, win = self.head_budgets[h % len(self.head_budgets)]
        return dataclasses.replace(self, top_k=k, window=win, head_budgets=())

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def units_per_layer(self) -> int:
        return self.batch * self.n_kv_heads

    @property
    def capacity(self) -> int:
        """Cache rows per (b, kv head): the prefill plus every appended token."""
        return self.T0 + self.steps + self.appends_after_decode

    def evicted(self, T: int) -> int:
        return max(0, T - self.n_sink - self.window)

    def n_blocks(self, T: int) -> int:
        return -(-self.evicted(T) // self.block_size)

    def exact_tokens(self, T: int) -> int:
        """|sinks| + |window| + tokens of the selected blocks (full blocks assumed)."""
        s = min(self.n_sink, T)
        w = T - max(self.n_sink, T - self.window) if T > self.n_sink else 0
        ev = self.evicted(T)
        nb = self.n_blocks(T)
        k = min(self.top_k, nb)
        # selected blocks are full except possibly the newest partial one
        return s + w + min(ev, k * self.block_size)

    def bytes_per_unit(self, T: int) -> dict:
        """Algorithmic bytes one decode reads/writes per (layer, b, kv head)."""
        d, G = self.head_dim, self.group
        return {
            "exact_kv": self.exact_tokens(T) * d * 2 * 2,
            "block_stats": self.n_blocks(T) * 2 * d * 4,
            "linear_state": (d * d + 2 * d + 1) * 4,
            "q_out": G * d * 2 + G * d * 4,
        }


def _w(**kw) -> Workload:
    return Workload(**kw)


# The workloads.  Names describe shape and context length.
WORKLOADS = {
    "tiny": _w(name="tiny", batch=1, layers=1, n_q_heads=4, n_kv_heads=1, head_dim=64,
               T0=1024, block_size=32, n_sink=4, window=64, top_k=4, steps=1,
               n_planted=2, appends_after_decode=16),
    "llama8b_32k_layer": _w(name="llama8b_32k_layer", batch=1, layers=1, n_q_heads=32,
                            n_kv_heads=8, head_dim=128, T0=32768, block_size=64, n_sink=4,
                            window=1024, top_k=16, steps=1, n_planted=8),
    "llama8b_32layers_b8_32k": _w(name="llama8b_32layers_b8_32k", batch=8, layers=32,
                                  n_q_heads=32, n_kv_heads=8, head_dim=128, T0=32768,
                                  block_size=64, n_sink=4, window=1024, top_k=16, steps=1,
                                  head_scale=True),
    # per-layer budgets (k, W) varying over the layers: the knob a layer-wise
    # budget allocation sets (the allocation itself needs calibration data)
    "llama8b_32layers_b8_32k_budgets": _w(name="llama8b_32layers_b8_32k_budgets", batch=8, layers=32,
                                          n_q_heads=32, n_kv_heads=8, head_dim=128, T0=32768,
                                          block_size=64, n_sink=4, window=1024, top_k=16, steps=1,
                                          head_scale=True,
                                          layer_budgets=((8, 512), (16, 1024), (24, 1536), (32, 2048))),
    # per-KV-head budgets (k, W) varying over the 8 KV heads of every layer
    "llama8b_32layers_b8_32k_head_budgets": _w(name="llama8b_32layers_b8_32k_head_budgets", batch=8, layers=32,
                                               n_q_heads=32, n_kv_heads=8, head_dim=128, T0=32768,
                                               block_size=64, n_sink=4, window=512, top_k=32, steps=1,
                                               head_scale=True,
                                               head_budgets=((8, 512), (16, 1024), (24, 1536), (32, 2048))),
    # token-granular exact set: blocks of one token, the top 1024 tokens exact
    # (the same exact budget as 16 blocks of 64)
    "llama8b_32k_layer_tokens": _w(name="llama8b_32k_layer_tokens", batch=1, layers=1, n_q_heads=32,
                                   n_kv_heads=8, head_dim=128, T0=32768, block_size=1, n_sink=4,
                                   window=1024, top_k=1024, steps=1, n_planted=8),
    "llama8b_32layers_b4_128k": _w(name="llama8b_32layers_b4_128k", batch=4, layers=32,
                                   n_q_heads=32, n_kv_heads=8, head_dim=128, T0=131072,
                                   block_size=64, n_sink=4, window=2048, top_k=32, steps=1,
                                   block_offset_std=0.5),
    "llama8b_256k_256steps": _w(name="llama8b_256k_256steps", batch=1, layers=1,
                                n_q_heads=32, n_kv_heads=8, head_dim=128, T0=262144,
                                block_size=128, n_sink=4, window=4096, top_k=32, steps=256,
                                n_planted=16),
}

# RNG stream ids (one independent stream per kind of draw).
STREAM_K = 1
STREAM_V = 2
STREAM_Q = 3
STREAM_HEAD_SCALE = 4
STREAM_BLOCK_OFFSET = 5
STREAM_PLANTED = 6

# Counter strides: element indices never depend on the cache capacity.
TOKEN_STRIDE = 1 << 20      # >= max positions per (layer, b, kv head)
BLOCK_STRIDE = 1 << 16      # >= max grid blocks per (layer, b, kv head)
STEP_STRIDE = 1 << 12       # >= max decode steps per workload


def get_workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    if overrides:
        w = dataclasses.replace(w, **overrides)
    assert w.n_q_heads % w.n_kv_heads == 0
    assert w.capacity < TOKEN_STRIDE
    assert w.steps < STEP_STRIDE
    assert math.ceil(w.capacity / w.block_size) < BLOCK_STRIDE
    return w
