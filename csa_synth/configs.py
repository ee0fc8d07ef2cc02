"""Workload presets (shapes, formats, seeds) of the CSA/HCA attention operator.

The five workloads are the decode and prefill shapes the operator is measured
on.  Hyper-parameters m=4, top-k=1024, m'=128, window 128 and rotary on the
last 64 dimensions follow "DeepSeek-V4: Making a Million Tokens Affordable",
section "Two ways to shrink attention, interleaved"; the storage formats
(BF16 rotary part, FP8 remainder) follow "DeepSeek-V4 Explained: Compressed
Sparse Attention and 1M Context at 10% KV", section "The attention stack, and
why it is two mechanisms".
"""

from dataclasses import dataclass, field, replace
from typing import Optional


@dataclass(frozen=True)
class Layer:
    """One attention layer's hyper-parameters."""

    kind: str                 # "csa" (compress + index + top-k) or "hca" (compress + dense)
    m: int                    # group size (tokens per compressed entry)
    ov: int                   # 1: each entry pools 2m rows (own m + previous m); 0: own m only
    top_k: int                # CSA only; 0 for HCA
    H: int                    # query heads (share one KV head)
    D: int                    # KV / head dim
    d_rope: int = 64          # rotary dims (the last d_rope of D)
    rope_base: float = 10000.0
    window: int = 128         # sliding-window rows (uncompressed, includes the current token)
    H_I: int = 0              # indexer heads (CSA)
    d_I: int = 0              # indexer head dim (CSA)
    kv_format: str = "bf16"   # "f32" | "bf16" | "mixed" (e4m3 non-rotary + bf16 rotary + fp32 scale)
    idx_format: str = "e4m3"  # "f32" | "e4m3" | "e2m1" (FP4 keys with block scales, e4m3 queries)
    act_format: str = "bf16"  # query / raw-row / gate / output dtype: "f32" | "bf16"
    eps: float = 1e-6
    idx_rank: int = 512       # CSA: width r of the query latent the index query is projected from


@dataclass(frozen=True)
class Workload:
    name: str
    mode: str                         # "decode" or "prefill"
    B: int
    n: int                            # raw tokens present, current one included (decode) / after the chunk (prefill)
    layers: tuple                     # one or more Layer
    seed: int
    Tq: int = 1                       # query tokens per sequence (prefill chunk length)
    pos0: int = 0
    note: str = ""
    extra: dict = field(default_factory=dict)

    def layer(self, i: int = 0) -> Layer:
        return self.layers[i]


CSA_TINY = Layer(kind="csa", m=4, ov=1, top_k=64, H=8, D=128, H_I=4, d_I=64,
                 kv_format="f32", idx_format="f32", act_format="f32")
HCA_128K = Layer(kind="hca", m=128, ov=0, top_k=0, H=64, D=512,
                 kv_format="bf16", idx_format="e4m3", act_format="bf16")
CSA_PRO = Layer(kind="csa", m=4, ov=1, top_k=1024, H=128, D=512, H_I=32, d_I=128,
                kv_format="mixed", idx_format="e4m3", act_format="bf16")
HCA_PRO = Layer(kind="hca", m=128, ov=0, top_k=0, H=128, D=512,
                kv_format="mixed", idx_format="e4m3", act_format="bf16")
CSA_PREFILL = Layer(kind="csa", m=4, ov=1, top_k=1024, H=64, D=512, H_I=32, d_I=128,
                    kv_format="bf16", idx_format="e4m3", act_format="bf16")

WORKLOADS = {
    "csa_decode_tiny_2k": Workload(
        name="csa_decode_tiny_2k", mode="decode", B=1, n=2048, layers=(CSA_TINY,), seed=0,
        note="CSA decode, batch 1, 2,048 raw tokens (512 entries), top-k 64, fp32"),
    "hca_decode_128k": Workload(
        name="hca_decode_128k", mode="decode", B=4, n=131072, layers=(HCA_128K,), seed=1,
        note="HCA decode, batch 4, 131,072 tokens, m'=128 (1,024 entries), 64 heads, BF16"),
    "csa_decode_128k": Workload(
        name="csa_decode_128k", mode="decode", B=8, n=131072, layers=(CSA_PRO,), seed=2,
        note="CSA decode, batch 8, 131,072 tokens (32,768 entries), top-k 1024, 128 heads, mixed BF16/FP8"),
    "csa_hca_decode_1m": Workload(
        name="csa_hca_decode_1m", mode="decode", B=1, n=1 << 20, layers=(CSA_PRO, HCA_PRO), seed=3,
        note="interleaved CSA (262,144 entries, top-k 1024) + HCA (8,192 entries) decode at 1,048,576 tokens"),
    "csa_prefill_8k": Workload(
        name="csa_prefill_8k", mode="prefill", B=1, n=65536 + 8192, Tq=8192, layers=(CSA_PREFILL,), seed=4,
        note="CSA chunked prefill: 8,192 queries appended to a 65,536-token prefix, 64 heads, BF16"),
}


def get_workload(name: str, **overrides) -> Workload:
    """Return a preset, optionally with fields replaced (for scaled-down test cases)."""
    w = WORKLOADS[name]
    if overrides:
        w = replace(w, **overrides)
    return w


def scaled_layer(layer: Layer, **overrides) -> Layer:
    return replace(layer, **overrides)


def row_bytes(layer: Layer) -> int:
    """Bytes per stored KV row (entry or window row) for the layer's format."""
    if layer.kv_format == "f32":
        return 4 * layer.D
    if layer.kv_format == "bf16":
        return 2 * layer.D
    if layer.kv_format == "mixed":
        return layer.D + 80
    raise ValueError(layer.kv_format)


def raw_ring_rows(layer: Layer) -> int:
    """Capacity of the decode ring of uncompressed rows: one entry's source window."""
    return (1 + layer.ov) * layer.m
