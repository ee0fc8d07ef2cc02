"""KV-cache and per-token FLOP accounting of the hybrid attention stack, by context length.

Host arithmetic only (no kernels): the cost model behind the pages' efficiency figures, so that their
shape can be reproduced from layer counts and the operator's own storage formats.

What the pages fix, and this module takes as given:
  * groups of m = 4 (CSA) and m' = 128 (HCA) tokens per entry, top-k = 1024, a 128-token window, the
    two layer kinds alternating ("DeepSeek-V4: Making a Million Tokens Affordable", "Two ways to
    shrink attention, interleaved"; "DeepSeek-V4 Explained: ...", "The attention stack, and why it is
    two mechanisms");
  * 61 layers and 49B activated parameters for V4-Pro, 43 layers and 13B for V4-Flash ("Decoding
    DeepSeek-V4", "Two models"; "DeepSeek-V4 Explained: ...", "Key results"), 37B activated for
    V3.2 (same "Key results");
  * entries stored with BF16 rotary dims and FP8 for the rest, the indexer run in FP4 (same "Two
    ways" section), a 512-wide latent for the latent-attention cache ("DeepSeek-V4, explained.", its
    first lever: a 512 latent against a 4096-wide K/V is an 8x smaller cache);
  * the reported results: at 1M tokens V4-Pro needs 27% of V3.2's single-token FLOPs and 10% of its
    KV cache (3.7x and 9.5x), V4-Flash 10% and 7% (9.8x and 13.7x); against BF16 GQA-8 with head
    dim 128 the V4 cache is roughly 2%, and mixed storage about halves it.

Readings (the pages do not give these; each is a parameter below):
  * R-A1  alternation = one CSA layer, then one HCA layer; an odd count starts and ends with CSA.
  * R-A2  KV dim 512 with 64 rotary dims (the operator's row: 448 FP8 codes + 64 BF16 + a 4-byte
          scale = 580 bytes); index keys of 128 dims with a 4-byte scale per entry.
  * R-A3  V3.2 caches one latent row per token (512 latent + 64 rotary dims, in the same mixed
          format) plus one index key per token, and its indexer (64 heads x 128 dims, FP8) scores
          every past token; it attends its top 2048 tokens with 128 heads.  V4-Flash runs 64 heads.
  * R-A4  "FP8-equivalent" FLOPs: an FP8 FLOP counts 1, a BF16 FLOP 2, an FP4 FLOP 0.5; the
          model's projections count 2 FLOPs per activated parameter at FP8 cost.
  * R-A5  the entries a query sees count only complete groups (floor(n/m)); the pages' "7,813" at
          one million tokens counts the trailing partial group as well (ceil), which
          `entries_seen(..., partial=True)` gives.

Run `python -m long_context_sparse_csa_b200.accounting` for the table of both models against V3.2
and GQA-8 over context lengths.
"""

from dataclasses import dataclass

GIB = float(1 << 30)


@dataclass(frozen=True)
class AttentionKind:
    """Per-layer attention parameters that set its cache and its per-token compute."""

    name: str
    m: int = 1                    # tokens per cached entry (1: every token cached)
    top_k: int = 0                # selected entries per query (0: attend every visible entry)
    window: int = 0               # uncompressed recent tokens attended besides the entries
    heads: int = 128              # query heads (all share one KV head)
    qk_dim: int = 512             # dims of the query-key product
    v_dim: int = 512              # dims of the value product
    row_bytes: float = 580.0      # stored bytes of one entry
    window_row_bytes: float = 580.0
    idx_heads: int = 0            # indexer heads (0: no indexer)
    idx_dim: int = 128
    idx_key_bytes: float = 0.0    # stored bytes of one entry's index key (with its scale)
    idx_cost: float = 1.0         # FP8-equivalent cost of one indexer FLOP (FP8 1, FP4 0.5)
    attn_cost: float = 2.0        # FP8-equivalent cost of one attention FLOP (BF16 2)


@dataclass(frozen=True)
class Model:
    name: str
    layers: tuple                  # one AttentionKind per layer, in order
    active_params: float          # activated parameters per token
    param_cost: float = 1.0       # FP8-equivalent cost of one projection FLOP


def entries_seen(n: int, m: int, partial: bool = False) -> int:
    """Entries a query at context n attends over when every m tokens become one (R-A5)."""
    return -(-n // m) if partial else n // m


def layer_kv_bytes(k: AttentionKind, n: int) -> float:
    """Cache bytes one layer holds for a context of n tokens (entries, index keys, window)."""
    e = entries_seen(n, k.m)
    w = min(k.window, n)
    return e * (k.row_bytes + k.idx_key_bytes) + w * k.window_row_bytes


def layer_flops(k: AttentionKind, n: int) -> dict:
    """FLOPs of one generated token in one layer at context n: indexer and core attention."""
    e = entries_seen(n, k.m)
    att_rows = (min(k.top_k, e) if k.top_k else e) + min(k.window, n)
    idx = 2.0 * k.idx_heads * k.idx_dim * e if k.idx_heads else 0.0
    att = 2.0 * k.heads * (k.qk_dim + k.v_dim) * att_rows
    return {"indexer": idx, "attention": att, "fp8_equiv": idx * k.idx_cost + att * k.attn_cost}


def model_kv_bytes(model: Model, n: int) -> float:
    return sum(layer_kv_bytes(k, n) for k in model.layers)


def model_flops(model: Model, n: int) -> float:
    """FP8-equivalent FLOPs of one generated token at context n (projections + every layer)."""
    return 2.0 * model.active_params * model.param_cost + sum(layer_flops(k, n)["fp8_equiv"] for k in model.layers)


# ----------------------------------------------------------------------------- the configurations

def _v4_kinds(heads: int, idx_cost: float = 0.5):
    csa = AttentionKind("csa", m=4, top_k=1024, window=128, heads=heads, idx_heads=32, idx_dim=128,
                        idx_key_bytes=132.0, idx_cost=idx_cost)
    hca = AttentionKind("hca", m=128, top_k=0, window=128, heads=heads)
    return csa, hca


def alternating(n_layers: int, first, second) -> tuple:
    """first, second, first, ... (R-A1)."""
    return tuple(first if i % 2 == 0 else second for i in range(n_layers))


def v4_pro() -> Model:
    csa, hca = _v4_kinds(128)
    return Model("V4-Pro", alternating(61, csa, hca), 49e9)


def v4_flash() -> Model:
    csa, hca = _v4_kinds(64)
    return Model("V4-Flash", alternating(43, csa, hca), 13e9)


def v3_2() -> Model:
    """The latent-attention baseline with a token-level indexer (R-A3)."""
    dsa = AttentionKind("dsa", m=1, top_k=2048, window=0, heads=128, qk_dim=576, v_dim=512,
                        row_bytes=512 + 2 * 64 + 4, idx_heads=64, idx_dim=128, idx_key_bytes=132.0, idx_cost=1.0)
    return Model("V3.2", tuple(dsa for _ in range(61)), 37e9)


def gqa8_bf16_kv_bytes_per_layer(n: int, head_dim: int = 128) -> float:
    """Dense GQA with 8 KV heads stored in BF16: one key and one value per head and token."""
    return n * 2 * 8 * head_dim * 2.0


def mixed_vs_bf16_row_ratio(D: int = 512, d_rope: int = 64) -> float:
    """Stored bytes of a mixed row (FP8 codes + BF16 rotary dims + a 4-byte scale) over a BF16 row."""
    return ((D - d_rope) + 2 * d_rope + 4) / (2.0 * D)


def figure1(contexts=(8192, 32768, 131072, 262144, 524288, 1 << 20, 10 ** 6)) -> list:
    """Rows (context, model, FLOPs, KV bytes, and each as a fraction of V3.2)."""
    base = v3_2()
    out = []
    for n in contexts:
        bf, bk = model_flops(base, n), model_kv_bytes(base, n)
        for mdl in (base, v4_pro(), v4_flash()):
            f, kv = model_flops(mdl, n), model_kv_bytes(mdl, n)
            out.append({"context": n, "model": mdl.name, "gflop_per_token": f / 1e9, "kv_gib": kv / GIB,
                        "flops_vs_v3_2": f / bf, "kv_vs_v3_2": kv / bk})
    return out


def gqa8_comparison(n: int = 10 ** 6) -> dict:
    """V4-Pro's per-layer-average cache at n tokens against dense BF16 GQA-8 (head dim 128), with the
    operator's mixed rows and with the same rows in BF16 (the pages' "roughly 2%, halved again")."""
    pro = v4_pro()
    mixed = model_kv_bytes(pro, n) / len(pro.layers)
    csa, hca = _v4_kinds(128)
    bf16 = [AttentionKind(k.name, m=k.m, top_k=k.top_k, window=k.window, heads=k.heads, row_bytes=1024.0,
                          window_row_bytes=1024.0, idx_heads=k.idx_heads, idx_key_bytes=k.idx_key_bytes)
            for k in (csa, hca)]
    bf16_layers = alternating(61, *bf16)
    bf16_avg = sum(layer_kv_bytes(k, n) for k in bf16_layers) / len(bf16_layers)
    g = gqa8_bf16_kv_bytes_per_layer(n)
    return {"context": n, "mixed_vs_gqa8": mixed / g, "bf16_vs_gqa8": bf16_avg / g,
            "mixed_vs_bf16": mixed / bf16_avg}


def main():
    rows = figure1()
    print(f"{'context':>9} {'model':>9} {'GFLOP/token':>12} {'KV GiB':>8} {'FLOPs/V3.2':>11} {'KV/V3.2':>8}")
    for r in rows:
        print(f"{r['context']:>9} {r['model']:>9} {r['gflop_per_token']:>12.1f} {r['kv_gib']:>8.2f} "
              f"{100 * r['flops_vs_v3_2']:>10.1f}% {100 * r['kv_vs_v3_2']:>7.1f}%")
    g = gqa8_comparison()
    print(f"V4-Pro cache per layer at 1M vs BF16 GQA-8: {100 * g['mixed_vs_gqa8']:.2f}% (mixed rows), "
          f"{100 * g['bf16_vs_gqa8']:.2f}% (BF16 rows); mixed / BF16 = {g['mixed_vs_bf16']:.2f}")
    print(f"entries at 10^6 tokens: {entries_seen(10 ** 6, 4)} (m=4), {entries_seen(10 ** 6, 128, True)} "
          f"(m'=128, partial group counted)")


if __name__ == "__main__":
    main()
