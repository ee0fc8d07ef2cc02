"""The CSA / HCA attention layer, step by step, in float64 (oracle; test infrastructure only).

Notation follows the pages: m tokens per compressed entry (m' for HCA), top-k
selected entries, a window of w = 128 uncompressed recent tokens, H query
heads sharing one KV head of dimension D, rotary on the last d_r = 64 dims.

Readings taken where the pages are silent (each repeated at its function):

R1  Overlap is look-back: entry i pools raw rows [(i-ov)m, (i+1)m), clipped at
    row 0.  The pages have each entry read 2m source rows while the sequence
    still shrinks m-fold ("DeepSeek-V4: Making a Million Tokens Affordable",
    "Two ways to shrink attention, interleaved").  HCA uses ov=0.
R2  The learned per-token compression weights and positional biases of the same
    section = one gate logit per raw row and channel plus one bias per window
    slot and channel, normalised by a softmax over the window's rows, per
    channel.
R3  Entry i is rotated at position pos0 + i*m and is visible to a query at
    position t iff its last row pos0 + (i+1)m - 1 <= t (causally complete).
R4  Window rows are the most recent w raw rows including the current one,
    rotated at their own positions, not normalised; entries and window rows
    are separate key sets and nothing is de-duplicated.
R5  Index score s_i = sum_h w_h * ReLU(sigma_q,h * sigma_k,i * <q_h, k_i>)
    over H_I indexer heads.  The pages give no formula; the glossary of
    "DeepSeek-V4, explained." says outright that V4's exact scorer is not given.
R6  Top-k: the k largest scores, ties to the smaller entry index; returned in
    ascending entry order; fewer than k visible entries -> all of them, then -1.
R7  Logits l_j = <q~, k~_j> / sqrt(D); sink: p_j = e^{l_j} / (e^{s_h} + sum e^{l}).
R8  RoPE: interleaved pairs (D-64+2u, D-64+2u+1), theta_u = base^(-2u/64),
    angle pos*theta_u in float64.
R9  RMSNorm eps = 1e-6 with a learnable per-channel weight gamma.
R14 Index keys come from an index-key stream compressed like the KV stream: every token carries
    an index row and a row of gate logits of d_I channels, and the key of entry i pools the same
    window rows with the same per-channel softmax of gate + slot bias (its own bias table), with
    no RMSNorm and no rotation; it is stored as e4m3 codes with one power-of-two scale per key
    (the R10 rule), or as float32.  "DeepSeek-V4 Explained: ...", "The attention stack, and why it
    is two mechanisms", has the indexer score the compressed entries; the keys it scores are read
    here as compressed the same way.
R15 The low-rank index query: the query token's low-rank latent c (r values, an input) is mapped
    by a learned up-projection W [H_I * d_I, r] to the H_I index-query heads, q_h = W_h c, each head
    stored as e4m3 codes with its own power-of-two scale (R10).  The same section calls the
    indexer low-rank; this is its plainest form.  Head weights w_h stay inputs.
"""

import numpy as np

from . import formats as F


# --------------------------------------------------------------------------- rotary / norm

def rope_cos_sin(pos, d_rope: int, base: float):
    """cos, sin of pos * theta_u for u < d_rope/2 (R8), float64 [..., d_rope/2].

    Only the last 64 dimensions are rotated ("DeepSeek-V4: Making a Million Tokens
    Affordable", "Two ways to shrink attention, interleaved").
    """
    pos = np.asarray(pos, dtype=np.float64)
    u = np.arange(d_rope // 2, dtype=np.float64)
    theta = np.power(float(base), -2.0 * u / d_rope)
    ang = pos[..., None] * theta
    return np.cos(ang), np.sin(ang)


def rope(x, pos, d_rope: int, base: float):
    """Rotate the last d_rope dims of x [..., D] by position pos (broadcast on x's leading dims)."""
    x = np.array(x, dtype=np.float64, copy=True)
    D = x.shape[-1]
    c, s = rope_cos_sin(pos, d_rope, base)
    a = x[..., D - d_rope::2].copy()
    b = x[..., D - d_rope + 1::2].copy()
    x[..., D - d_rope::2] = a * c - b * s
    x[..., D - d_rope + 1::2] = a * s + b * c
    return x


def rms_norm(x, gamma, eps: float):
    """x / sqrt(mean(x^2) + eps) * gamma (R9).

    Queries and compressed entries are RMS-normalised before the core attention
    ("DeepSeek-V4: Making a Million Tokens Affordable", "Two ways to shrink
    attention, interleaved").
    """
    x = np.asarray(x, dtype=np.float64)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r * np.asarray(gamma, dtype=np.float64)


# --------------------------------------------------------------------------- compression (a2)

def entry_rows(i: int, m: int, ov: int):
    """Raw row indices (relative to pos0) pooled into entry i, and their window slots (R1)."""
    lo = (i - ov) * m
    rows = np.arange(max(lo, 0), (i + 1) * m)
    return rows, rows - lo


def pool_entry(raw_rows, gate_rows, bias, slots):
    """Per-channel softmax-weighted sum of one entry's source rows (R2).

    raw_rows, gate_rows: [r, D]; bias: [(1+ov)m, D]; slots: window slot of each row.
    Each group of m consecutive tokens is pooled into one entry with learned
    weights and position biases ("DeepSeek-V4 Explained: ...", "The attention
    stack, and why it is two mechanisms").
    """
    z = np.asarray(gate_rows, np.float64) + np.asarray(bias, np.float64)[slots]
    z = z - z.max(axis=0, keepdims=True)
    a = np.exp(z)
    a = a / a.sum(axis=0, keepdims=True)
    return (a * np.asarray(raw_rows, np.float64)).sum(axis=0)


def compress(raw, gate, bias, gamma, m, ov, d_rope, base, pos0, entries, raw_first_row=0):
    """Entries (float64 [len(entries), D]) from uncompressed rows.

    raw, gate: float64 [n_rows, D] holding raw rows raw_first_row.. (relative to
    pos0).  Each entry: pool (R1, R2) -> RMSNorm (R9) -> rotate at pos0 + i*m (R3).
    """
    out = []
    for i in entries:
        rows, slots = entry_rows(int(i), m, ov)
        idx = rows - raw_first_row
        assert idx.min() >= 0 and idx.max() < raw.shape[0], "source rows not provided"
        e = pool_entry(raw[idx], gate[idx], bias, slots)
        e = rms_norm(e, gamma, 1e-6)
        out.append(rope(e, pos0 + int(i) * m, d_rope, base))
    return np.stack(out) if out else np.zeros((0, raw.shape[1]))


def compress_index_keys(raw_i, gate_i, bias_i, m, ov, entries, raw_first_row=0):
    """Index-key values (float64 [len(entries), d_I]) of the given entries (R14): pool only.

    raw_i, gate_i: float64 [n_rows, d_I] index rows and gate logits of raw rows raw_first_row..;
    bias_i: [(1+ov)m, d_I].
    """
    out = []
    for i in entries:
        rows, slots = entry_rows(int(i), m, ov)
        idx = rows - raw_first_row
        assert idx.min() >= 0 and idx.max() < raw_i.shape[0], "source rows not provided"
        out.append(pool_entry(raw_i[idx], gate_i[idx], bias_i, slots))
    return np.stack(out) if out else np.zeros((0, raw_i.shape[1]))


def index_query(c, W, H_I: int, d_I: int):
    """Index-query heads [H_I, d_I] from the query's low-rank latent c [r] (R15): q = W c."""
    W = np.asarray(W, np.float64)
    c = np.asarray(c, np.float64)
    return (W @ c).reshape(H_I, d_I)


# --------------------------------------------------------------------------- visibility

def n_visible(t, pos0: int, m: int):
    """Number of causally complete entries for a query at position t (R3)."""
    return (np.asarray(t, np.int64) - pos0 + 1) // m


def window_row_ids(t: int, pos0: int, w: int):
    """Raw row indices of the sliding window of a query at position t (R4)."""
    r = t - pos0
    return np.arange(max(0, r - w + 1), r + 1)


# --------------------------------------------------------------------------- indexer (a3) and top-k (a4)

def index_scores(iq, iq_scale, head_w, ik, ik_scale):
    """s_i = sum_h w_h * ReLU(sigma_q,h * sigma_k,i * <q_h, k_i>) (R5).

    iq [H_I, d_I], iq_scale [H_I], head_w [H_I], ik [N, d_I], ik_scale [N].
    The indexer is a cheap low-rank scorer ("DeepSeek-V4 Explained: ...") made of
    a few small FP8 heads that score each past entry ("DeepSeek-V4, explained.",
    step 3).
    """
    dots = np.asarray(ik, np.float64) @ np.asarray(iq, np.float64).T          # [N, H_I]
    z = dots * np.asarray(ik_scale, np.float64)[:, None] * np.asarray(iq_scale, np.float64)[None, :]
    return np.maximum(z, 0.0) @ np.asarray(head_w, np.float64)


def index_operands(L, q_codes, k_codes, k_scales):
    """(query values before their scale, key values, key scales) of the indexer in float64.

    e4m3 / f32 keys keep their per-key scale apart; FP4 keys (idx_format "e2m1", read as the pages'
    FP4 indexer: "DeepSeek-V4: Making a Million Tokens Affordable", "Two ways to shrink attention,
    interleaved") are decoded with their block scales applied and a key scale of 1.  With FP4 keys the
    index queries are e4m3 (the pages put the indexer's attention in FP4; the keys are its stored side).
    """
    if L.idx_format == "e2m1":
        return (F.decode_idx(q_codes, "e4m3"), F.decode_fp4_keys(k_codes, k_scales),
                np.ones(len(k_scales), np.float64))
    return F.decode_idx(q_codes, L.idx_format), F.decode_idx(k_codes, L.idx_format), k_scales


def top_k(scores, k: int):
    """Indices of the k largest scores, ties to the smaller index, ascending, -1 padded (R6).

    Only the k best-scoring entries reach the core attention ("DeepSeek-V4,
    explained.", step 4; "DeepSeek-V4: Making a Million Tokens Affordable").
    """
    s = np.asarray(scores, np.float64)
    order = sorted(range(len(s)), key=lambda i: (-s[i], i))   # stable, explicit tie rule
    keep = np.array(sorted(order[:k]), dtype=np.int64)
    out = np.full(k, -1, dtype=np.int64)
    out[:len(keep)] = keep
    return out


def top_k_fast(scores, k: int):
    """Same result as top_k via a stable sort (for large N)."""
    s = np.asarray(scores, np.float64)
    order = np.argsort(-s, kind="stable")
    keep = np.sort(order[:k])
    out = np.full(k, -1, dtype=np.int64)
    out[:len(keep)] = keep
    return out


# --------------------------------------------------------------------------- core attention (a5 / a6)

def prep_query(q, gamma_q, t, d_rope, base, eps=1e-6):
    """q~ = RoPE_t(RMSNorm(q) * gamma_q) per head (a1)."""
    return rope(rms_norm(q, gamma_q, eps), t, d_rope, base)


def attend(q, t, rows, sinks, gamma_q, d_rope, base, scale=None, eps=1e-6):
    """Shared-KV multi-query attention with sinks and inverse RoPE on the output.

    q [H, D] (raw), rows [R, D] (keys = values), sinks [H] -> o [H, D].
    An entry is both key and value; the output is rotated back by the query's
    position so only relative positions matter; a learned per-head sink can take
    part of a head's attention weight ("DeepSeek-V4: Making a Million Tokens
    Affordable", "Two ways to shrink attention, interleaved"), so the weights on
    the keys can sum to less than one ("DeepSeek-V4 Explained: ...").  Readings
    R7, R8, R9.
    """
    rows = np.asarray(rows, np.float64)
    D = rows.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    qt = prep_query(q, gamma_q, t, d_rope, base, eps)
    logits = (qt @ rows.T) * scale                                   # [H, R]
    s = np.asarray(sinks, np.float64)
    M = np.maximum(s, logits.max(axis=1) if logits.shape[1] else s)
    e = np.exp(logits - M[:, None])
    Z = np.exp(s - M) + e.sum(axis=1)
    p = e / Z[:, None]
    o = p @ rows
    return rope(o, -float(t), d_rope, base)


def attention_probs(q, t, rows, sinks, gamma_q, d_rope, base, scale=None, eps=1e-6):
    """The attention weights p [H, R] of `attend` (for the sink pins)."""
    rows = np.asarray(rows, np.float64)
    D = rows.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    qt = prep_query(q, gamma_q, t, d_rope, base, eps)
    logits = (qt @ rows.T) * scale
    s = np.asarray(sinks, np.float64)
    M = np.maximum(s, logits.max(axis=1))
    e = np.exp(logits - M[:, None])
    return e / (np.exp(s - M) + e.sum(axis=1))[:, None]


# --------------------------------------------------------------------------- one decode step (a7)

class LayerSpec:
    """The hyper-parameters one step needs (plain attributes, no behaviour)."""

    def __init__(self, kind, m, ov, top_k, H, D, d_rope=64, rope_base=10000.0, window=128,
                 H_I=0, d_I=0, kv_format="bf16", idx_format="e4m3", act_format="bf16",
                 eps=1e-6, pos0=0, scale=None):
        self.kind, self.m, self.ov, self.top_k = kind, m, ov, top_k
        self.H, self.D, self.d_rope, self.rope_base, self.window = H, D, d_rope, rope_base, window
        self.H_I, self.d_I = H_I, d_I
        self.kv_format, self.idx_format, self.act_format = kv_format, idx_format, act_format
        self.eps, self.pos0, self.scale = eps, pos0, scale

    @classmethod
    def of(cls, layer, pos0=0):
        return cls(layer.kind, layer.m, layer.ov, layer.top_k, layer.H, layer.D, layer.d_rope,
                   layer.rope_base, layer.window, layer.H_I, layer.d_I, layer.kv_format,
                   layer.idx_format, layer.act_format, layer.eps, pos0)


def append_window_row(L, x_row, t):
    """Stored window row of the token at position t: RoPE_t(x), not normalised (R4)."""
    return F.encode_rows(rope(x_row, t, L.d_rope, L.rope_base), L.kv_format, L.d_rope)


def decode_step(L, st, b: int):
    """One decode step of sequence b: append -> compress (if a group completes) -> select -> attend.

    ``st`` holds the state and step inputs in storage form (the keys of
    csa_synth.decode_inputs); it is not modified.  Returns a dict with the
    output o [H, D] (float64), the new window row and (when a group completed)
    the new entry's index and stored row, the scores and the selected indices.
    """
    t = int(st["t"][b])
    r = t - L.pos0
    m, ov, D = L.m, L.ov, L.D
    rr = (1 + ov) * m
    res = {}
    x_new = F.decode_act(st["x_new"][b], L.act_format)
    g_new = F.decode_act(st["g_new"][b], L.act_format)
    # append the new token to the window ring and the uncompressed ring
    wrow = append_window_row(L, x_new, t)
    res["window_row"] = wrow
    window = st["window"][b].copy()
    window[r % L.window] = wrow
    raw_ring = F.decode_act(st["raw_ring"][b], L.act_format).copy()
    gate_ring = F.decode_act(st["gate_ring"][b], L.act_format).copy()
    raw_ring[r % rr] = x_new
    gate_ring[r % rr] = g_new
    # compress the entry completed by this token
    entries = st["entries"][b]
    new_entry = None
    if (r + 1) % m == 0:
        i = (r + 1) // m - 1
        rows, slots = entry_rows(i, m, ov)
        e = pool_entry(raw_ring[rows % rr], gate_ring[rows % rr], st["pos_bias"], slots)
        e = rope(rms_norm(e, st["gamma_kv"], L.eps), L.pos0 + i * m, L.d_rope, L.rope_base)
        new_entry = (i, F.encode_rows(e, L.kv_format, L.d_rope))
        res["entry"] = new_entry
    n_vis = int(n_visible(t, L.pos0, m))

    def entry_values(ids):
        raw_bytes = entries[ids].copy()
        if new_entry is not None:
            raw_bytes[ids == new_entry[0]] = new_entry[1]
        return F.decode_rows(raw_bytes, L.kv_format, D, L.d_rope)

    if L.kind == "csa":
        iq, ik, iks = index_operands(L, st["idx_q"][b], st["idx_k"][b][:n_vis], st["idx_k_scale"][b][:n_vis])
        s = index_scores(iq, st["idx_q_scale"][b], st["head_w"][b], ik, iks)
        sel = top_k_fast(s, L.top_k)
        res["scores"], res["topk"] = s, sel
        ent = entry_values(sel[sel >= 0])
    else:
        ent = entry_values(np.arange(n_vis))
    wids = window_row_ids(t, L.pos0, L.window)
    win = F.decode_rows(window[wids % L.window], L.kv_format, D, L.d_rope)
    rows = np.concatenate([ent, win], axis=0)
    q = F.decode_act(st["q"][b], L.act_format)
    res["o"] = attend(q, t, rows, st["sinks"], st["gamma_q"], L.d_rope, L.rope_base, L.scale, L.eps)
    res["n_rows"] = rows.shape[0]
    return res


def decode_step_indexed(L, st, b: int):
    """decode_step with the index side produced in the step (R14, R15): the new token's index row
    and gate row go into the index rings, the index key of the entry the token completes is
    compressed from them, and the index query comes from the latent c through W.  st holds
    decode_step's keys plus idx_raw_ring / idx_gate_ring [B, (1+ov)m, d_I], idx_x_new / idx_g_new
    [B, d_I] (act format), idx_pos_bias [(1+ov)m, d_I], c_q [B, r] and W_iq [H_I*d_I, r] (act format).
    Returns decode_step's result plus "index_key" (i, codes, scale) when a group completed and
    "idx_q" (codes, scales)."""
    t = int(st["t"][b])
    r = t - L.pos0
    m, ov = L.m, L.ov
    rr = (1 + ov) * m
    st2 = dict(st)
    extra = {}
    raw_i = F.decode_act(st["idx_raw_ring"][b], L.act_format).copy()
    gate_i = F.decode_act(st["idx_gate_ring"][b], L.act_format).copy()
    raw_i[r % rr] = F.decode_act(st["idx_x_new"][b], L.act_format)
    gate_i[r % rr] = F.decode_act(st["idx_g_new"][b], L.act_format)
    if (r + 1) % m == 0:
        i = (r + 1) // m - 1
        rows, slots = entry_rows(i, m, ov)
        key = pool_entry(raw_i[rows % rr], gate_i[rows % rr], st["idx_pos_bias"], slots)
        codes, scale = F.encode_idx(key[None], L.idx_format, "key")
        idx_k = np.array(st["idx_k"], copy=True)
        idx_ks = np.array(st["idx_k_scale"], copy=True)
        idx_k[b, i] = codes[0]
        idx_ks[b, i] = scale[0]
        st2["idx_k"], st2["idx_k_scale"] = idx_k, idx_ks
        extra["index_key"] = (i, codes[0], scale[0])
    q = index_query(F.decode_act(st["c_q"][b], L.act_format), F.decode_act(st["W_iq"], L.act_format), L.H_I, L.d_I)
    qc, qs = F.encode_idx(q, L.idx_format, "query")
    iq = np.array(st["idx_q"], copy=True)
    iqs = np.array(st["idx_q_scale"], copy=True)
    iq[b], iqs[b] = qc, qs
    st2["idx_q"], st2["idx_q_scale"] = iq, iqs
    extra["idx_q"] = (qc, qs)
    res = decode_step(L, st2, b)
    res.update(extra)
    return res


# --------------------------------------------------------------------------- chunked prefill

def prefill_caches(L, pf, b: int):
    """Entries and window ring after appending a prefill chunk (compress + append).

    pf holds csa_synth.prefill_inputs' keys.  Returns (entries bytes, window
    bytes, first new entry, number of new entries).
    """
    m, ov = L.m, L.ov
    prefix, n, Tq = pf["prefix"], pf["n"], pf["Tq"]
    raw = F.decode_act(pf["raw"][b], L.act_format)
    gate = F.decode_act(pf["gate"][b], L.act_format)
    first = pf["raw_first_row"]
    window = pf["window"][b].copy()
    cap = window.shape[0]
    for r in range(prefix, n):
        window[r % cap] = append_window_row(L, raw[r - first], L.pos0 + r)
    e0, e1 = prefix // m, n // m
    entries = pf["entries"][b].copy()
    if e1 > e0:
        vals = compress(raw, gate, pf["pos_bias"], pf["gamma_kv"], m, ov, L.d_rope, L.rope_base,
                        L.pos0, range(e0, e1), raw_first_row=first)
        entries[e0:e1] = F.encode_rows(vals, L.kv_format, L.d_rope)
    return entries, window, e0, e1 - e0


def prefill_query(L, pf, entries, window, b: int, j: int):
    """Output of query j of the chunk (position prefix + j) given the updated caches."""
    t = int(pf["t"][b, j])
    n_vis = int(n_visible(t, L.pos0, L.m))
    res = {}
    if L.kind == "csa":
        iq, ik, iks = index_operands(L, pf["idx_q"][b, j], pf["idx_k"][b][:n_vis], pf["idx_k_scale"][b][:n_vis])
        s = index_scores(iq, pf["idx_q_scale"][b, j], pf["head_w"][b, j], ik, iks)
        sel = top_k_fast(s, L.top_k)
        res["scores"], res["topk"] = s, sel
        ids = sel[sel >= 0]
    else:
        ids = np.arange(n_vis)
    ent = F.decode_rows(entries[ids], L.kv_format, L.D, L.d_rope)
    wids = window_row_ids(t, L.pos0, L.window)
    win = F.decode_rows(window[wids % window.shape[0]], L.kv_format, L.D, L.d_rope)
    rows = np.concatenate([ent, win], axis=0)
    q = F.decode_act(pf["q"][b, j], L.act_format)
    res["o"] = attend(q, t, rows, pf["sinks"], pf["gamma_q"], L.d_rope, L.rope_base, L.scale, L.eps)
    return res
