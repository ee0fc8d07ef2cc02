"""Helpers shared by the GPU parity tests: device transfer and comparison rules.

Comparison rules (from the operator's stated bar, with the arithmetic behind them):

* Stored rows written by the CUDA path (compressed entries, window rows) must
  lie within one quantum of the storage format around the oracle's exact
  value: round-to-nearest gives half a quantum, and float32 arithmetic on the
  GPU against float64 in the oracle may push a value across a rounding
  midpoint, never further.  For the mixed format the quantum uses the larger
  of the two sides' row scales (they differ only when the row maximum sits on
  a power-of-two boundary).
* Top-k sets must be equal, except that indices whose oracle score lies
  within 1e-4 (relative) of the k-th largest score may be swapped.
* Attention outputs: max-abs <= 2e-2 and mean-abs <= 2e-3 on BF16/FP8 inputs;
  relative L2 error is reported and bounded as well (bf16 rounding of the
  query, the probabilities and the output gives ~2^-8 relative per term).
"""

import numpy as np
import torch

from oracle import csa as O
from oracle import formats as F


def dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def host(t):
    a = t.detach().cpu().numpy()
    if a.dtype == np.int16:
        a = a.view(np.uint16)
    return a


def out_values(t, act_format):
    """Attention output tensor -> float64 numpy."""
    a = host(t)
    return F.decode_act(a, act_format)


def _quantum_bf16(x):
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(ax)) - 7)


def _quantum_e4m3(y):
    ay = np.abs(y)
    e = np.floor(np.log2(np.maximum(ay, 2.0 ** -6)))
    return np.exp2(np.maximum(e, -6) - 3)


def assert_rows_match(gpu_rows, ref_vals, fmt, D, d_rope=64, slack_rel=2e-5, max_code_mismatch=2e-3):
    """GPU-written stored rows vs the oracle's exact float64 values (before encoding)."""
    g = F.decode_rows(gpu_rows, fmt, D, d_rope)
    x = np.asarray(ref_vals, np.float64)
    # float32 rounding in the kernel is relative to the row's scale (the summands), not to a value
    # that happens to land near zero: allow 2e-6 of the row's rms on top of one quantum.
    row_rms = np.sqrt(np.mean(x * x, axis=-1, keepdims=True))
    if fmt == "f32":
        tol = 1e-5 * np.abs(x) + 2e-6 * row_rms
    elif fmt == "bf16":
        tol = _quantum_bf16(x) + slack_rel * np.abs(x) + 2e-6 * row_rms
    else:
        dn = D - d_rope
        sig_g = np.ascontiguousarray(gpu_rows[..., D + 64:D + 68]).view(np.float32)[..., 0].astype(np.float64)
        sig_o = F.pow2_scale(np.max(np.abs(x[..., :dn]), axis=-1))
        sig = np.maximum(sig_g, sig_o)[..., None]
        tol = np.empty_like(x)
        tol[..., :dn] = _quantum_e4m3(x[..., :dn] / sig) * sig
        tol[..., dn:] = _quantum_bf16(x[..., dn:])
        tol += slack_rel * np.abs(x) + 2e-6 * row_rms
        assert np.mean(sig_g == sig_o) > 0.99, "row scales disagree on more than 1% of rows"
    err = np.abs(g - x)
    bad = err > tol
    assert not bad.any(), f"{bad.sum()} values beyond one quantum; worst {err[bad].max()} at {np.argwhere(bad)[:3]}"
    if fmt != "f32":
        ref_rows = F.encode_rows(x, fmt, d_rope)
        mism = np.mean(ref_rows != gpu_rows)
        assert mism <= max_code_mismatch, f"code mismatch fraction {mism}"


def check_topk(gpu_idx, oracle_scores, k, rel=1e-4):
    """Validates one query's GPU top-k list against the oracle's scores; returns #swapped (tie band)."""
    gpu_idx = np.asarray(gpu_idx, np.int64)
    n = len(oracle_scores)
    nsel = min(k, n)
    sel = gpu_idx[:nsel]
    assert np.all(gpu_idx[nsel:] == -1), "padding must be -1"
    assert np.all(sel >= 0) and np.all(sel < n), "indices out of range"
    assert np.all(np.diff(sel) > 0), "indices must be strictly ascending"
    ref = O.top_k_fast(oracle_scores, k)[:nsel]
    diff = set(sel.tolist()) ^ set(ref.tolist())
    if diff:
        s = np.asarray(oracle_scores, np.float64)
        sk = np.sort(s)[::-1][k - 1]
        band = np.abs(s - sk) <= rel * abs(sk)
        outside = [i for i in diff if not band[i]]
        assert not outside, f"top-k differs outside the tie band: {outside[:5]} (k-th score {sk})"
    return len(diff) // 2


STATS = []


def assert_out_close(gpu, ref, max_abs=2e-2, mean_abs=2e-3, rel_l2=1e-2, tag=""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    d = np.abs(gpu - ref)
    rl2 = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30)
    STATS.append({"tag": tag, "max_abs": float(d.max()), "mean_abs": float(d.mean()), "rel_l2": float(rl2),
                  "ref_rms": float(np.sqrt(np.mean(ref * ref)))})
    assert d.max() <= max_abs, f"max-abs {d.max()}"
    assert d.mean() <= mean_abs, f"mean-abs {d.mean()}"
    assert rl2 <= rel_l2, f"relative L2 {rl2}"
    return d.max(), d.mean(), rl2
