"""Device-side state of one attention layer (caches + learned parameters).

Holds the torch tensors the C ABI points into and builds the csa_layer_t /
csa_cache_t / csa_params_t structs over them.  Marshalling only.
"""

import numpy as np
import torch

from . import binding as C


def to_device(a, device="cuda"):
    """numpy array -> torch tensor on `device` (bf16 bit patterns travel as int16)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(device)


class LayerState:
    """Caches and parameters of one layer for B sequences."""

    def __init__(self, spec, B, pos0=0, *, entries, window, raw=None, gate=None, idx_keys=None,
                 idx_key_scale=None, pos_bias=None, gamma_kv=None, gamma_q=None, sinks=None, raw_base=0):
        self.spec, self.B, self.pos0 = spec, B, pos0
        self.L = C.layer_from_spec(spec, B, pos0)
        self.entries, self.window, self.raw, self.gate = entries, window, raw, gate
        self.idx_keys, self.idx_key_scale = idx_keys, idx_key_scale
        self.pos_bias, self.gamma_kv, self.gamma_q, self.sinks = pos_bias, gamma_kv, gamma_q, sinks
        self.raw_base = raw_base

    def cache(self) -> C.CsaCache:
        return C.make_cache(self.entries, self.window, self.raw, self.gate, self.idx_keys, self.idx_key_scale,
                            self.raw_base)

    def params(self) -> C.CsaParams:
        return C.make_params(self.pos_bias, self.gamma_kv, self.gamma_q, self.sinks)

    @classmethod
    def from_arrays(cls, spec, B, d, device="cuda", pos0=0, raw_key="raw_ring", gate_key="gate_ring", raw_base=0):
        """Build from a dict of numpy arrays (entries, window, raw/gate rings, idx keys, parameters)."""
        g = lambda k: to_device(d[k], device) if k in d and d[k] is not None else None  # noqa: E731
        return cls(spec, B, pos0, entries=g("entries"), window=g("window"), raw=g(raw_key), gate=g(gate_key),
                   idx_keys=g("idx_k"), idx_key_scale=g("idx_k_scale"),
                   pos_bias=to_device(np.asarray(d["pos_bias"], np.float32), device),
                   gamma_kv=to_device(np.asarray(d["gamma_kv"], np.float32), device),
                   gamma_q=to_device(np.asarray(d["gamma_q"], np.float32), device),
                   sinks=to_device(np.asarray(d["sinks"], np.float32), device), raw_base=raw_base)

    def workspace(self, op, Tq, n_max):
        n = C.csa_workspace_size(self.L, op, Tq, n_max)
        return torch.zeros(max(n, 256), dtype=torch.uint8, device=self.entries.device)
