"""Seeded synthetic inputs for the CSA/HCA attention operator.

This package is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It only draws random numbers and lays them out in the storage
formats the operator reads; it performs none of the operator's arithmetic
(no pooling, normalisation, rotary embedding, scoring, selection or softmax).

Every tensor is drawn from its own counter-based Philox stream (numpy's
``Philox`` bit generator, Salmon et al., SC'11), keyed by the workload's seed
and a fixed per-tensor tag, so each tensor is reproducible on its own.
"""

from .configs import WORKLOADS, Workload, get_workload  # noqa: F401
from .generate import (  # noqa: F401
    decode_inputs,
    prefill_inputs,
    compress_inputs,
    stream,
)
