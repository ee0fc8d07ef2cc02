"""B200-native (sm_100a) CSA / HCA compressed attention: one attention layer of
DeepSeek-V4's hybrid attention behind a C ABI (include/csa.h, libcsa.so).

The compute path is the library's CUDA kernels; this package holds the ctypes
binding (same entry-point names as the C ABI), the in-tree build and a small
device-state helper.  There is no CPU fallback: importing `binding.lib()`
without the built library raises.
"""

from .binding import (  # noqa: F401
    CsaError,
    csa_append,
    csa_compress,
    csa_decode_step,
    csa_device_error,
    csa_index_topk,
    csa_prefill,
    csa_row_bytes,
    csa_sparse_attend,
    csa_version,
    csa_workspace_size,
    hca_attend,
    hca_decode_step,
    lib,
    make_cache,
    make_layer,
    make_params,
)
