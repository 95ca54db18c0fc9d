"""B200-native (sm_100a) CSA + HCA compressed attention.

The library is libcsahca.so (C ABI in include/csahca.h); ``api`` holds the
torch-facing wrappers with the same names as the C entry points, ``native``
the ctypes mirror, ``synth`` the seeded synthetic inputs.
"""

from .api import (  # noqa: F401
    compressed_attn_decode,
    compressed_attn_prefill,
    csa_compress,
    device_error,
    hca_compress,
    indexer_topk,
)
