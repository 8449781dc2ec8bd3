"""DSA sparse attention for NVIDIA B200 (sm_100a): indexer -> top-k -> sparse MLA attention.

The compute lives in libdsa.so (hand-written CUDA behind the C ABI in include/dsa.h);
`binding` is a ctypes layer with the same function names, `pipeline.DeviceBatch` keeps a
batch resident in device memory and enqueues the three calls, and `workloads` draws the
seeded synthetic inputs.
"""
from . import binding  # noqa: F401
from .binding import (DSAError, dsa_batch_t, dsa_indexer_scores, dsa_read_device_status,  # noqa: F401
                      dsa_sparse_attn_decode, dsa_sparse_attn_prefill, dsa_topk, dsa_workspace_size, make_batch)

__version__ = "0.1.0"
