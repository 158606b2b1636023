"""HATA (hash-aware top-k attention) decode path for NVIDIA B200 (sm_100a).

The compute lives in libhata.so (hand-written CUDA, C ABI in include/hata.h);
``hata`` is its ctypes binding and ``workloads`` draws seeded synthetic
inputs.  Build the library with ``python -m hash_aware_top_hata_b200.build``.
"""
from .hata import (HataError, hata_abi_version, hata_append_code, hata_decode_step,  # noqa: F401
                   hata_decode_workspace_size, hata_dense_decode, hata_dense_workspace_size,
                   hata_dist_row_bytes, hata_hash_keys, hata_status_string,
                   hata_workspace_check)
