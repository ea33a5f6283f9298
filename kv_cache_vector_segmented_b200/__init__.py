"""Wave-index decode path of RetroInfer for NVIDIA B200 (sm_100a).

Python face of the C ABI in include/retroinfer.h (libretroinfer.so, built
in-tree by `python -m kv_cache_vector_segmented_b200.build`).  PyTorch supplies
device memory and streams; every computation runs in the library's kernels.
"""
from ._binding import (  # noqa: F401
    LIB_PATH, CIndex, DecodeConfig, Geometry, Index, IndexConfig, RIError, STATUS_CODES,
    STATUS_NAMES, alloc_workspace, attend_selected, build_index, build_workspace_bytes,
    decode, decode_workspace_bytes, default_budgets, geometry, lib, read_device_status,
    select_clusters, selftest_wait_timeout)
