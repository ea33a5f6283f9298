"""Wave-index decode path of RetroInfer for NVIDIA B200 (sm_100a).

Python face of the C ABI in include/retroinfer.h (libretroinfer.so, built
in-tree by `python -m kv_cache_vector_segmented_b200.build`).  PyTorch supplies
device memory and streams; every computation runs in the library's kernels.

The library is loaded on first use of any name below, so the build module can
be imported before the library exists; using the API without the library
raises ImportError (there is no fallback).
"""
import importlib

_EXPORTS = (
    "LIB_PATH", "CIndex", "DecodeConfig", "Geometry", "Index", "IndexConfig", "RIError",
    "STATUS_CODES", "STATUS_NAMES", "alloc_workspace", "attend_selected", "build_index",
    "build_workspace_bytes", "decode", "decode_workspace_bytes", "default_budgets", "geometry",
    "lib", "read_device_status", "select_clusters", "selftest_wait_timeout", "decode_static",
    "STATIC_SCRATCH_BYTES", "BlockCache", "CopyDesc", "gather_blocks", "SRC_HOST", "SRC_CACHE",
    "SRC_EXEC", "DST_EXEC", "DST_CACHE", "max_retrieval_rows", "selftest_decode_timeout",
    "FAULT_SCORE_COPY", "FAULT_SCORE_COMMIT", "FAULT_SCORE_SIZES", "CacheWorker",
    "Decoder", "index_open", "index_append", "index_append_workspace_bytes",
    "gather_shape")

__all__ = list(_EXPORTS)


def __getattr__(name):
    if name in _EXPORTS:
        binding = importlib.import_module("._binding", __name__)
        return getattr(binding, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")
