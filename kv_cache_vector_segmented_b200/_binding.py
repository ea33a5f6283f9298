"""ctypes binding of libretroinfer.so (the C ABI in include/retroinfer.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, and their device pointers plus torch's current CUDA stream are
passed to the library.  Every step of the path runs in the library's CUDA
kernels; there is no fallback.  Importing works without a GPU (host-only calls
such as geometry and budget queries run anywhere); compute calls need CUDA.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import re
from typing import Optional

import numpy as np

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libretroinfer.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m kv_cache_vector_segmented_b200.build` "
        "(nvcc, sm_100a). The wave-index path has no CPU fallback.")

lib = ctypes.CDLL(LIB_PATH)

RI_OK = 0
STATUS_NAMES = {0: "RI_OK", 1: "RI_ERR_INVALID_ARG", 2: "RI_ERR_UNSUPPORTED",
                3: "RI_ERR_WORKSPACE", 4: "RI_ERR_CAPACITY", 5: "RI_ERR_CUDA",
                6: "RI_ERR_TIMEOUT", 7: "RI_ERR_HOST"}
STATUS_CODES = {v: k for k, v in STATUS_NAMES.items()}


class RIError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.ri_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")


class IndexConfig(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("group_size", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("seq_len", ctypes.c_int32), ("seg_len", ctypes.c_int32),
                ("clusters_per_seg", ctypes.c_int32), ("iters", ctypes.c_int32),
                ("steady_initial", ctypes.c_int32), ("steady_recent", ctypes.c_int32),
                ("base_len", ctypes.c_int32), ("capacity", ctypes.c_int32)]

    @classmethod
    def make(cls, batch: int, num_kv_heads: int, group_size: int, seq_len: int,
             seg_len: int = 8192, clusters_per_seg: int = 512, iters: int = 10,
             steady_initial: int = 4, steady_recent: int = 64, head_dim: int = 128,
             base_len: int = 0, capacity: int = 0):
        return cls(batch, num_kv_heads, group_size, head_dim, seq_len, seg_len,
                   clusters_per_seg, iters, steady_initial, steady_recent, base_len, capacity)

    def copy(self) -> "IndexConfig":
        return IndexConfig(*[getattr(self, f) for f, _ in self._fields_])


class Geometry(ctypes.Structure):
    _fields_ = [("middle", ctypes.c_int32), ("num_segments", ctypes.c_int32),
                ("clusters", ctypes.c_int32), ("steady", ctypes.c_int32),
                ("cluster_stride", ctypes.c_int32), ("row_stride", ctypes.c_int32)]


class CIndex(ctypes.Structure):
    _fields_ = [("Kp", ctypes.c_void_p), ("Vp", ctypes.c_void_p), ("perm", ctypes.c_void_p),
                ("centroid", ctypes.c_void_p), ("counts", ctypes.c_void_p),
                ("offsets", ctypes.c_void_p), ("vsum", ctypes.c_void_p),
                ("Ks", ctypes.c_void_p), ("Vs", ctypes.c_void_p),
                ("labels", ctypes.c_void_p), ("objective", ctypes.c_void_p)]


class DecodeConfig(ctypes.Structure):
    _fields_ = [("k_retrieval", ctypes.c_int32), ("k_estimation", ctypes.c_int32)]


_P = ctypes.POINTER
_vp = ctypes.c_void_p
_sz = ctypes.c_size_t

lib.ri_status_string.restype = ctypes.c_char_p
lib.ri_status_string.argtypes = [ctypes.c_int]
lib.ri_last_error.restype = ctypes.c_char_p
lib.ri_last_error.argtypes = []
lib.ri_index_geometry.restype = ctypes.c_int
lib.ri_index_geometry.argtypes = [_P(IndexConfig), _P(Geometry)]
lib.ri_default_budgets.restype = ctypes.c_int
lib.ri_default_budgets.argtypes = [ctypes.c_int32, _P(DecodeConfig)]
lib.ri_build_index_workspace.restype = _sz
lib.ri_build_index_workspace.argtypes = [_P(IndexConfig)]
lib.ri_build_index.restype = ctypes.c_int
lib.ri_build_index.argtypes = [_P(IndexConfig), _vp, _vp, _vp, _P(CIndex), _vp, _sz, _vp]
lib.ri_decode_workspace.restype = _sz
lib.ri_decode_workspace.argtypes = [_P(IndexConfig), _P(DecodeConfig)]
lib.ri_decode_attention.restype = ctypes.c_int
lib.ri_decode_attention.argtypes = [_P(IndexConfig), _P(DecodeConfig), _vp, _P(CIndex), _vp,
                                    _vp, _vp, _vp, _sz, _vp]
lib.ri_decode_attention_host.restype = ctypes.c_int
lib.ri_decode_attention_host.argtypes = [_P(IndexConfig), _P(DecodeConfig), _vp, _vp, _P(CIndex),
                                         _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
lib.ri_decode_attention_static.restype = ctypes.c_int
lib.ri_decode_attention_static.argtypes = [_P(IndexConfig), _P(DecodeConfig), _vp, _P(CIndex),
                                           _vp, _vp, _vp, _vp, _vp]
lib.ri_select_clusters.restype = ctypes.c_int
lib.ri_select_clusters.argtypes = [_P(IndexConfig), _P(DecodeConfig), _vp, _P(CIndex), _vp,
                                   _vp, _vp, _sz, _vp]
lib.ri_attend_selected.restype = ctypes.c_int
lib.ri_attend_selected.argtypes = [_P(IndexConfig), _P(DecodeConfig), _vp, _P(CIndex), _vp,
                                   _vp, ctypes.c_int32, _vp, _vp, _vp, _sz, _vp]
lib.ri_read_device_status.restype = ctypes.c_int
lib.ri_read_device_status.argtypes = [_vp, _vp]
lib.ri_selftest_wait_timeout.restype = ctypes.c_int
lib.ri_selftest_wait_timeout.argtypes = [_vp, ctypes.c_uint64, _vp]
lib.ri_selftest_decode_timeout.restype = ctypes.c_int
lib.ri_index_open.restype = ctypes.c_int
lib.ri_index_open.argtypes = [_P(IndexConfig), _P(CIndex), _P(CIndex), _vp]
lib.ri_index_append_workspace.restype = ctypes.c_size_t
lib.ri_index_append_workspace.argtypes = [_P(IndexConfig)]
lib.ri_index_append.restype = ctypes.c_int
lib.ri_index_append.argtypes = [_P(IndexConfig), _vp, _vp, _P(CIndex), _vp, _vp, _sz, _vp]
lib.ri_selftest_decode_timeout.argtypes = [_P(IndexConfig), _P(DecodeConfig), _vp, _P(CIndex),
                                           _vp, _vp, _sz, ctypes.c_int32, ctypes.c_uint64, _vp]


class CopyDesc(ctypes.Structure):
    _fields_ = [("unit", ctypes.c_int32), ("src_kind", ctypes.c_int32),
                ("src_row", ctypes.c_int32), ("dst_kind", ctypes.c_int32),
                ("dst_row", ctypes.c_int32), ("n_rows", ctypes.c_int32)]


class CacheConfig(ctypes.Structure):
    _fields_ = [("units", ctypes.c_int32), ("blocks_per_unit", ctypes.c_int32),
                ("block_rows", ctypes.c_int32)]


class CacheStats(ctypes.Structure):
    _fields_ = [("hit_clusters", ctypes.c_int64), ("miss_clusters", ctypes.c_int64),
                ("uncached_clusters", ctypes.c_int64), ("hit_rows", ctypes.c_int64),
                ("miss_rows", ctypes.c_int64), ("empty_clusters", ctypes.c_int64)]


class GatherBuffers(ctypes.Structure):
    _fields_ = [("host_K", _vp), ("host_V", _vp), ("cache_K", _vp), ("cache_V", _vp),
                ("exec_K", _vp), ("exec_V", _vp), ("units", ctypes.c_int32),
                ("M", ctypes.c_int32), ("pool_rows", ctypes.c_int32),
                ("exec_rows", ctypes.c_int32)]


SRC_HOST, SRC_CACHE, SRC_EXEC = 0, 1, 2
DST_EXEC, DST_CACHE = 0, 1

lib.ri_cache_create.restype = ctypes.c_int
lib.ri_cache_create.argtypes = [_P(CacheConfig), _P(_vp)]
lib.ri_cache_destroy.restype = None
lib.ri_cache_destroy.argtypes = [_vp]
lib.ri_cache_plan.restype = ctypes.c_int
lib.ri_cache_plan.argtypes = [_vp, _vp, ctypes.c_int32, ctypes.c_int32, _vp, _vp,
                              ctypes.c_int32, _vp, ctypes.c_int32, _P(ctypes.c_int32), _vp,
                              ctypes.c_int32, _P(ctypes.c_int32), _P(CacheStats)]
lib.ri_max_retrieval_rows.restype = ctypes.c_int
lib.ri_max_retrieval_rows.argtypes = [_vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _vp]
lib.ri_gather_blocks.restype = ctypes.c_int
lib.ri_gather_blocks.argtypes = [_P(GatherBuffers), _vp, ctypes.c_int32, _vp, _vp]
lib.ri_gather_blocks_shaped.restype = ctypes.c_int
lib.ri_gather_blocks_shaped.argtypes = [_P(GatherBuffers), _vp, ctypes.c_int32, ctypes.c_int32,
                                        ctypes.c_int32, _vp, _vp]
lib.ri_gather_shape.restype = ctypes.c_int
lib.ri_gather_shape.argtypes = [ctypes.c_int64, ctypes.c_int64, _P(ctypes.c_int32),
                                _P(ctypes.c_int32)]
lib.ri_cache_resident.restype = ctypes.c_int
lib.ri_cache_resident.argtypes = [_vp, ctypes.c_int32, ctypes.c_int32, _vp, ctypes.c_int32,
                                  _P(ctypes.c_int32)]
lib.ri_cache_validate.restype = ctypes.c_int
lib.ri_cache_validate.argtypes = [_vp]


class CacheWorkerConfig(ctypes.Structure):
    _fields_ = [("bufs", GatherBuffers), ("admit_dev", _vp), ("admit_host", _vp),
                ("admit_cap", ctypes.c_int32), ("gather_workspace", _vp),
                ("side_stream", _vp), ("device", ctypes.c_int32),
                ("wait_limit_ns", ctypes.c_uint64), ("lookup_threads", ctypes.c_int32)]


lib.ri_cache_worker_create.restype = ctypes.c_int
lib.ri_cache_worker_create.argtypes = [_vp, _P(CacheWorkerConfig), _P(_vp)]
lib.ri_cache_worker_destroy.restype = ctypes.c_int
lib.ri_cache_worker_destroy.argtypes = [_vp]
lib.ri_cache_lookup.restype = ctypes.c_int
lib.ri_cache_lookup.argtypes = [_vp, _vp, ctypes.c_int32, ctypes.c_int32, _vp, _vp,
                                ctypes.c_int32, _vp, ctypes.c_int32, _P(ctypes.c_int32),
                                _P(CacheStats), _vp]
lib.ri_cache_update_async.restype = ctypes.c_int
lib.ri_cache_update_async.argtypes = [_vp, _vp]
lib.ri_cache_worker_wait.restype = ctypes.c_int
lib.ri_cache_worker_wait.argtypes = [_vp, _P(CacheStats), _P(ctypes.c_int32)]
lib.ri_cache_worker_test_hooks.restype = ctypes.c_int
lib.ri_cache_worker_test_hooks.argtypes = [_vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_uint32]


def check(status: int, where: str) -> None:
    if status != RI_OK:
        raise RIError(status, where)


def geometry(cfg: IndexConfig) -> Geometry:
    g = Geometry()
    check(lib.ri_index_geometry(ctypes.byref(cfg), ctypes.byref(g)), "ri_index_geometry")
    return g


def default_budgets(clusters: int) -> DecodeConfig:
    d = DecodeConfig()
    check(lib.ri_default_budgets(clusters, ctypes.byref(d)), "ri_default_budgets")
    return d


def build_workspace_bytes(cfg: IndexConfig) -> int:
    n = lib.ri_build_index_workspace(ctypes.byref(cfg))
    if n == 0:
        raise RIError(STATUS_CODES["RI_ERR_INVALID_ARG"], "ri_build_index_workspace")
    return n


def decode_workspace_bytes(cfg: IndexConfig, dcfg: DecodeConfig) -> int:
    n = lib.ri_decode_workspace(ctypes.byref(cfg), ctypes.byref(dcfg))
    if n == 0:
        raise RIError(STATUS_CODES["RI_ERR_INVALID_ARG"], "ri_decode_workspace")
    return n


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape: tuple, device=None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """Caller-owned scratch for the library, 1024-byte aligned, with its
    status region (the first 256 bytes) zeroed."""
    raw = torch.empty(nbytes + 1024, dtype=torch.uint8, device=device)
    off = (-raw.data_ptr()) % 1024
    ws = raw[off:off + nbytes]
    ws[:min(256, nbytes)].zero_()
    return ws


@dataclasses.dataclass
class Index:
    """Device tensors of a wave index (layouts as in include/retroinfer.h)."""

    cfg: IndexConfig
    geom: Geometry
    Kp: torch.Tensor
    Vp: torch.Tensor
    perm: torch.Tensor
    centroid: torch.Tensor
    counts: torch.Tensor
    offsets: torch.Tensor
    vsum: torch.Tensor
    Ks: torch.Tensor
    Vs: torch.Tensor
    labels: Optional[torch.Tensor] = None
    objective: Optional[torch.Tensor] = None

    def c_struct(self) -> CIndex:
        return CIndex(_ptr(self.Kp), _ptr(self.Vp), _ptr(self.perm), _ptr(self.centroid),
                      _ptr(self.counts), _ptr(self.offsets), _ptr(self.vsum), _ptr(self.Ks),
                      _ptr(self.Vs), _ptr(self.labels), _ptr(self.objective))

    @property
    def device(self) -> torch.device:
        return self.offsets.device

    @classmethod
    def empty(cls, cfg: IndexConfig, device, labels: bool = True, objective: bool = True):
        g = geometry(cfg)
        B, H, d = cfg.batch, cfg.num_kv_heads, cfg.head_dim
        M, C, S, ns = g.row_stride, g.cluster_stride, g.num_segments, g.steady
        bf, i32, f32 = torch.bfloat16, torch.int32, torch.float32
        return cls(cfg=cfg, geom=g,
                   Kp=torch.empty((B, H, M, d), dtype=bf, device=device),
                   Vp=torch.empty((B, H, M, d), dtype=bf, device=device),
                   perm=torch.empty((B, H, M), dtype=i32, device=device),
                   centroid=torch.empty((B, H, C, d), dtype=bf, device=device),
                   counts=torch.empty((B, H, C), dtype=i32, device=device),
                   offsets=torch.empty((B, H, C + 1), dtype=i32, device=device),
                   vsum=torch.empty((B, H, C, d), dtype=f32, device=device),
                   Ks=torch.empty((B, H, ns, d), dtype=bf, device=device),
                   Vs=torch.empty((B, H, ns, d), dtype=bf, device=device),
                   labels=torch.empty((B, H, M), dtype=i32, device=device) if labels else None,
                   objective=torch.empty((B, H, S), dtype=f32, device=device) if objective else None)

    def check_shapes(self) -> None:
        cfg, g = self.cfg, self.geom
        B, H, d = cfg.batch, cfg.num_kv_heads, cfg.head_dim
        M, C, ns = g.row_stride, g.cluster_stride, g.steady
        dev = self.device
        _need(self.Kp, "Kp", torch.bfloat16, (B, H, M, d), dev)
        _need(self.Vp, "Vp", torch.bfloat16, (B, H, M, d), dev)
        _need(self.perm, "perm", torch.int32, (B, H, M), dev)
        _need(self.centroid, "centroid", torch.bfloat16, (B, H, C, d), dev)
        _need(self.counts, "counts", torch.int32, (B, H, C), dev)
        _need(self.offsets, "offsets", torch.int32, (B, H, C + 1), dev)
        _need(self.vsum, "vsum", torch.float32, (B, H, C, d), dev)
        _need(self.Ks, "Ks", torch.bfloat16, (B, H, ns, d), dev)
        _need(self.Vs, "Vs", torch.bfloat16, (B, H, ns, d), dev)


def build_index(K: torch.Tensor, V: torch.Tensor, cfg: IndexConfig,
                init_pos: Optional[torch.Tensor] = None, out: Optional[Index] = None,
                workspace: Optional[torch.Tensor] = None) -> Index:
    """Segmented k-means index build (ri_build_index) on K's device and torch's
    current stream.  Asynchronous; returns the (possibly given) Index."""
    dev = K.device
    if dev.type != "cuda":
        raise ValueError("build_index needs CUDA tensors")
    B, H, N, d = cfg.batch, cfg.num_kv_heads, cfg.seq_len, cfg.head_dim
    _need(K, "K", torch.bfloat16, (B, H, N, d), dev)
    _need(V, "V", torch.bfloat16, (B, H, N, d), dev)
    g = geometry(cfg)
    if init_pos is not None:
        _need(init_pos, "init_pos", torch.int32, (B, H, g.clusters), dev)
    idx = out if out is not None else Index.empty(cfg, dev)
    idx.check_shapes()
    nbytes = build_workspace_bytes(cfg)
    ws = workspace if workspace is not None else alloc_workspace(nbytes, dev)
    cidx = idx.c_struct()
    check(lib.ri_build_index(ctypes.byref(cfg), K.data_ptr(), V.data_ptr(), _ptr(init_pos),
                             ctypes.byref(cidx), ws.data_ptr(), ws.numel(), _stream(dev)),
          "ri_build_index")
    idx._build_ws = ws  # keep the status word reachable
    return idx


def decode(q: torch.Tensor, index: Index, dcfg: Optional[DecodeConfig] = None,
           workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
           lse: Optional[torch.Tensor] = None, want_lse: bool = True,
           want_sel: bool = False):
    """One tripartite decode step (ri_decode_attention).  Returns
    (out bf16 [B][H_q][d], lse fp32 [B][H_q] or None, sel int32 or None)."""
    cfg = index.cfg
    dev = index.device
    B, H, G, d = cfg.batch, cfg.num_kv_heads, cfg.group_size, cfg.head_dim
    _need(q, "q", torch.bfloat16, (B, H * G, d), dev)
    if dcfg is None:
        dcfg = default_budgets(index.geom.clusters)
    nbytes = decode_workspace_bytes(cfg, dcfg)
    ws = workspace if workspace is not None else alloc_workspace(nbytes, dev)
    if ws.numel() < nbytes:
        raise ValueError(f"workspace needs {nbytes} bytes")
    if out is None:
        out = torch.empty((B, H * G, d), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (B, H * G, d), dev)
    if lse is None and want_lse:
        lse = torch.empty((B, H * G), dtype=torch.float32, device=dev)
    sel = (torch.empty((B, H, dcfg.k_retrieval + dcfg.k_estimation), dtype=torch.int32,
                       device=dev) if want_sel else None)
    cidx = index.c_struct()
    check(lib.ri_decode_attention(ctypes.byref(cfg), ctypes.byref(dcfg), q.data_ptr(),
                                  ctypes.byref(cidx), out.data_ptr(), _ptr(lse), _ptr(sel),
                                  ws.data_ptr(), ws.numel(), _stream(dev)),
          "ri_decode_attention")
    return out, lse, sel


def index_open(compact: Index, capacity: int) -> Index:
    """ri_index_open: a growing copy of a compact index (built over the
    prefill), with room for `capacity` tokens per sequence."""
    c = compact.cfg
    cfg = IndexConfig.make(c.batch, c.num_kv_heads, c.group_size, c.seq_len, c.seg_len,
                           c.clusters_per_seg, c.iters, c.steady_initial, c.steady_recent,
                           c.head_dim, base_len=c.seq_len, capacity=capacity)
    dev = compact.device
    out = Index.empty(cfg, dev, labels=False, objective=False)
    cc, co = compact.c_struct(), out.c_struct()
    check(lib.ri_index_open(ctypes.byref(cfg), ctypes.byref(cc), ctypes.byref(co), _stream(dev)),
          "ri_index_open")
    return out


def index_append_workspace_bytes(cfg: IndexConfig) -> int:
    n = lib.ri_index_append_workspace(ctypes.byref(cfg))
    if n == 0:
        raise RIError(STATUS_CODES["RI_ERR_INVALID_ARG"], "ri_index_append_workspace")
    return n


def index_append(index: Index, k_new: torch.Tensor, v_new: torch.Tensor,
                 workspace: torch.Tensor, assigned: Optional[torch.Tensor] = None) -> None:
    """ri_index_append for token index.cfg.seq_len (k_new, v_new bf16
    [B][H_kv][d]); advances index.cfg.seq_len and index.geom by one."""
    cfg = index.cfg
    dev = index.device
    B, H, d = cfg.batch, cfg.num_kv_heads, cfg.head_dim
    _need(k_new, "k_new", torch.bfloat16, (B, H, d), dev)
    _need(v_new, "v_new", torch.bfloat16, (B, H, d), dev)
    if assigned is not None:
        _need(assigned, "assigned", torch.int32, (B, H), dev)
    cidx = index.c_struct()
    check(lib.ri_index_append(ctypes.byref(cfg), k_new.data_ptr(), v_new.data_ptr(),
                              ctypes.byref(cidx), _ptr(assigned), workspace.data_ptr(),
                              workspace.numel(), _stream(dev)),
          "ri_index_append")
    cfg.seq_len += 1
    index.geom = geometry(cfg)


class Decoder:
    """ri_decode_attention with the arguments marshalled once: a fixed index,
    budgets, workspace and output tensors; each call passes only the query's
    device pointer (same checks on the query's shape, dtype and device as
    `decode`).  For callers that decode step after step on one layer."""

    def __init__(self, index: Index, dcfg: Optional[DecodeConfig] = None,
                 workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, want_lse: bool = True):
        cfg = index.cfg
        dev = index.device
        B, H, G, d = cfg.batch, cfg.num_kv_heads, cfg.group_size, cfg.head_dim
        self.dcfg = dcfg if dcfg is not None else default_budgets(index.geom.clusters)
        nbytes = decode_workspace_bytes(cfg, self.dcfg)
        self.ws = workspace if workspace is not None else alloc_workspace(nbytes, dev)
        if self.ws.numel() < nbytes:
            raise ValueError(f"workspace needs {nbytes} bytes")
        self.out = out if out is not None else torch.empty((B, H * G, d), dtype=torch.bfloat16,
                                                            device=dev)
        _need(self.out, "out", torch.bfloat16, (B, H * G, d), dev)
        if lse is None and want_lse:
            lse = torch.empty((B, H * G), dtype=torch.float32, device=dev)
        self.lse = lse
        self.index, self.dev = index, dev
        self._qshape = (B, H * G, d)
        self._cfg, self._cidx = cfg, index.c_struct()
        self._args = (ctypes.byref(cfg), ctypes.byref(self.dcfg))
        self._tail = (ctypes.byref(self._cidx), self.out.data_ptr(), _ptr(self.lse), None,
                      self.ws.data_ptr(), self.ws.numel())

    def __call__(self, q: torch.Tensor, stream: Optional[torch.cuda.Stream] = None):
        if q.dtype != torch.bfloat16 or q.device != self.dev or \
                tuple(q.shape) != self._qshape or not q.is_contiguous():
            _need(q, "q", torch.bfloat16, self._qshape, self.dev)
        s = (stream or torch.cuda.current_stream(self.dev)).cuda_stream
        check(lib.ri_decode_attention(*self._args, q.data_ptr(), *self._tail, s),
              "ri_decode_attention")
        return self.out, self.lse

    def step_host(self, q_host: torch.Tensor, out_host: torch.Tensor,
                  stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """One step with host buffers (ri_decode_attention_host): q_host is
        copied to the device, the step runs, the output comes back into
        out_host (both CPU bf16 tensors of the query's shape, page-locked for
        asynchronous copies); returns out_host once it holds the output."""
        for t, name in ((q_host, "q_host"), (out_host, "out_host")):
            if t.device.type != "cpu" or t.dtype != torch.bfloat16 or \
                    tuple(t.shape) != self._qshape or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous CPU bfloat16 tensor of shape "
                                 f"{self._qshape}")
        if not hasattr(self, "_qdev"):
            self._qdev = torch.empty(self._qshape, dtype=torch.bfloat16, device=self.dev)
        s = (stream or torch.cuda.current_stream(self.dev)).cuda_stream
        check(lib.ri_decode_attention_host(*self._args, q_host.data_ptr(), self._qdev.data_ptr(),
                                           ctypes.byref(self._cidx), self.out.data_ptr(),
                                           out_host.data_ptr(), _ptr(self.lse),
                                           self.ws.data_ptr(), self.ws.numel(), s),
              "ri_decode_attention_host")
        return out_host


STATIC_SCRATCH_BYTES = 4 << 20  # RI_STATIC_SCRATCH_BYTES


def decode_static(q: torch.Tensor, index: Index, dcfg: Optional[DecodeConfig] = None,
                  out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                  want_lse: bool = True, want_sel: bool = False,
                  device_status: Optional[torch.Tensor] = None):
    """ri_decode_attention_static: one decode step whose scratch is the
    library's fixed device array (no workspace argument).  Returns
    (out, lse or None, sel or None)."""
    cfg = index.cfg
    dev = index.device
    B, H, G, d = cfg.batch, cfg.num_kv_heads, cfg.group_size, cfg.head_dim
    _need(q, "q", torch.bfloat16, (B, H * G, d), dev)
    if dcfg is None:
        dcfg = default_budgets(index.geom.clusters)
    if out is None:
        out = torch.empty((B, H * G, d), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (B, H * G, d), dev)
    if lse is None and want_lse:
        lse = torch.empty((B, H * G), dtype=torch.float32, device=dev)
    sel = (torch.empty((B, H, dcfg.k_retrieval + dcfg.k_estimation), dtype=torch.int32,
                       device=dev) if want_sel else None)
    if device_status is not None:
        _need(device_status, "device_status", torch.int32, (1,), dev)
    cidx = index.c_struct()
    # the library uses the current device's array: make the index's device current
    with torch.cuda.device(dev):
        check(lib.ri_decode_attention_static(ctypes.byref(cfg), ctypes.byref(dcfg), q.data_ptr(),
                                             ctypes.byref(cidx), out.data_ptr(), _ptr(lse),
                                             _ptr(sel), _ptr(device_status), _stream(dev)),
              "ri_decode_attention_static")
    return out, lse, sel


def select_clusters(q: torch.Tensor, index: Index, dcfg: DecodeConfig, workspace: torch.Tensor,
                    sel: Optional[torch.Tensor] = None, retr_rows: Optional[torch.Tensor] = None):
    """Steps S1-S2 alone (ri_select_clusters); the selection stays in
    `workspace` for attend_selected.  Returns (sel, retr_rows)."""
    cfg = index.cfg
    dev = index.device
    B, H, G, d = cfg.batch, cfg.num_kv_heads, cfg.group_size, cfg.head_dim
    _need(q, "q", torch.bfloat16, (B, H * G, d), dev)
    k = dcfg.k_retrieval + dcfg.k_estimation
    if sel is None:
        sel = torch.empty((B, H, k), dtype=torch.int32, device=dev)
    if retr_rows is None:
        retr_rows = torch.empty((B, H, dcfg.k_retrieval + 1), dtype=torch.int32, device=dev)
    cidx = index.c_struct()
    check(lib.ri_select_clusters(ctypes.byref(cfg), ctypes.byref(dcfg), q.data_ptr(),
                                 ctypes.byref(cidx), sel.data_ptr(), retr_rows.data_ptr(),
                                 workspace.data_ptr(), workspace.numel(), _stream(dev)),
          "ri_select_clusters")
    return sel, retr_rows


def attend_selected(q: torch.Tensor, index: Index, dcfg: DecodeConfig, workspace: torch.Tensor,
                    exec_K: Optional[torch.Tensor] = None, exec_V: Optional[torch.Tensor] = None,
                    out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None):
    """Steps S4-S6 on the selection in `workspace` (ri_attend_selected)."""
    cfg = index.cfg
    dev = index.device
    B, H, G, d = cfg.batch, cfg.num_kv_heads, cfg.group_size, cfg.head_dim
    _need(q, "q", torch.bfloat16, (B, H * G, d), dev)
    if out is None:
        out = torch.empty((B, H * G, d), dtype=torch.bfloat16, device=dev)
    rows = 0
    if exec_K is not None:
        rows = exec_K.shape[2]
        _need(exec_K, "exec_K", torch.bfloat16, (B, H, rows, d), dev)
        _need(exec_V, "exec_V", torch.bfloat16, (B, H, rows, d), dev)
    cidx = index.c_struct()
    check(lib.ri_attend_selected(ctypes.byref(cfg), ctypes.byref(dcfg), q.data_ptr(),
                                 ctypes.byref(cidx), _ptr(exec_K), _ptr(exec_V), rows,
                                 out.data_ptr(), _ptr(lse), workspace.data_ptr(),
                                 workspace.numel(), _stream(dev)),
          "ri_attend_selected")
    return out, lse


def read_device_status(workspace: torch.Tensor) -> int:
    """Synchronises torch's current stream and returns the workspace status
    (a failure read is cleared)."""
    return lib.ri_read_device_status(workspace.data_ptr(), _stream(workspace.device))


FAULT_SCORE_COPY, FAULT_SCORE_COMMIT, FAULT_SCORE_SIZES = 1, 2, 3


def selftest_decode_timeout(q: torch.Tensor, index: Index, dcfg: DecodeConfig,
                            workspace: torch.Tensor, hand_off: int, limit_ns: int,
                            out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """ri_selftest_decode_timeout: one decode step with one hand-off inside
    the kernel left unreleased and every wait limited to limit_ns."""
    cfg = index.cfg
    dev = index.device
    B, H, G, d = cfg.batch, cfg.num_kv_heads, cfg.group_size, cfg.head_dim
    _need(q, "q", torch.bfloat16, (B, H * G, d), dev)
    if out is None:
        out = torch.empty((B, H * G, d), dtype=torch.bfloat16, device=dev)
    cidx = index.c_struct()
    check(lib.ri_selftest_decode_timeout(ctypes.byref(cfg), ctypes.byref(dcfg), q.data_ptr(),
                                         ctypes.byref(cidx), out.data_ptr(), workspace.data_ptr(),
                                         workspace.numel(), hand_off, limit_ns, _stream(dev)),
          "ri_selftest_decode_timeout")
    return out


def selftest_wait_timeout(workspace: torch.Tensor, limit_ns: int) -> None:
    check(lib.ri_selftest_wait_timeout(workspace.data_ptr(), limit_ns,
                                       _stream(workspace.device)),
          "ri_selftest_wait_timeout")


class BlockCache:
    """Host state of the GPU block cache (ri_cache_*): per unit a mapping
    table cluster -> blocks and an LRU order; the device pool itself is a
    pair of caller-owned tensors [units][blocks_per_unit * block_rows][128]."""

    def __init__(self, units: int, blocks_per_unit: int, block_rows: int = 8):
        self.cfg = CacheConfig(units, blocks_per_unit, block_rows)
        h = _vp()
        check(lib.ri_cache_create(ctypes.byref(self.cfg), ctypes.byref(h)), "ri_cache_create")
        self._h = h
        self._destroy = lib.ri_cache_destroy  # still reachable at interpreter exit

    def _grow(self, cap: int) -> None:
        self._out_cap = cap
        self._fetch = np.empty((cap, 6), dtype=np.int32)
        self._admit = np.empty((cap, 6), dtype=np.int32)

    @property
    def pool_rows(self) -> int:
        return self.cfg.blocks_per_unit * self.cfg.block_rows

    def plan(self, sel_ids: np.ndarray, k_retrieval: int, counts: np.ndarray,
             offsets: np.ndarray):
        """One step (ri_cache_plan) on host arrays: sel_ids int32 [units][stride]
        (R first, id order, -1 padded), counts int32 [units][C], offsets int32
        [units][C + 1].  Returns (fetch int32 [n][6], admit int32 [m][6], stats)."""
        sel = np.ascontiguousarray(sel_ids, dtype=np.int32).reshape(self.cfg.units, -1)
        cnt = np.ascontiguousarray(counts, dtype=np.int32).reshape(self.cfg.units, -1)
        off = np.ascontiguousarray(offsets, dtype=np.int32).reshape(self.cfg.units, -1)
        C = cnt.shape[1]
        # output lists reused across steps (the library writes every entry it
        # reports; the used prefixes are copied out below).  A list that would
        # overflow makes the library refuse with RI_ERR_CAPACITY and leave its
        # state unchanged: grow and plan again.
        if getattr(self, "_out_cap", 0) < 1:
            self._grow(max(1024, 4 * self.cfg.units * max(1, k_retrieval)))
        nf, na = ctypes.c_int32(0), ctypes.c_int32(0)
        st = CacheStats()
        while True:
            rc = lib.ri_cache_plan(self._h, sel.ctypes.data, sel.shape[1], k_retrieval,
                                   cnt.ctypes.data, off.ctypes.data, C, self._fetch.ctypes.data,
                                   self._out_cap, ctypes.byref(nf), self._admit.ctypes.data,
                                   self._out_cap, ctypes.byref(na), ctypes.byref(st))
            if rc != STATUS_CODES["RI_ERR_CAPACITY"]:
                break
            self._grow(2 * self._out_cap)
        check(rc, "ri_cache_plan")
        fetch, admit = self._fetch, self._admit
        stats = {f: getattr(st, f) for f, _ in CacheStats._fields_}
        return fetch[:nf.value].copy(), admit[:na.value].copy(), stats

    def resident(self, unit: int, cluster: int) -> list:
        """Blocks holding a cluster, in row order ([] when not resident)."""
        buf = np.zeros(64, dtype=np.int32)
        n = ctypes.c_int32(0)
        rc = lib.ri_cache_resident(self._h, unit, cluster, buf.ctypes.data, buf.size,
                                   ctypes.byref(n))
        if rc == STATUS_CODES["RI_ERR_CAPACITY"]:
            buf = np.zeros(n.value, dtype=np.int32)
            rc = lib.ri_cache_resident(self._h, unit, cluster, buf.ctypes.data, buf.size,
                                       ctypes.byref(n))
        check(rc, "ri_cache_resident")
        return [int(b) for b in buf[:n.value]]

    def validate(self) -> None:
        """ri_cache_validate: raises RIError naming the first broken invariant."""
        check(lib.ri_cache_validate(self._h), "ri_cache_validate")

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()


class CacheWorker:
    """Asynchronous update path of a BlockCache (ri_cache_worker_*).

    Each step: `lookup` (the critical path: waits for the previous update,
    reads the mapping table, returns the fetch list), the caller's fetch
    gather on `stream`, then `update_async` (the worker thread applies the
    LRU replacement and, with device buffers, runs the admit copies on its
    side stream).  Without exec_K / cache_K the worker is host-only: no device
    work, the admit list of the last update is returned by `wait`."""

    def __init__(self, cache: BlockCache, admit_cap: Optional[int] = None, *,
                 host_K: Optional[torch.Tensor] = None, host_V: Optional[torch.Tensor] = None,
                 cache_K: Optional[torch.Tensor] = None, cache_V: Optional[torch.Tensor] = None,
                 exec_K: Optional[torch.Tensor] = None, exec_V: Optional[torch.Tensor] = None,
                 gather_workspace: Optional[torch.Tensor] = None,
                 side_stream: Optional[torch.cuda.Stream] = None, wait_limit_ns: int = 0,
                 lookup_threads: int = 0):
        self.cache = cache
        units = cache.cfg.units
        self.device_mode = exec_K is not None
        cfg = CacheWorkerConfig()
        cfg.wait_limit_ns = wait_limit_ns
        cfg.lookup_threads = lookup_threads
        if self.device_mode:
            dev = exec_K.device
            B, H, rows, d = exec_K.shape
            if admit_cap is None:
                admit_cap = max(1, units * rows)  # ceil(n / block_rows) <= n per cluster
            if not (host_K.is_pinned() and host_V.is_pinned()):
                raise ValueError("host_K and host_V must be pinned")
            _need(exec_V, "exec_V", torch.bfloat16, tuple(exec_K.shape), dev)
            _need(cache_K, "cache_K", torch.bfloat16, (B, H, cache.pool_rows, d), dev)
            _need(cache_V, "cache_V", torch.bfloat16, (B, H, cache.pool_rows, d), dev)
            self._admit_dev = torch.empty((admit_cap, 6), dtype=torch.int32, device=dev)
            self._admit_host = torch.empty((admit_cap, 6), dtype=torch.int32).pin_memory()
            self._side = side_stream or torch.cuda.Stream(dev)
            self._gws = gather_workspace if gather_workspace is not None else \
                alloc_workspace(256, dev)
            self._keep = (host_K, host_V, cache_K, cache_V, exec_K, exec_V)
            cfg.bufs = GatherBuffers(host_K.data_ptr(), host_V.data_ptr(), cache_K.data_ptr(),
                                     cache_V.data_ptr(), exec_K.data_ptr(), exec_V.data_ptr(),
                                     B * H, host_K.shape[2], cache.pool_rows, rows)
            cfg.admit_dev = self._admit_dev.data_ptr()
            cfg.admit_host = self._admit_host.data_ptr()
            cfg.gather_workspace = self._gws.data_ptr()
            cfg.side_stream = self._side.cuda_stream
            cfg.device = dev.index if dev.index is not None else torch.cuda.current_device()
            self.dev = dev
            self._admit_np = self._admit_host.numpy()
        else:
            if admit_cap is None:
                raise ValueError("a host-only worker needs admit_cap")
            self._admit_np = np.empty((admit_cap, 6), dtype=np.int32)
            cfg.admit_host = self._admit_np.ctypes.data
            self.dev = None
        cfg.admit_cap = admit_cap
        self._cfg = cfg
        self._fetch_cap = 0
        self._fetch_copied = None  # event after the last H2D copy of the fetch list
        h = _vp()
        check(lib.ri_cache_worker_create(cache._h, ctypes.byref(cfg), ctypes.byref(h)),
              "ri_cache_worker_create")
        self._h = h
        self._destroy = lib.ri_cache_worker_destroy

    def _grow_fetch(self, cap: int) -> None:
        if self._fetch_copied is not None:
            self._fetch_copied.synchronize()
        self._fetch_cap = cap
        if self.device_mode:
            self._fetch_host = torch.empty((cap, 6), dtype=torch.int32).pin_memory()
            self._fetch_np = self._fetch_host.numpy()
            self._fetch_dev = torch.empty((cap, 6), dtype=torch.int32, device=self.dev)
        else:
            self._fetch_np = np.empty((cap, 6), dtype=np.int32)

    def _stream_ptr(self, stream) -> int:
        if not self.device_mode:
            return 0
        return (stream or torch.cuda.current_stream(self.dev)).cuda_stream

    def lookup(self, sel_ids: np.ndarray, k_retrieval: int, counts: np.ndarray,
               offsets: np.ndarray, stream: Optional[torch.cuda.Stream] = None):
        """ri_cache_lookup.  Returns (fetch int32 [n][6] numpy view, valid until the
        next lookup, and the lookup stats)."""
        units = self.cache.cfg.units
        sel = np.ascontiguousarray(sel_ids, dtype=np.int32).reshape(units, -1)
        cnt = np.ascontiguousarray(counts, dtype=np.int32).reshape(units, -1)
        off = np.ascontiguousarray(offsets, dtype=np.int32).reshape(units, -1)
        if self._fetch_cap < 1:
            self._grow_fetch(max(1024, 4 * units * max(1, k_retrieval)))
        elif self._fetch_copied is not None:
            self._fetch_copied.synchronize()  # the pinned list is read by the last copy
        nf = ctypes.c_int32(0)
        st = CacheStats()
        while True:
            rc = lib.ri_cache_lookup(self._h, sel.ctypes.data, sel.shape[1], k_retrieval,
                                     cnt.ctypes.data, off.ctypes.data, cnt.shape[1],
                                     self._fetch_np.ctypes.data, self._fetch_cap,
                                     ctypes.byref(nf), ctypes.byref(st),
                                     self._stream_ptr(stream))
            if rc != STATUS_CODES["RI_ERR_CAPACITY"]:
                break
            # a list that could overflow is refused with the state unchanged:
            # grow the fetch list when it is the one, and look up again
            m = re.match(r"cache lookup: (\d+) fetch / up to \d+ admit", lib_last_error())
            if not m or int(m.group(1)) <= self._fetch_cap:
                break
            self._grow_fetch(int(m.group(1)))
        check(rc, "ri_cache_lookup")
        self._n_fetch = nf.value
        return self._fetch_np[:nf.value], {f: getattr(st, f) for f, _ in CacheStats._fields_}

    def fetch_to_device(self, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """The last lookup's fetch list copied (non-blocking, pinned) to the
        device on `stream`: int32 [n][6]."""
        s = stream or torch.cuda.current_stream(self.dev)
        n = self._n_fetch
        with torch.cuda.stream(s):
            self._fetch_dev[:n].copy_(self._fetch_host[:n], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(s)
        self._fetch_copied = ev
        return self._fetch_dev[:n]

    def update_async(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        check(lib.ri_cache_update_async(self._h, self._stream_ptr(stream)),
              "ri_cache_update_async")

    def wait(self):
        """ri_cache_worker_wait: (stats of the last update, its admit list)."""
        st = CacheStats()
        na = ctypes.c_int32(0)
        check(lib.ri_cache_worker_wait(self._h, ctypes.byref(st), ctypes.byref(na)),
              "ri_cache_worker_wait")
        return {f: getattr(st, f) for f, _ in CacheStats._fields_}, \
            self._admit_np[:na.value].copy()

    def test_hooks(self, fail_update: int = -1, fail_after: int = 0, delay_us: int = 0) -> None:
        check(lib.ri_cache_worker_test_hooks(self._h, fail_update, fail_after, delay_us),
              "ri_cache_worker_test_hooks")

    def close(self) -> None:
        """Stops the worker (after every handed-over update); raises RIError
        for a failure not yet reported."""
        if getattr(self, "_h", None):
            h, self._h = self._h, None
            check(self._destroy(h), "ri_cache_worker_destroy")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def lib_last_error() -> str:
    return lib.ri_last_error().decode()


def max_retrieval_rows(counts: np.ndarray, k_retrieval: int) -> np.ndarray:
    """ri_max_retrieval_rows on host sizes int32 [units][C]: per unit the sum
    of the k_retrieval largest sizes (rows of the execution buffer)."""
    cnt = np.ascontiguousarray(counts, dtype=np.int32)
    cnt = cnt.reshape(-1, cnt.shape[-1])
    out = np.zeros(cnt.shape[0], dtype=np.int32)
    check(lib.ri_max_retrieval_rows(cnt.ctypes.data, cnt.shape[0], cnt.shape[1], k_retrieval,
                                    out.ctypes.data),
          "ri_max_retrieval_rows")
    return out


def gather_shape(host_copies: int, total_copies: int) -> tuple:
    """ri_gather_shape: (threads per block, blocks per SM) for a copy list."""
    t, b = ctypes.c_int32(0), ctypes.c_int32(0)
    check(lib.ri_gather_shape(host_copies, total_copies, ctypes.byref(t), ctypes.byref(b)),
          "ri_gather_shape")
    return t.value, b.value


def gather_blocks(desc: torch.Tensor, host_K: torch.Tensor, host_V: torch.Tensor,
                  exec_K: torch.Tensor, exec_V: torch.Tensor, workspace: torch.Tensor,
                  cache_K: Optional[torch.Tensor] = None,
                  cache_V: Optional[torch.Tensor] = None, shape: Optional[tuple] = None) -> None:
    """ri_gather_blocks: desc int32 [n][6] on the device; host_K/V pinned CPU
    bf16 [B][H][M][d]; exec_K/V device bf16 [B][H][rows][d]; cache_K/V device
    bf16 [B][H][pool_rows][d] or None."""
    dev = exec_K.device
    B, H, rows, d = exec_K.shape
    if not (host_K.is_pinned() and host_V.is_pinned()):
        raise ValueError("host_K and host_V must be pinned")
    _need(desc, "desc", torch.int32, (desc.shape[0], 6), dev)
    _need(exec_V, "exec_V", torch.bfloat16, tuple(exec_K.shape), dev)
    M = host_K.shape[2]
    pool = 0
    if cache_K is not None:
        pool = cache_K.shape[2]
        _need(cache_K, "cache_K", torch.bfloat16, (B, H, pool, d), dev)
        _need(cache_V, "cache_V", torch.bfloat16, (B, H, pool, d), dev)
    bufs = GatherBuffers(host_K.data_ptr(), host_V.data_ptr(), _ptr(cache_K), _ptr(cache_V),
                         exec_K.data_ptr(), exec_V.data_ptr(), B * H, M, pool, rows)
    threads, bps = shape if shape is not None else (0, 0)
    check(lib.ri_gather_blocks_shaped(ctypes.byref(bufs), desc.data_ptr(), desc.shape[0],
                                      threads, bps, workspace.data_ptr(), _stream(dev)),
          "ri_gather_blocks_shaped")
