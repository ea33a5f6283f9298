"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, derives the same geometry and budgets as the oracle, and rejects bad
arguments before touching the device.  No GPU needed."""
import ctypes
import os
import re
import subprocess

import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def R():
    import kv_cache_vector_segmented_b200 as R
    return R


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn), encoding="utf-8").read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(ri_[a-z0-9_]+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol(R):
    names = _declared_functions()
    assert len(names) >= 12
    out = subprocess.run(["nm", "-D", "--defined-only", R.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\b(ri_[a-z0-9_]+)\b", out))
    missing = names - exported
    assert not missing, f"declared but not exported: {sorted(missing)}"
    for n in names:
        assert hasattr(R.lib, n)


@pytest.mark.parametrize("N", [1, 50, 68, 69, 600, 8192, 8260, 8261, 20000, 131072, 1048576])
def test_geometry_matches_oracle(R, N):
    g = R.geometry(R.IndexConfig.make(1, 8, 4, N))
    m0, M = O.middle_range(N)
    segs = O.segments(M)
    assert g.middle == M
    assert g.num_segments == len(segs)
    assert g.clusters == sum(k for _, _, k in segs)
    assert g.steady == len(O.steady_positions(N))


@pytest.mark.parametrize("C", [0, 1, 27, 28, 55, 56, 512, 8192, 65536, 1000000])
def test_default_budgets_match_oracle(R, C):
    d = R.default_budgets(C)
    assert (d.k_retrieval, d.k_estimation) == O.default_budgets(C)


@pytest.mark.parametrize("field,value", [("batch", 0), ("num_kv_heads", 0), ("group_size", 9),
                                         ("group_size", 0), ("head_dim", 64), ("seq_len", 0),
                                         ("seg_len", 0), ("seg_len", 40000),
                                         ("clusters_per_seg", 513), ("clusters_per_seg", 0),
                                         ("iters", -1), ("steady_recent", -1)])
def test_invalid_config_rejected(R, field, value):
    cfg = R.IndexConfig.make(1, 8, 4, 131072)
    setattr(cfg, field, value)
    with pytest.raises(R.RIError) as e:
        R.geometry(cfg)
    assert e.value.status == R.STATUS_CODES["RI_ERR_INVALID_ARG"]
    assert R.lib.ri_build_index_workspace(ctypes.byref(cfg)) == 0


def _fake_index(R, ptr=4096):
    return R.CIndex(*([ptr] * 9), None, None)


def test_build_rejects_bad_arguments_before_launch(R):
    cfg = R.IndexConfig.make(1, 1, 4, 8192)
    idx = _fake_index(R)
    ws_need = R.build_workspace_bytes(cfg)
    lib = R.lib
    bad = R.STATUS_CODES
    # NULL keys
    assert lib.ri_build_index(ctypes.byref(cfg), None, 4096, None, ctypes.byref(idx), 4096,
                              ws_need, None) == bad["RI_ERR_INVALID_ARG"]
    # misaligned keys
    assert lib.ri_build_index(ctypes.byref(cfg), 4100, 4096, None, ctypes.byref(idx), 4096,
                              ws_need, None) == bad["RI_ERR_INVALID_ARG"]
    assert "aligned" in lib.ri_last_error().decode()
    # workspace too small
    assert lib.ri_build_index(ctypes.byref(cfg), 4096, 4096, None, ctypes.byref(idx), 4096,
                              ws_need - 1, None) == bad["RI_ERR_WORKSPACE"]
    # NULL index member
    idx2 = _fake_index(R)
    idx2.vsum = None
    assert lib.ri_build_index(ctypes.byref(cfg), 4096, 4096, None, ctypes.byref(idx2), 4096,
                              ws_need, None) == bad["RI_ERR_INVALID_ARG"]
    assert "vsum" in lib.ri_last_error().decode()


def test_decode_rejects_bad_arguments_before_launch(R):
    cfg = R.IndexConfig.make(1, 8, 4, 131072)
    d = R.default_budgets(R.geometry(cfg).clusters)
    idx = _fake_index(R)
    need = R.decode_workspace_bytes(cfg, d)
    lib = R.lib
    bad = R.STATUS_CODES
    assert lib.ri_decode_attention(ctypes.byref(cfg), ctypes.byref(d), None, ctypes.byref(idx),
                                   4096, None, None, 4096, need, None) == bad["RI_ERR_INVALID_ARG"]
    assert lib.ri_decode_attention(ctypes.byref(cfg), ctypes.byref(d), 4096, ctypes.byref(idx),
                                   4096, None, None, 4096, need - 4, None) == bad["RI_ERR_WORKSPACE"]
    d2 = R.DecodeConfig(-1, 5)
    assert lib.ri_decode_attention(ctypes.byref(cfg), ctypes.byref(d2), 4096, ctypes.byref(idx),
                                   4096, None, None, 4096, need, None) == bad["RI_ERR_INVALID_ARG"]
    d3 = R.DecodeConfig(9000, 5)
    assert lib.ri_decode_workspace(ctypes.byref(cfg), ctypes.byref(d3)) == 0
    # exec buffers must come in pairs
    assert lib.ri_attend_selected(ctypes.byref(cfg), ctypes.byref(d), 4096, ctypes.byref(idx),
                                  4096, None, 10, 4096, None, 4096, need, None) == bad["RI_ERR_INVALID_ARG"]
    assert lib.ri_selftest_wait_timeout(None, 1000, None) == bad["RI_ERR_INVALID_ARG"]
    # the host-buffer step: host pointers, device output and workspace checked first
    hq = ctypes.create_string_buffer(64)
    assert lib.ri_decode_attention_host(ctypes.byref(cfg), ctypes.byref(d), None, 4096,
                                        ctypes.byref(idx), 4096, hq, None, 4096, need,
                                        None) == bad["RI_ERR_INVALID_ARG"]
    assert "q_host" in lib.ri_last_error().decode()
    assert lib.ri_decode_attention_host(ctypes.byref(cfg), ctypes.byref(d), hq, 4096,
                                        ctypes.byref(idx), None, hq, None, 4096, need,
                                        None) == bad["RI_ERR_INVALID_ARG"]
    assert lib.ri_decode_attention_host(ctypes.byref(cfg), ctypes.byref(d), hq, 4096,
                                        ctypes.byref(idx), 4096, hq, None, 4096, need - 4,
                                        None) == bad["RI_ERR_WORKSPACE"]


def test_status_strings(R):
    for code, name in R.STATUS_NAMES.items():
        s = R.lib.ri_status_string(code).decode()
        assert s and s != "unknown status"
    assert R.lib.ri_status_string(99).decode() == "unknown status"


def test_workspace_sizes_scale(R):
    small = R.build_workspace_bytes(R.IndexConfig.make(1, 1, 4, 8192))
    big = R.build_workspace_bytes(R.IndexConfig.make(1, 8, 4, 131072))
    assert 0 < small < big
    cfg = R.IndexConfig.make(1, 8, 4, 131072)
    d = R.default_budgets(R.geometry(cfg).clusters)
    assert R.decode_workspace_bytes(cfg, d) < 8 << 20


@pytest.mark.parametrize("B,H,N", [(1, 1, 8192 + 68), (2, 3, 20000), (1, 8, 131072)])
def test_build_workspace_holds_every_array(R, B, H, N):
    """The build workspace is at least the sum of the arrays the build uses
    (sizes written out from their shapes): fp32 and bf16 centroids, the
    ||mu||^2 operand tiles, the per-unit maxima, sizes, labels, key norms,
    the fix-up queue (one 20-byte entry per key), the sorted member lists,
    their cluster starts and the per-centroid error terms."""
    g = R.geometry(R.IndexConfig.make(B, H, 4, N))
    BH, C, M = B * H, g.clusters, N - 68
    S = -(-M // 8192)
    need = (BH * C * 128 * 4 + BH * C * 128 * 2 + BH * S * 512 * 16 * 2 + BH * S * 2 * 4
            + BH * C * 4 + BH * M * 4 + BH * M * 4 + BH * M * 20 + BH * M * 4
            + BH * S * 513 * 4 + BH * S * 512 * 8)
    assert R.build_workspace_bytes(R.IndexConfig.make(B, H, 4, N)) >= need


# ---------------------------------------------------------------- growing index
@pytest.mark.parametrize("base_len,appended,seg_len,clusters", [
    (68 + 300, 0, 128, 16), (68 + 300, 127, 128, 16), (68 + 300, 128, 128, 16),
    (68 + 300, 300, 128, 16), (68 + 2 * 8192 + 700, 150, 8192, 512), (69, 5, 8192, 512)])
def test_growing_geometry_matches_oracle(R, base_len, appended, seg_len, clusters):
    """Live clusters of a growing index = the oracle's: the prefill's
    segments, one closed segment per seg_len appended tokens, K open ones."""
    cap = base_len + 400
    cfg = R.IndexConfig.make(1, 2, 4, base_len + appended, seg_len=seg_len,
                             clusters_per_seg=clusters, base_len=base_len, capacity=cap)
    g = R.geometry(cfg)
    pre = O.segments(base_len - 68, seg_len, clusters)
    K = min(clusters, seg_len)
    C = sum(k for _, _, k in pre) + (appended // seg_len) * K + K
    assert g.clusters == C
    assert g.middle == base_len + appended - 68
    Fmax = (cap - base_len) // seg_len
    assert g.cluster_stride == sum(k for _, _, k in pre) + Fmax * K + K
    assert g.row_stride == base_len - 68 + Fmax * seg_len + 2 * seg_len + K


def test_growing_calls_reject_bad_arguments(R):
    import torch
    cfg = R.IndexConfig.make(1, 2, 4, 368, seg_len=128, clusters_per_seg=16, base_len=368,
                             capacity=400)
    # the build makes compact indexes only
    assert R.lib.ri_build_index_workspace(ctypes.byref(cfg)) == 0
    bad = R.IndexConfig.make(1, 2, 4, 368, base_len=400, capacity=500)  # seq_len < base_len
    assert R.lib.ri_index_append_workspace(ctypes.byref(bad)) == 0
    compact = R.IndexConfig.make(1, 2, 4, 368, seg_len=128, clusters_per_seg=16)
    assert R.lib.ri_index_append_workspace(ctypes.byref(compact)) == 0
    full = R.IndexConfig.make(1, 2, 4, 400, seg_len=128, clusters_per_seg=16, base_len=368,
                              capacity=400)
    idx = R.CIndex()
    st = R.lib.ri_index_append(ctypes.byref(full), None, None, ctypes.byref(idx), None, None, 0,
                               None)
    assert st == R.STATUS_CODES["RI_ERR_CAPACITY"]
    st = R.lib.ri_index_append(ctypes.byref(cfg), None, None, ctypes.byref(idx), None, None, 0,
                               None)
    assert st == R.STATUS_CODES["RI_ERR_INVALID_ARG"]
    # open needs the config at its prefill (seq_len == base_len)
    later = R.IndexConfig.make(1, 2, 4, 370, seg_len=128, clusters_per_seg=16, base_len=368,
                               capacity=400)
    st = R.lib.ri_index_open(ctypes.byref(later), ctypes.byref(idx), ctypes.byref(idx), None)
    assert st == R.STATUS_CODES["RI_ERR_INVALID_ARG"]
    assert torch  # noqa


def test_gather_shape_per_hit_pattern(R):
    """Host-link bound lists and device-memory bound lists get their own
    launch shapes; bad counts are refused on the host."""
    host = R.gather_shape(20, 1000)      # any copy from host memory
    dev = R.gather_shape(0, 1000)        # device-only list
    assert host != dev and R.gather_shape(1000, 1000) == host
    for t, b in (host, dev):
        assert t % 32 == 0 and 32 <= t <= 512 and 1 <= b <= 64
    assert R.gather_shape(0, 0) == dev
    with pytest.raises(R.RIError):
        R.gather_shape(5, 4)
    with pytest.raises(R.RIError):
        R.gather_shape(-1, 4)
    bufs = R._binding.GatherBuffers()
    assert R.lib.ri_gather_blocks_shaped(ctypes.byref(bufs), None, 0, 48, 4, None, None) == \
        R.STATUS_CODES["RI_ERR_INVALID_ARG"]           # not a multiple of 32
    assert R.lib.ri_gather_blocks_shaped(ctypes.byref(bufs), None, 0, 1024, 4, None, None) == \
        R.STATUS_CODES["RI_ERR_INVALID_ARG"]           # above 512
