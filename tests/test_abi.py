"""C-ABI checks that need no GPU: the library loads, exports every entry point the
header declares, and rejects unsupported geometry on the host (fail closed)
before any CUDA work."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for f in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if f.endswith(".h"):
            with open(os.path.join(ROOT, "include", f)) as fh:
                src = fh.read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(ssd_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("ssd_scan_fwd", "ssd_state_update", "ssd_scan_fwd_workspace_size",
              "ssd_get_device_status", "ssd_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(ssd):
    lib = ctypes.CDLL(ssd.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def _dims(ssd, **kw):
    base = dict(T=256, H=8, P=64, G=2, N=128, dtype_code=ssd.SSD_DTYPE_BF16, batch=1, seqlen=256)
    base.update(kw)
    return ssd.make_dims(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(H=6, G=4), "UNSUPPORTED"),        # H % G != 0
    (dict(P=48), "UNSUPPORTED"),
    (dict(P=256), "UNSUPPORTED"),
    (dict(N=8), "UNSUPPORTED"),
    (dict(N=96), "UNSUPPORTED"),
    (dict(H=0), "INVALID_ARG"),
    (dict(batch=-1), "INVALID_ARG"),
])
def test_bad_geometry_fails_closed(ssd, kw, status):
    d = _dims(ssd, **kw)
    if "batch" not in kw:         # the size query also accepts the packed reading of dims
        with pytest.raises(ssd.SSDError, match=status):
            ssd.workspace_size(d, 128)
    rc = ssd._lib.ssd_scan_fwd(None, None, None, None, None, None, None, None, None, None, None,
                               ctypes.byref(d), 128, None)
    assert rc == getattr(ssd, "SSD_ERR_" + status)
    assert ssd._lib.ssd_last_error().decode()
    if "batch" not in kw:
        assert ssd.scan_variant(d, 128) == ""


@pytest.mark.parametrize("chunk", [0, 32, 100, 512])
def test_bad_chunk_fails_closed(ssd, chunk):
    with pytest.raises(ssd.SSDError, match="UNSUPPORTED"):
        ssd.workspace_size(_dims(ssd), chunk)


def test_null_and_misaligned_pointers_rejected_on_host(ssd):
    d = _dims(ssd)
    p = 1 << 20                       # never dereferenced: validation stops first
    rc = ssd._lib.ssd_scan_fwd(p, p, p, p, p, p, p, None, None, None, None, ctypes.byref(d), 128, None)
    assert rc == ssd.SSD_ERR_INVALID_ARG          # y is NULL
    rc = ssd._lib.ssd_scan_fwd(p + 2, p, p, p, p, p, p, None, None, p, None, ctypes.byref(d), 128, None)
    assert rc == ssd.SSD_ERR_INVALID_ARG          # x misaligned
    d1 = _dims(ssd, seqlen=2)
    rc = ssd._lib.ssd_state_update(p, p, p, p, p, p, p, p, p, ctypes.byref(d1), None)
    assert rc == ssd.SSD_ERR_INVALID_ARG          # decode needs seqlen == 1
    too_small = _dims(ssd)
    too_small.workspace, too_small.workspace_bytes = p, 16
    rc = ssd._lib.ssd_scan_fwd(p, p, p, p, p, p, p, None, None, p, None, ctypes.byref(too_small), 128, None)
    assert rc == ssd.SSD_ERR_INVALID_ARG          # workspace too small


def test_workspace_size_grows_with_tokens(ssd):
    a = ssd.workspace_size(_dims(ssd, T=256, seqlen=256), 128)
    b = ssd.workspace_size(_dims(ssd, T=4096, seqlen=4096), 128)
    assert 0 < a < b
    packed = ssd.make_dims(1000, 8, 64, 2, 128, ssd.SSD_DTYPE_BF16, nseq=7)
    assert ssd.workspace_size(packed, 64) > 0


def test_variant_names(ssd):
    assert ssd.scan_variant(_dims(ssd), 128) in ("tc", "simt")
    assert ssd.scan_variant(_dims(ssd, dtype_code=ssd.SSD_DTYPE_F32, P=16, N=16, H=4, G=1), 64) == "simt"


def test_snapshot_count_and_workspace(ssd):
    import torch
    dense = _dims(ssd, T=1000, batch=2, seqlen=500)
    assert ssd.snapshot_count(dense, 128) == 2 * (500 // 128)
    assert ssd.snapshot_count(dense, 1000) == 0
    packed = ssd.make_dims(1217, 8, 64, 2, 128, ssd.SSD_DTYPE_BF16, nseq=3)
    cu = torch.tensor([0, 300, 317, 1217], dtype=torch.int32)
    assert ssd.snapshot_count(packed, 128, cu) == 300 // 128 + 0 + 900 // 128
    assert ssd.snapshot_workspace_size(dense, 128, 256) >= ssd.workspace_size(dense, 128)


@pytest.mark.parametrize("snap,dims_kw,chunk,status", [
    (0, {}, 128, "INVALID_ARG"),
    (-128, {}, 128, "INVALID_ARG"),
    (200, {}, 128, "UNSUPPORTED"),                                       # tensor-core path: multiple of 128
    (96, dict(dtype_code=1 - 1, P=16, N=16, H=4, G=1), 64, "UNSUPPORTED"),  # CUDA-core path: multiple of chunk
])
def test_bad_snapshot_interval_fails_closed(ssd, snap, dims_kw, chunk, status):
    kw = dict(dims_kw)
    if "dtype_code" in kw:
        kw["dtype_code"] = ssd.SSD_DTYPE_F32
    with pytest.raises(ssd.SSDError, match=status):
        ssd.snapshot_workspace_size(_dims(ssd, **kw), chunk, snap)


def test_strict_entry_points_fail_closed_on_host(ssd):
    """Strict mode rejects bad chunk lengths and missing caches before any CUDA work."""
    d = _dims(ssd)
    b = ctypes.c_size_t(0)
    assert ssd._lib.ssd_strict_scan_fwd_workspace_size(ctypes.byref(d), 96, ctypes.byref(b)) == \
        ssd.SSD_ERR_UNSUPPORTED
    assert ssd._lib.ssd_strict_scan_fwd_workspace_size(ctypes.byref(d), 128, ctypes.byref(b)) == ssd.SSD_OK
    assert b.value > 0
    rc = ssd._lib.ssd_strict_scan_fwd(None, None, None, None, None, None, None, None, None, None, None, 0,
                                      ctypes.byref(d), 128, None)
    assert rc == ssd.SSD_ERR_INVALID_ARG and "cache" in ssd._lib.ssd_last_error().decode()
    empty = ssd.SSDChunkCache()
    dd = _dims(ssd, T=1, batch=1, seqlen=1)
    rc = ssd._lib.ssd_strict_state_update(ctypes.byref(empty), None, None, None, None, None, None, None, None,
                                          ctypes.byref(dd), 128, None)
    assert rc == ssd.SSD_ERR_INVALID_ARG
    rc = ssd._lib.ssd_strict_state_update(ctypes.byref(empty), None, None, None, None, None, None, None, None,
                                          ctypes.byref(dd), 100, None)
    assert rc == ssd.SSD_ERR_UNSUPPORTED


@pytest.mark.parametrize("batch,seqlen,H,G,expect", [
    (1, 65536, 64, 8, 7296),      # 9 segments of 57 chunks: 288 chunk-scan CTAs, about two full waves
    (4, 4096, 64, 8, 2048),       # 8 segments: 256 chunk-scan CTAs, 128 segment-state CTAs
    (256, 2048, 64, 8, 2048),     # one segment per sequence
    (1, 2049, 8, 2, 256),         # small problem: shortest segments, every CTA in one wave
])
def test_dense_segment_planner(ssd, batch, seqlen, H, G, expect):
    """The tensor-core segment length chosen for dense batches (host logic, no GPU; 148 SMs
    assumed when no device answers)."""
    d = ssd.make_dims(batch * seqlen, H, 64, G, 128, ssd.SSD_DTYPE_BF16, batch=batch, seqlen=seqlen)
    assert ssd.scan_variant(d, 256) == "tc"
    assert ssd.segment_tokens(d, 256) == expect


def test_varlen_segment_planner(ssd):
    """Packed calls: the longest power-of-two segment whose chunk-scan grid fills a wave."""
    d = ssd.make_dims(68177, 64, 64, 8, 128, ssd.SSD_DTYPE_BF16, nseq=16)
    assert ssd.segment_tokens(d, 128) == 8192
    d = ssd.make_dims(3000, 64, 64, 8, 128, ssd.SSD_DTYPE_BF16, nseq=2)
    assert ssd.segment_tokens(d, 128) == 512


def test_segment_override(ssd):
    """ssd_set_segment_tokens forces the segment length and 0 restores the planner."""
    d = ssd.make_dims(65536, 64, 64, 8, 128, ssd.SSD_DTYPE_BF16, batch=1, seqlen=65536)
    try:
        ssd.set_segment_tokens(384)
        assert ssd.segment_tokens(d, 256) == 384
        ssd.set_segment_tokens(100)        # not a multiple of 128: planner again
        assert ssd.segment_tokens(d, 256) == 7296
    finally:
        ssd.set_segment_tokens(0)
    assert ssd.segment_tokens(d, 256) == 7296


def test_strict_binding_checks_before_the_library(ssd):
    """The strict-mode binding validates cache shapes and devices on the host (no GPU)."""
    import torch
    c = ssd.ChunkCache.empty(2, 8, 64, 2, 128, 128, torch.bfloat16, "cpu")
    assert tuple(c.state.shape) == (2, 8, 64, 128) and tuple(c.B.shape) == (2, 2, 128, 128)
    assert c.state_pn() is c.state
    x = torch.zeros(2, 8, 64, dtype=torch.bfloat16)
    dt = torch.zeros(2, 8)
    B = torch.zeros(2, 2, 128, dtype=torch.bfloat16)
    h = torch.zeros(8)
    with pytest.raises(ValueError, match="must be on"):
        ssd.strict_state_update(c, x, dt, h, h, B, B, h)
    bad = ssd.ChunkCache.empty(2, 8, 64, 2, 128, 64, torch.bfloat16, "cpu")
    bad.len = torch.zeros(3, 8, dtype=torch.int32)
    with pytest.raises(ValueError):
        bad._check(2, 8, 64, 2, 128, torch.bfloat16, torch.device("cpu"))


def test_noalloc_scratch_fits_the_named_prefill_workloads_except_packed(ssd):
    """ssd_scan_fwd_noalloc has 32 MiB of scratch: the tiny, batched and long-context
    workloads fit; the 16-sequence packed workload (one segment state per sequence and
    per segment) does not, so that entry point refuses it (host logic, no GPU)."""
    from mamba_ssd_state_02_b200 import workloads as W
    limit = 32 << 20
    for k in (0, 1, 2, 3):
        w = W.config(k)
        code = ssd.SSD_DTYPE_BF16 if w.dtype.itemsize == 2 else ssd.SSD_DTYPE_F32
        if w.varlen:
            d = ssd.make_dims(w.total_tokens, w.nheads, w.headdim, w.ngroups, w.dstate, code, nseq=w.nseq)
        else:
            d = ssd.make_dims(w.total_tokens, w.nheads, w.headdim, w.ngroups, w.dstate, code,
                              batch=w.nseq, seqlen=w.seqlens[0])
        assert (ssd.workspace_size(d, w.chunk) <= limit) == (k != 3), k
