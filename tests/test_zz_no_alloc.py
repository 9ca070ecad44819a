"""The no-allocation prefill entry point, ssd_scan_fwd_noalloc.

Some callers cannot allocate device memory while they run: serving engines that reserve
their whole memory budget when they start and forbid later allocations, and
latency-critical loops where a cudaMalloc/cudaFree (or a caching allocator's slow path)
in the middle of a step is not acceptable. For them the library offers
ssd_scan_fwd_noalloc, which takes its scratch from an array compiled into the library.

These tests call it through the C ABI and check that it gives bit for bit the same
outputs as ssd_scan_fwd (both run the same deterministic kernels), on calls in a row with
different problems (so a later call cannot lean on what an earlier one left in the shared
scratch: segment tables, orders and states of a larger problem), and that it refuses a
problem whose scratch would not fit. This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from mamba_ssd_state_02_b200 import workloads as W
from parity_util import TOL_STATE, TOL_Y, oracle_scan, rel_err

pytestmark = pytest.mark.gpu


def _case(dev, seqlens, varlen, dtype, H, P, G, N, chunk, init, seed):
    w = W.Workload("noalloc", nheads=H, headdim=P, ngroups=G, dstate=N, chunk=chunk, dtype=dtype,
                   seqlens=seqlens, varlen=varlen, init=init, seed=seed)
    return w, W.make_all(w, device=dev)


def _call(fn, w, d):
    if w.varlen:
        return fn(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                  init_state=d["init_state"], cu_seqlens=d["cu_seqlens"], chunk=w.chunk)
    b, L = w.nseq, w.seqlens[0]
    r = lambda t: t.reshape(b, L, *t.shape[1:])
    return fn(r(d["x"]), r(d["dt_raw"]), d["dt_bias"], d["A"], r(d["B"]), r(d["C"]), d["D"],
              init_state=d["init_state"], chunk=w.chunk)


def test_noalloc_matches_scan_fwd_on_two_calls_in_a_row(ssd, cuda_dev):
    cases = [
        # tensor-core pipeline, packed sequences, zero initial state
        _case(cuda_dev, [300, 17, 900], True, torch.bfloat16, 8, 64, 2, 128, 128, "zero", 91),
        # CUDA-core pipeline, dense batch, random initial state
        _case(cuda_dev, [700, 700], False, torch.float32, 4, 32, 2, 64, 64, "normal", 92),
    ]
    refs = []
    for w, d in cases:
        y, f = _call(ssd.scan_fwd, w, d)
        refs.append((y.clone(), f.clone()))
    outs = []
    for w, d in cases:                           # two no-allocation calls back to back
        outs.append(_call(ssd.scan_fwd_noalloc, w, d))
    ssd.device_status()
    for (w, _), (y_ref, f_ref), (y, f) in zip(cases, refs, outs):
        assert torch.equal(y, y_ref)
        assert torch.equal(f, f_ref)


def test_noalloc_smaller_tensor_core_call_after_a_larger_one(ssd, cuda_dev):
    # A larger packed problem (more sequences, more segments, longer segment table and
    # segment order) leaves its tables and states in the shared scratch; the smaller one
    # after it, with other lengths, must not read any of them.
    big_w, big = _case(cuda_dev, [2600, 5, 1300, 4100, 640], True, torch.bfloat16, 8, 64, 2, 128, 128,
                       "normal", 93)
    small_w, small = _case(cuda_dev, [900, 333], True, torch.bfloat16, 8, 64, 2, 128, 128, "normal", 94)
    ssd.set_segment_tokens(256)                 # many segments in both calls
    try:
        y_ref, f_ref = _call(ssd.scan_fwd, small_w, small)
        y_ref, f_ref = y_ref.clone(), f_ref.clone()
        _call(ssd.scan_fwd_noalloc, big_w, big)
        y, f = _call(ssd.scan_fwd_noalloc, small_w, small)
        ssd.device_status()
    finally:
        ssd.set_segment_tokens(0)
    assert torch.equal(y, y_ref)
    assert torch.equal(f, f_ref)
    y_o, f_o = oracle_scan(small_w, small)
    assert rel_err(y, y_o) <= TOL_Y[small_w.dtype]
    assert rel_err(f, f_o) <= TOL_STATE


def test_noalloc_rejects_problems_beyond_its_scratch(ssd, cuda_dev):
    # 32 x 32768 tokens, 64 heads: at least 64 segments (at most 16384 tokens each), whose
    # states alone need at least 128 MiB > 32 MiB.
    d = ssd.make_dims(32 * 32768, 64, 64, 8, 128, ssd.SSD_DTYPE_BF16, batch=32, seqlen=32768)
    assert ssd.workspace_size(d, 256) > 32 << 20
    p = 1 << 20                                  # never dereferenced: rejected on the host
    rc = ssd._lib.ssd_scan_fwd_noalloc(p, p, p, p, p, p, p, None, None, p, None, ctypes.byref(d), 256,
                                       None)
    assert rc == ssd.SSD_ERR_UNSUPPORTED
    assert "scratch" in ssd._lib.ssd_last_error().decode()
