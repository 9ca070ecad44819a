"""Tensor-core path checks: the UMMA operand-format diagnostic against a plain
matmul, and oracle parity of the tcgen05 prefill pipeline on cases that stress its
two-level structure (segments and 128-token chunks): ragged chunks, sequences
shorter than a chunk, sequences spanning many segments, and one-chunk segments
(the longest chain of segment states)."""
import os

import pytest
import torch

from mamba_ssd_state_02_b200 import workloads as W
from parity_util import TOL_STATE, oracle_scan, rel_err, run_gpu_scan

pytestmark = pytest.mark.gpu


def test_umma_operand_formats(ssd, cuda_dev):
    g = torch.Generator().manual_seed(0)
    X1 = torch.randn(128, 128, generator=g).bfloat16()
    X2 = torch.randn(128, 128, generator=g).bfloat16()
    out = ssd.selftest_umma(X1.to(cuda_dev), X2.to(cuda_dev))
    torch.cuda.synchronize()
    ssd.device_status()
    a, b = X1.double(), X2.double()
    ref = [a @ b.T, a @ b[:, :64], a.T @ b[:, :64], a @ b[:, :64], a @ b[:, :64]]
    got = out.cpu().double()
    for i, r in enumerate(ref):
        cols = r.shape[1]
        assert rel_err(got[i, :, :cols], r) < 1e-5, f"product {i}"


def _tc_wl(seqlens, varlen, init="normal", H=8, G=2, seed=41, dt_range=(1e-3, 0.1)):
    return W.Workload("tc", nheads=H, headdim=64, ngroups=G, dstate=128, chunk=128, dtype=torch.bfloat16,
                      seqlens=seqlens, varlen=varlen, init=init, seed=seed, dt_range=dt_range)


def _check(ssd, dev, w):
    dims = ssd.make_dims(w.total_tokens, w.nheads, 64, w.ngroups, 128, ssd.SSD_DTYPE_BF16,
                         nseq=w.nseq) if w.varlen else ssd.make_dims(
        w.total_tokens, w.nheads, 64, w.ngroups, 128, ssd.SSD_DTYPE_BF16, batch=w.nseq, seqlen=w.seqlens[0])
    assert ssd.scan_variant(dims, 128) == "tc"
    inp = W.make_all(w)
    y, fin = run_gpu_scan(ssd, w, inp, dev)
    ssd.device_status()
    y_ref, fin_ref = oracle_scan(w, inp)
    ey, ef = rel_err(y, y_ref), rel_err(fin, fin_ref)
    assert ey <= 1e-2 and ef <= TOL_STATE, (ey, ef)


@pytest.mark.parametrize("seqlens", [[1, 127, 128, 129, 300], [1000, 2500, 5], [4096]])
def test_tc_varlen_ragged(ssd, cuda_dev, seqlens):
    _check(ssd, cuda_dev, _tc_wl(seqlens, True))


@pytest.fixture
def segment_tokens(ssd):
    """Force the tensor-core segment length for one test, then restore the planner."""
    yield ssd.set_segment_tokens
    ssd.set_segment_tokens(0)


@pytest.mark.parametrize("seg", [128, 256, 384])
def test_tc_short_segments(ssd, cuda_dev, seg, segment_tokens):
    segment_tokens(seg)
    _check(ssd, cuda_dev, _tc_wl([1500, 700], True, seed=43, dt_range=(1e-4, 0.5)))


@pytest.mark.parametrize("seg", [2048, 4096, 7296, 8192])
def test_tc_long_segments(ssd, cuda_dev, seg, segment_tokens):
    # Segments of 16 to 64 chunks with ragged last segments and a sequence shorter than one.
    segment_tokens(seg)
    _check(ssd, cuda_dev, _tc_wl([9000, 4500, 130], True, seed=46, dt_range=(1e-4, 0.5)))


def test_tc_dense_heads_per_group_16(ssd, cuda_dev):
    _check(ssd, cuda_dev, _tc_wl([600, 600], False, H=16, G=1, seed=44))


def test_tc_zero_init_wide_dt(ssd, cuda_dev):
    _check(ssd, cuda_dev, _tc_wl([2049], False, init="zero", seed=45, dt_range=(1e-4, 0.5)))


@pytest.mark.parametrize("seqlens,H,G,seg", [
    ([3000, 2000, 1], 8, 2, 128),      # 41 one-chunk segments: the longest chains, more CTAs than SMs
    ([1024, 1000], 64, 8, 128),        # 16 segments of all 64 heads: 512 chunk-scan CTAs
    ([4096] * 4, 64, 8, 512),          # the batched workload's shape with 512-token segments
])
def test_tc_many_segments(ssd, cuda_dev, seqlens, H, G, seg, segment_tokens):
    """Many short segments: grids of several waves in both passes and long segment chains."""
    segment_tokens(seg)
    _check(ssd, cuda_dev, _tc_wl(seqlens, len(set(seqlens)) > 1, H=H, G=G, seed=48))


@pytest.mark.parametrize("seg", [384, 1024])
def test_tc_dense_table_from_the_grid(ssd, cuda_dev, seg, segment_tokens):
    """A dense batch builds its segment table inside the segment-state pass (no table
    kernel): three sequences of 1000 tokens cut into segments of 384 (three per sequence,
    the last ragged) or 1024 (one, shorter than the segment)."""
    segment_tokens(seg)
    _check(ssd, cuda_dev, _tc_wl([1000] * 3, False, seed=49, dt_range=(1e-4, 0.5)))

