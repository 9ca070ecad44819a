"""State snapshots (ssd_scan_fwd_snapshots): each sequence's state after every
multiple of `snapshot_tokens` tokens, for prefix-cache reuse and chunked prefill.
Checked against the FP64 oracle's snapshots on both pipelines (tensor-core bf16 and
CUDA-core fp32), dense and packed, and against the GPU's own final state of the
prefix cut at the snapshot (the definition of a snapshot)."""
import pytest
import torch

from mamba_ssd_state_02_b200 import workloads as W
from oracle import oracle as O
from parity_util import TOL_STATE, TOL_Y, rel_err

pytestmark = pytest.mark.gpu


def _run(ssd, dev, w, d, I, chunk=None):
    g = lambda t: None if t is None else t.to(dev)
    q = w.chunk if chunk is None else chunk
    if w.varlen:
        return ssd.scan_fwd(g(d["x"]), g(d["dt_raw"]), g(d["dt_bias"]), g(d["A"]), g(d["B"]), g(d["C"]),
                            g(d["D"]), init_state=g(d["init_state"]), cu_seqlens=g(d["cu_seqlens"]), chunk=q,
                            snapshot_tokens=I)
    b, L = w.nseq, w.seqlens[0]
    rs = lambda t: g(t).reshape(b, L, *t.shape[1:])
    y, f, sn = ssd.scan_fwd(rs(d["x"]), rs(d["dt_raw"]), g(d["dt_bias"]), g(d["A"]), rs(d["B"]), rs(d["C"]),
                            g(d["D"]), init_state=g(d["init_state"]), chunk=q, snapshot_tokens=I)
    return y.reshape(b * L, *y.shape[2:]), f, sn


def _oracle(w, d, I):
    return O.ssd_scan(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                      init_state=d["init_state"], cu_seqlens=d["cu_seqlens"],
                      batch=None if w.varlen else w.nseq, snapshot_tokens=I)


CASES = [
    # tensor-core pipeline: ragged packed sequences, intervals that are and are not the
    # default segment length, a sequence shorter than the interval
    ("tc", [700, 17, 1300, 256], True, torch.bfloat16, 8, 64, 2, 128, 128, 256),
    ("tc", [700, 17, 1300, 256], True, torch.bfloat16, 8, 64, 2, 128, 128, 384),
    ("tc", [1024, 1024], False, torch.bfloat16, 8, 64, 2, 128, 128, 512),
    # CUDA-core pipeline
    ("simt", [300, 5, 260], True, torch.float32, 4, 16, 2, 16, 64, 64),
    ("simt", [256, 256], False, torch.float32, 4, 32, 1, 32, 128, 128),
]


@pytest.mark.parametrize("variant,seqlens,varlen,dtype,H,P,G,N,chunk,I", CASES)
def test_snapshots_match_oracle(ssd, cuda_dev, variant, seqlens, varlen, dtype, H, P, G, N, chunk, I):
    w = W.Workload("snap", nheads=H, headdim=P, ngroups=G, dstate=N, chunk=chunk, dtype=dtype,
                   seqlens=seqlens, varlen=varlen, init="normal", seed=71)
    dims = (ssd.make_dims(w.total_tokens, H, P, G, N, ssd.SSD_DTYPE_BF16 if dtype == torch.bfloat16 else
                          ssd.SSD_DTYPE_F32, nseq=w.nseq) if varlen else
            ssd.make_dims(w.total_tokens, H, P, G, N, ssd.SSD_DTYPE_BF16 if dtype == torch.bfloat16 else
                          ssd.SSD_DTYPE_F32, batch=w.nseq, seqlen=seqlens[0]))
    assert ssd.scan_variant(dims, chunk) == variant
    d = W.make_all(w)
    y, fin, sn = _run(ssd, cuda_dev, w, d, I)
    ssd.device_status()
    y_ref, fin_ref, sn_ref = _oracle(w, d, I)
    assert sn.shape == sn_ref.shape == (sum(L // I for L in seqlens), H, P, N)
    assert rel_err(y, y_ref) <= TOL_Y[dtype]
    assert rel_err(fin, fin_ref) <= TOL_STATE
    for k in range(sn.shape[0]):                 # every snapshot on its own scale
        assert rel_err(sn[k], sn_ref[k]) <= TOL_STATE, k


def test_snapshot_equals_final_state_of_the_prefix(ssd, cuda_dev):
    """Snapshot m of a sequence is the final state of the same call cut after m*I tokens
    (GPU against GPU, tensor-core pipeline)."""
    I = 256
    w = W.Workload("snap", nheads=8, headdim=64, ngroups=2, dstate=128, chunk=128, dtype=torch.bfloat16,
                   seqlens=[1100], varlen=True, init="normal", seed=73)
    d = W.make_all(w)
    _, _, sn = _run(ssd, cuda_dev, w, d, I)
    g = lambda t: t.to(cuda_dev)
    for m in (1, 3, 4):
        L = m * I
        sl = slice(0, L)
        _, f = ssd.scan_fwd(g(d["x"][sl]), g(d["dt_raw"][sl]), g(d["dt_bias"]), g(d["A"]), g(d["B"][sl]),
                            g(d["C"][sl]), g(d["D"]), init_state=g(d["init_state"]),
                            cu_seqlens=torch.tensor([0, L], dtype=torch.int32, device=cuda_dev), chunk=128)
        assert rel_err(sn[m - 1], f[0]) <= TOL_STATE, m
    ssd.device_status()


def test_snapshot_interval_not_supported(ssd, cuda_dev):
    w = W.Workload("snap", nheads=8, headdim=64, ngroups=2, dstate=128, chunk=128, dtype=torch.bfloat16,
                   seqlens=[512], varlen=True, init="zero", seed=75)
    d = W.make_all(w, device=cuda_dev)
    with pytest.raises(ssd.SSDError, match="UNSUPPORTED"):
        ssd.scan_fwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                     cu_seqlens=d["cu_seqlens"], chunk=128, snapshot_tokens=200)


@pytest.mark.parametrize("seqlens,varlen,seg,I", [
    # cuts inside segments that do not line up with the segment boundaries
    ([2600, 17, 1300, 4100, 640], True, 1024, 384),
    ([2600, 17, 1300, 4100, 640], True, 1152, 256),
    ([3072, 3072], False, 1536, 512),
    # a cut after every chunk of a segment
    ([2048, 300], True, 2048, 128),
])
def test_snapshots_inside_long_segments(ssd, cuda_dev, seqlens, varlen, seg, I):
    """Tensor-core pipeline with segments longer than the interval: each segment's state is
    cut at the snapshot positions inside it, and the chain walks the pieces."""
    w = W.Workload("snap", nheads=8, headdim=64, ngroups=2, dstate=128, chunk=128, dtype=torch.bfloat16,
                   seqlens=seqlens, varlen=varlen, init="normal", seed=77)
    d = W.make_all(w)
    ssd.set_segment_tokens(seg)
    try:
        y, fin, sn = _run(ssd, cuda_dev, w, d, I)
        ssd.device_status()
    finally:
        ssd.set_segment_tokens(0)
    y_ref, fin_ref, sn_ref = _oracle(w, d, I)
    assert sn.shape == sn_ref.shape == (sum(L // I for L in seqlens), 8, 64, 128)
    assert rel_err(y, y_ref) <= TOL_Y[torch.bfloat16]
    assert rel_err(fin, fin_ref) <= TOL_STATE
    for k in range(sn.shape[0]):
        assert rel_err(sn[k], sn_ref[k]) <= TOL_STATE, k



@pytest.mark.slow
def test_snapshots_long_context_full_size(ssd, cuda_dev):
    """The long-context workload (1 x 65536 tokens, 64 heads, chunk 256) with snapshots
    every 2048 tokens. The planner keeps its 7296-token segments, so every segment is cut
    into pieces at the snapshot positions. One head per B/C group is checked against the
    oracle at all 32 snapshots, and at the final state."""
    w = W.config(2)
    L, I = w.seqlens[0], 2048
    dims = ssd.make_dims(L, w.nheads, w.headdim, w.ngroups, w.dstate, ssd.SSD_DTYPE_BF16, batch=1, seqlen=L)
    assert ssd.segment_tokens(dims, w.chunk) % I != 0          # cuts inside segments
    inp = W.make_all(w, device=cuda_dev)
    rs = lambda t: t.reshape(1, L, *t.shape[1:])
    y, fin, sn = ssd.scan_fwd(rs(inp["x"]), rs(inp["dt_raw"]), inp["dt_bias"], inp["A"], rs(inp["B"]),
                              rs(inp["C"]), inp["D"], init_state=inp["init_state"], chunk=w.chunk,
                              snapshot_tokens=I)
    ssd.device_status()
    assert sn.shape == (L // I, w.nheads, w.headdim, w.dstate)
    heads = [0, 9, 18, 27, 36, 45, 54, 63]                     # one head in each of the 8 groups
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    _, fin_ref, sn_ref = O.ssd_scan(cpu["x"], cpu["dt_raw"], cpu["dt_bias"], cpu["A"], cpu["B"], cpu["C"],
                                    cpu["D"], init_state=cpu["init_state"], batch=1,
                                    pairs=[(0, h) for h in heads], want_y=False, snapshot_tokens=I)
    for k, h in enumerate(heads):
        assert rel_err(fin[0, h], fin_ref[k]) <= TOL_STATE, h
        for m in range(L // I):
            assert rel_err(sn[m, h], torch.as_tensor(sn_ref[k][m])) <= TOL_STATE, (h, m)
