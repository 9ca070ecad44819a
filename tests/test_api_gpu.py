"""C-ABI behaviour on the GPU: device-detected errors, workspace handling, empty
inputs and launch accounting (fail closed: RL-Kernel issue page §4.1 and §7)."""
import pytest
import torch

from mamba_ssd_state_02_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _inp(dev, seqlens=(200, 50), varlen=True, init="normal"):
    w = W.Workload("api", nheads=8, headdim=64, ngroups=2, dstate=128, chunk=64, dtype=torch.bfloat16,
                   seqlens=list(seqlens), varlen=varlen, init=init, seed=3)
    return w, W.make_all(w, device=dev)


def _call(ssd, d, cu=None, A=None, chunk=64, **kw):
    return ssd.scan_fwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"] if A is None else A, d["B"], d["C"],
                        d["D"], init_state=d["init_state"], cu_seqlens=d["cu_seqlens"] if cu is None else cu,
                        chunk=chunk, **kw)


@pytest.mark.parametrize("cu", [[0, 300, 250], [1, 100, 250], [0, 100, 249]])
def test_bad_cu_seqlens_latched_on_device(ssd, cuda_dev, cu):
    _, d = _inp(cuda_dev)
    ssd.device_status()
    y, fin = _call(ssd, d, cu=torch.tensor(cu, dtype=torch.int32, device=cuda_dev))
    with pytest.raises(ssd.SSDError, match="INVALID_ARG"):
        ssd.device_status()
    ssd.device_status()          # the word was cleared by the read


def test_positive_A_latched_on_device(ssd, cuda_dev):
    _, d = _inp(cuda_dev)
    A = d["A"].clone()
    A[3] = 0.5
    _call(ssd, d, A=A)
    with pytest.raises(ssd.SSDError, match="INVALID_ARG"):
        ssd.device_status()


def test_caller_workspace_matches_internal(ssd, cuda_dev):
    _, d = _inp(cuda_dev)
    y1, f1 = _call(ssd, d)
    dims = ssd.make_dims(d["x"].shape[0], 8, 64, 2, 128, ssd.SSD_DTYPE_BF16, nseq=2)
    nbytes = ssd.workspace_size(dims, 64)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=cuda_dev)
    y2, f2 = _call(ssd, d, workspace=ws)
    ssd.device_status()
    assert torch.equal(y1, y2) and torch.equal(f1, f2)
    with pytest.raises(ssd.SSDError, match="INVALID_ARG"):
        _call(ssd, d, workspace=ws[: nbytes // 2])


def test_empty_inputs(ssd, cuda_dev):
    _, d = _inp(cuda_dev, seqlens=(0, 0, 0))
    y, fin = _call(ssd, d)
    ssd.device_status()
    assert y.numel() == 0 and torch.equal(fin, d["init_state"])
    # dense with seqlen 0: final state == initial state
    w, d = _inp(cuda_dev, seqlens=(5, 5), varlen=False)
    e = lambda t: t[:0].reshape(1, 0, *t.shape[1:]).expand(2, 0, *t.shape[1:]).contiguous()
    y, fin = ssd.scan_fwd(e(d["x"]), e(d["dt_raw"]), d["dt_bias"], d["A"], e(d["B"]), e(d["C"]), d["D"],
                          init_state=d["init_state"], chunk=128)
    ssd.device_status()
    assert torch.equal(fin, d["init_state"])
    # batch 0: nothing launched
    y, fin = ssd.scan_fwd(e(d["x"])[:0], e(d["dt_raw"])[:0], d["dt_bias"], d["A"], e(d["B"])[:0],
                          e(d["C"])[:0], d["D"], chunk=128)
    assert fin.numel() == 0 and ssd.last_launch_count() == 0


def test_misaligned_input_rejected(ssd, cuda_dev):
    _, d = _inp(cuda_dev)
    buf = torch.empty(d["x"].numel() + 1, dtype=torch.bfloat16, device=cuda_dev)
    xm = buf[1:].view_as(d["x"])
    xm.copy_(d["x"])
    with pytest.raises(ssd.SSDError, match="INVALID_ARG"):
        ssd.scan_fwd(xm, d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                     init_state=d["init_state"], cu_seqlens=d["cu_seqlens"], chunk=64)


def test_launch_count_reported(ssd, cuda_dev):
    _, d = _inp(cuda_dev)
    _call(ssd, d)
    assert ssd.last_launch_count() >= 1
    st = torch.zeros(2, 8, 64, 128, device=cuda_dev)
    ssd.state_update(st, d["x"][:2], d["dt_raw"][:2], d["dt_bias"], d["A"], d["B"][:2], d["C"][:2], d["D"])
    assert ssd.last_launch_count() == 1
