"""The tensor-core prefill's fail-closed path (RL-Kernel issue page, §4.1 and §7: fail
closed). Every wait on a shared-memory barrier between the kernels' warps is bounded
(about 2 s); the test hook ssd_test_stall makes one pass's UMMA warp wait on a barrier
that nothing arrives at, so that the wait runs out. The call must end (no hang), latch
SSD_ERR_TIMEOUT, and leave the context usable: the same call made afterwards is
correct. No copy or MMA is left in flight when a CTA gives up (its TMA and UMMA warps
wait for what they issued), so nothing faults."""
import pytest
import torch

from mamba_ssd_state_02_b200 import workloads as W
from parity_util import TOL_STATE, TOL_Y, oracle_scan, rel_err

pytestmark = pytest.mark.gpu


def _call(ssd, w, d):
    if w.varlen:
        return ssd.scan_fwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                            init_state=d["init_state"], cu_seqlens=d["cu_seqlens"], chunk=w.chunk)
    L = w.seqlens[0]
    r4 = lambda t: t.view(w.nseq, L, *t.shape[1:])
    y, f = ssd.scan_fwd(r4(d["x"]), r4(d["dt_raw"]), d["dt_bias"], d["A"], r4(d["B"]), r4(d["C"]), d["D"],
                        init_state=d["init_state"], chunk=w.chunk)
    return y.reshape(-1, *y.shape[2:]), f


@pytest.mark.parametrize("varlen", [True, False])
@pytest.mark.parametrize("stalled_pass", [1, 2])
def test_wait_runs_out_fails_closed_and_context_stays_usable(ssd, cuda_dev, stalled_pass, varlen):
    # packed: the table kernel builds the segments; dense: the segment-state pass does
    seqlens = [1500, 700, 90] if varlen else [1100, 1100]
    w = W.Workload("timeout", nheads=8, headdim=64, ngroups=2, dstate=128, chunk=128, dtype=torch.bfloat16,
                   seqlens=seqlens, varlen=varlen, init="normal", seed=81)
    d = W.make_all(w, device=cuda_dev)
    dims = (ssd.make_dims(w.total_tokens, 8, 64, 2, 128, ssd.SSD_DTYPE_BF16, nseq=w.nseq) if varlen else
            ssd.make_dims(w.total_tokens, 8, 64, 2, 128, ssd.SSD_DTYPE_BF16, batch=w.nseq, seqlen=seqlens[0]))
    assert ssd.scan_variant(dims, w.chunk) == "tc"
    ssd.device_status()                          # nothing latched before
    ssd.test_stall(stalled_pass)
    try:
        _call(ssd, w, d)
        torch.cuda.synchronize()
        with pytest.raises(ssd.SSDError, match="TIMEOUT"):
            ssd.device_status()
    finally:
        ssd.test_stall(0)
    ssd.device_status()                          # the status was read and cleared
    y, f = _call(ssd, w, d)
    ssd.device_status()
    y_o, f_o = oracle_scan(w, d)
    assert rel_err(y, y_o) <= TOL_Y[torch.bfloat16]
    assert rel_err(f, f_o) <= TOL_STATE
