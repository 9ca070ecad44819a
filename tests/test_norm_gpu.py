"""Gated group RMSNorm on the GPU (ssd_gated_rmsnorm) against the FP64 oracle: bf16 and
float32, group sizes 256/512/1024, a token count that is not a multiple of the kernel's
token run, in place (out aliasing y), and chained after the tensor-core scan. Outputs
are compared after rounding to the input dtype (max error over max |ref|: 4e-3 for
bf16, 1e-5 for float32)."""
import numpy as np
import pytest
import torch

from mamba_ssd_state_02_b200 import workloads as W
from oracle import norm_oracle as NO
from parity_util import rel_err

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 4e-3, torch.float32: 1e-5}


def _inputs(T, C, dtype, seed):
    y = W.to_input_dtype(W.normal(seed, 30, T * C), dtype).view(T, C)
    z = W.to_input_dtype(W.normal(seed, 31, T * C), dtype).view(T, C)
    w = (W.uniform(seed, 32, C) + 0.5).to(torch.float32)
    return y, z, w


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("gs", [256, 512, 1024])
def test_gated_rmsnorm_matches_oracle(ssd, cuda_dev, dtype, gs):
    y, z, w = _inputs(1001, 2048, dtype, 21)
    out = ssd.gated_rmsnorm(y.to(cuda_dev), z.to(cuda_dev), w.to(cuda_dev), group_size=gs, eps=1e-6)
    ssd.device_status()
    ref = NO.gated_rmsnorm(y, z, w, group_size=gs, eps=1e-6)
    assert rel_err(out, torch.from_numpy(ref)) <= TOL[dtype]


def test_gated_rmsnorm_in_place(ssd, cuda_dev):
    y, z, w = _inputs(300, 4096, torch.bfloat16, 22)
    yd = y.to(cuda_dev)
    out = ssd.gated_rmsnorm(yd, z.to(cuda_dev), w.to(cuda_dev), out=yd)
    ssd.device_status()
    assert out.data_ptr() == yd.data_ptr()
    assert rel_err(out, torch.from_numpy(NO.gated_rmsnorm(y, z, w))) <= TOL[torch.bfloat16]


def test_scan_then_gated_rmsnorm(ssd, cuda_dev):
    """Tensor-core scan -> gated norm (group 512 = 8 heads of 64), with the oracle norm
    applied to the GPU's own scan output, so the check isolates the norm stage."""
    w = W.Workload("norm", nheads=16, headdim=64, ngroups=2, dstate=128, chunk=128, dtype=torch.bfloat16,
                   seqlens=[700, 300], varlen=True, init="normal", seed=23)
    d = W.make_all(w, device=cuda_dev)
    y, _ = ssd.scan_fwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                        init_state=d["init_state"], cu_seqlens=d["cu_seqlens"], chunk=128)
    _, z, nw = _inputs(w.total_tokens, 16 * 64, torch.bfloat16, 24)
    yf = y.view(w.total_tokens, -1)
    out = ssd.gated_rmsnorm(yf, z.to(cuda_dev), nw.to(cuda_dev))
    ssd.device_status()
    assert rel_err(out, torch.from_numpy(NO.gated_rmsnorm(yf.cpu(), z, nw))) <= TOL[torch.bfloat16]


def test_bad_group_fails_closed(ssd, cuda_dev):
    y = torch.zeros(4, 768, dtype=torch.bfloat16, device=cuda_dev)
    with pytest.raises(ssd.SSDError, match="UNSUPPORTED"):
        ssd.gated_rmsnorm(y, y, torch.ones(768, device=cuda_dev), group_size=512)
