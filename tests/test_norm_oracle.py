"""Pins of the gated group RMSNorm oracle: torch's own rms_norm applied group by group
(a library routine), scipy's logistic function for the gate, and the invariances the
definition fixes (scale invariance without eps, unit RMS of every group)."""
import numpy as np
import pytest
import torch
from scipy.special import expit

from oracle import norm_oracle as NO


def _inputs(T=37, C=1024, seed=0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(T, C, generator=g, dtype=torch.float64), torch.randn(T, C, generator=g, dtype=torch.float64),
            torch.rand(C, generator=g, dtype=torch.float64) + 0.5)


@pytest.mark.parametrize("gs", [256, 512, 1024])
def test_matches_torch_rms_norm_per_group(gs):
    y, z, w = _inputs()
    out = NO.gated_rmsnorm(y, z, w, group_size=gs, eps=1e-6)
    gate = torch.from_numpy(y.numpy() * z.numpy() * expit(z.numpy()))
    ref = torch.nn.functional.rms_norm(gate.view(37, -1, gs), (gs,), eps=1e-6).view(37, -1) * w
    assert np.abs(out - ref.numpy()).max() < 1e-12


def test_scale_invariance_and_unit_rms():
    y, z, w = _inputs(seed=1)
    a = NO.gated_rmsnorm(y, z, torch.ones_like(w), group_size=512, eps=0.0)
    b = NO.gated_rmsnorm(y * 7.5, z, torch.ones_like(w), group_size=512, eps=0.0)
    assert np.abs(a - b).max() < 1e-12
    rms = np.sqrt((a.reshape(37, -1, 512) ** 2).mean(axis=-1))
    assert np.abs(rms - 1.0).max() < 1e-12
