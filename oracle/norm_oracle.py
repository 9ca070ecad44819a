"""FP64 oracle of the gated group RMSNorm stage (test infrastructure only: tests/, the
smoke check and bench.py's CPU baseline may use it; the library never does).

From its definition (RL-Kernel issue page, Figure 2: the scan output gated by SiLU of the
z branch and normalised over groups of 512 channels; the JAX Nemotron 3 Nano page's
configuration gives the epsilon): for token t and channel c in group G,

    g[t][c]   = y[t][c] * z[t][c] * sigmoid(z[t][c])
    out[t][c] = g[t][c] / sqrt(mean_{c' in G} g[t][c']^2 + eps) * weight[c]

with inputs taken at the exact values the GPU receives, widened to float64.
"""
from __future__ import annotations

import numpy as np
import torch


def gated_rmsnorm(y, z, weight, group_size=512, eps=1e-6):
    """y, z [..., C]; weight [C]. Returns out [..., C] float64."""
    yv = y.detach().to("cpu", torch.float64).numpy()
    zv = z.detach().to("cpu", torch.float64).numpy()
    w = weight.detach().to("cpu", torch.float64).numpy()
    shape = yv.shape
    C = shape[-1]
    g = yv * zv / (1.0 + np.exp(-zv))
    gg = g.reshape(-1, C // group_size, group_size)
    ms = (gg * gg).mean(axis=-1, keepdims=True)
    return (gg / np.sqrt(ms + eps)).reshape(shape) * w
