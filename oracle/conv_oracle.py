"""FP64 oracle of the causal conv1d + bias + SiLU prologue (test infrastructure only:
tests/, the smoke check and bench.py's CPU baseline may use it; the library never does).

Written straight from its definition (RL-Kernel issue page, Figure 2: causal conv1d of
width K over the xBC channels, plus bias, then SiLU, with a conv-state cache per
sequence, §1 item 2). For each sequence, channel c and token t, with the sequence's
previous K-1 inputs (the incoming conv state, zeros if none) placed before its first
token:

    pre[t][c] = bias[c] + sum_{k=0}^{K-1} w[c][k] * in[t - (K-1) + k][c]
    out[t][c] = pre[t][c] * sigmoid(pre[t][c])

and the outgoing conv state is the last K-1 entries of that extended input sequence.
Inputs are taken at the exact values the GPU receives (bf16 or float32 widened to
float64). Plain numpy loops over the K taps; no blocking or fusion.
"""
from __future__ import annotations

import numpy as np
import torch


def _f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def seq_offsets(T: int, cu_seqlens=None, batch=None):
    if cu_seqlens is not None:
        return np.asarray(torch.as_tensor(cu_seqlens).cpu(), dtype=np.int64)
    L = T // batch
    return np.arange(batch + 1, dtype=np.int64) * L


def conv1d_fwd(xbc, weight, bias=None, conv_state=None, cu_seqlens=None, batch=None, act=True):
    """xbc [T, D]; weight [D, K]; bias [D] or None; conv_state [nseq, D, K-1] or None.
    Returns (out [T, D] float64 (pre-activation if act is False), final state
    [nseq, D, K-1] float64)."""
    x = _f64(xbc)
    w = _f64(weight)
    T, D = x.shape
    K = w.shape[1]
    b = np.zeros(D) if bias is None else _f64(bias)
    off = seq_offsets(T, cu_seqlens, batch)
    nseq = len(off) - 1
    st0 = np.zeros((nseq, D, K - 1)) if conv_state is None else _f64(conv_state)
    out = np.zeros((T, D))
    fin = np.zeros((nseq, D, K - 1))
    for s in range(nseq):
        seg = x[off[s]:off[s + 1]]                       # [len, D]
        ext = np.concatenate([st0[s].T, seg], axis=0)    # [K-1+len, D]: state first, oldest first
        L = seg.shape[0]
        pre = np.tile(b, (L, 1))
        for k in range(K):
            pre += w[:, k][None, :] * ext[k:k + L]       # tap k sees input t-(K-1)+k
        out[off[s]:off[s + 1]] = pre * (1.0 / (1.0 + np.exp(-pre))) if act else pre
        fin[s] = ext[L:L + K - 1].T                      # last K-1 entries
    return out, fin


def conv1d_update(conv_state, xbc, weight, bias=None):
    """One decode step: conv_state [nseq, D, K-1], xbc [nseq, D]. Returns
    (out [nseq, D], new state [nseq, D, K-1]) float64."""
    st = _f64(conv_state)
    x = _f64(xbc)
    w = _f64(weight)
    K = w.shape[1]
    b = np.zeros(x.shape[1]) if bias is None else _f64(bias)
    ext = np.concatenate([st, x[:, :, None]], axis=2)    # [nseq, D, K]
    pre = b[None, :] + (w[None, :, :] * ext).sum(axis=2)
    return pre * (1.0 / (1.0 + np.exp(-pre))), ext[:, :, 1:]


def split_xbc(out, H, P, G, N):
    """[T, D] -> x [T,H,P], B [T,G,N], C [T,G,N] (the scan's input layouts)."""
    T = out.shape[0]
    HP, GN = H * P, G * N
    return (out[:, :HP].reshape(T, H, P), out[:, HP:HP + GN].reshape(T, G, N),
            out[:, HP + GN:].reshape(T, G, N))
