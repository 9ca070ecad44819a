"""Pins of the FP64 conv1d prologue oracle against things other than itself: numpy's
convolution for the linear part (a reversed or shifted tap order fails), scipy's
logistic function for the SiLU, and the conv-state cache semantics (handoff across a
split sequence, a decode step, a sequence shorter than the state, empty sequences)."""
import numpy as np
import pytest
import torch
from scipy.special import expit

from mamba_ssd_state_02_b200 import workloads as W
from oracle import conv_oracle as CO


def _wl(seqlens, dtype=torch.float32, seed=3):
    return W.Workload("conv", nheads=2, headdim=16, ngroups=1, dstate=16, chunk=64, dtype=dtype,
                      seqlens=seqlens, varlen=True, init="zero", seed=seed)


@pytest.mark.parametrize("K", [2, 3, 4])
def test_linear_part_is_numpy_convolution(K):
    w = _wl([50, 2, 70])
    ci = W.make_conv_inputs(w, K)
    pre, _ = CO.conv1d_fwd(ci["xbc"], ci["weight"], ci["bias"], ci["conv_state"], ci["cu_seqlens"], act=False)
    x, wt, b = ci["xbc"].double().numpy(), ci["weight"].double().numpy(), ci["bias"].double().numpy()
    cu = ci["cu_seqlens"].tolist()
    for s in range(3):
        for c in (0, 17, 63):
            seq = np.concatenate([ci["conv_state"][s, c].double().numpy(), x[cu[s]:cu[s + 1], c]])
            ref = np.convolve(seq, wt[c][::-1])[K - 1:K - 1 + cu[s + 1] - cu[s]] + b[c]
            assert np.abs(pre[cu[s]:cu[s + 1], c] - ref).max() < 1e-12


def test_activation_is_silu():
    w = _wl([40])
    ci = W.make_conv_inputs(w, 4)
    pre, _ = CO.conv1d_fwd(ci["xbc"], ci["weight"], ci["bias"], ci["conv_state"], ci["cu_seqlens"], act=False)
    out, _ = CO.conv1d_fwd(ci["xbc"], ci["weight"], ci["bias"], ci["conv_state"], ci["cu_seqlens"])
    assert np.abs(out - pre * expit(pre)).max() < 1e-12


def test_state_handoff_and_decode_step():
    """Running a sequence in two pieces, the second starting from the first's final
    state, equals running it whole; a decode step equals a one-token prefill."""
    w = _wl([90])
    ci = W.make_conv_inputs(w, 4)
    full, fin = CO.conv1d_fwd(ci["xbc"], ci["weight"], ci["bias"], ci["conv_state"], batch=1)
    a, fa = CO.conv1d_fwd(ci["xbc"][:37], ci["weight"], ci["bias"], ci["conv_state"], batch=1)
    b, fb = CO.conv1d_fwd(ci["xbc"][37:], ci["weight"], ci["bias"], torch.from_numpy(fa), batch=1)
    assert np.array_equal(np.concatenate([a, b]), full) and np.array_equal(fb, fin)
    o1, s1 = CO.conv1d_update(torch.from_numpy(fa), ci["xbc"][37:38], ci["weight"], ci["bias"])
    assert np.abs(o1 - b[:1]).max() < 1e-12
    assert np.array_equal(s1, CO.conv1d_fwd(ci["xbc"][37:38], ci["weight"], ci["bias"], torch.from_numpy(fa),
                                            batch=1)[1])


def test_short_and_empty_sequences_keep_the_incoming_state():
    w = _wl([2, 0, 5])
    ci = W.make_conv_inputs(w, 4)
    _, fin = CO.conv1d_fwd(ci["xbc"], ci["weight"], ci["bias"], ci["conv_state"], ci["cu_seqlens"])
    st = ci["conv_state"].double().numpy()
    x = ci["xbc"].double().numpy()
    # sequence 0 has 2 tokens: its final state is [oldest state entry, x0, x1]
    assert np.array_equal(fin[0][:, 0], st[0][:, 2]) and np.array_equal(fin[0][:, 1:], x[0:2].T)
    assert np.array_equal(fin[1], st[1])                 # empty sequence: state unchanged
    assert np.array_equal(fin[2], x[4:7].T)              # last 3 of its 5 tokens
