"""Host-side checks of the seeded input generator (no SSD arithmetic involved)."""
import math

import torch

from mamba_ssd_state_02_b200 import workloads as W


def test_splitmix64_known_values():
    # splitmix64 outputs for state 0 (Vigna's reference generator: the first three
    # outputs of a generator seeded with 0 are the finaliser at counters 0, 1, 2
    # when the golden-ratio increment is applied once per call).
    z = torch.tensor([0], dtype=torch.int64)
    out = []
    state = 0
    for _ in range(3):
        out.append(int(W._splitmix64(torch.tensor([state], dtype=torch.int64))[0]) & ((1 << 64) - 1))
        state = (state + 0x9E3779B97F4A7C15) & ((1 << 64) - 1)
        state = state - (1 << 64) if state >= (1 << 63) else state
    assert out == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_rows_match_contiguous_draws():
    w = W.config(1)
    full = W.make_tokens(w, 40, 60)
    rows = torch.tensor([41, 59, 40])
    part = W.make_tokens(w, 0, 0, rows=rows)
    for k in ("x", "dt_raw", "B", "C"):
        assert torch.equal(part[k][0], full[k][1])
        assert torch.equal(part[k][1], full[k][19])
        assert torch.equal(part[k][2], full[k][0])


def test_deterministic_and_distributions():
    w = W.config(1)
    a = W.make_tokens(w, 0, 64)
    b = W.make_tokens(w, 0, 64)
    assert all(torch.equal(a[k], b[k]) for k in a)
    x = a["x"].float()
    assert abs(x.mean().item()) < 0.02 and abs(x.std().item() - 1) < 0.02
    Bs = a["B"].float().std().item() * math.sqrt(w.dstate)
    assert abs(Bs - 1) < 0.05
    assert a["x"].dtype == torch.bfloat16 and a["dt_raw"].dtype == torch.float32


def test_params_ranges():
    for k, (lo, hi) in ((1, (1e-3, 0.1)), (2, (1e-4, 0.5))):
        p = W.make_params(W.config(k))
        dt0 = torch.nn.functional.softplus(p["dt_bias"].double())
        assert dt0.min() >= lo * 0.999 and dt0.max() <= hi * 1.001
        assert (p["A"] <= -1).all() and (p["A"] >= -16).all()
        assert (p["D"] >= 0).all() and (p["D"] < 1).all()


def test_varlen_lengths_and_offsets():
    w = W.config(3)
    assert w.nseq == 16 and all(512 <= L <= 8192 for L in w.seqlens)
    cu = W.cu_seqlens(w)
    assert cu[0] == 0 and cu[-1] == w.total_tokens and (cu[1:] >= cu[:-1]).all()


def test_init_state_std():
    w = W.config(1)
    w.seqlens = [64]
    s = W.make_init_state(w)
    assert s.shape == (1, 64, 64, 128) and abs(s.std().item() - 0.1) < 0.002
