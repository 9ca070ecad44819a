"""Pins for the FP64 oracle: each checks it against something other than itself.

* the quadratic closed form of the SSD map, brute-forced on tiny inputs;
* the A = 0, D = 0 case, where the scan is a cumulative sum (numpy.cumsum), and
  its N = 1, B = C = 1 special case, a plain prefix sum of dt * x;
* worked-by-hand scalar examples under tests/golden/ (recurrence, dt, D skip,
  varlen reset with initial states);
* degenerate cases (C = 0, B = 0, memoryless strong decay), linearity in (x, h0),
  the contiguous head -> group map, split invariance (prefill then continue from
  the final state, including single-token decode steps);
* a mutation check: every deliberate mistake planted in the oracle makes at least
  one of these pins fail.

The recurrence: RL-Kernel issue page (Nemotron-3-Nano-30B-A3B) section 1 and
Figure 2; D skip and B/C groups: JAX Nemotron 3 Nano page ("Key Components",
NemotronConfig); split invariance: RL-Kernel issue page section 4.1.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O
from mamba_ssd_state_02_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LN2 = math.log(2.0)


def _rand_problem(seed, L, H, P, G, N, dtype=torch.float32, with_h0=False, nseq=1):
    g = torch.Generator().manual_seed(seed)
    T = L * nseq
    x = torch.randn(T, H, P, generator=g).to(dtype)
    dt_raw = torch.randn(T, H, generator=g)
    dt_bias = torch.rand(H, generator=g) * 2 - 3        # softplus ~ 0.05 .. 0.3
    A = -torch.exp(torch.rand(H, generator=g) * math.log(16))
    B = (torch.randn(T, G, N, generator=g) / math.sqrt(N)).to(dtype)
    C = (torch.randn(T, G, N, generator=g) / math.sqrt(N)).to(dtype)
    D = torch.rand(H, generator=g)
    h0 = torch.randn(nseq, H, P, N, generator=g, dtype=torch.float64) if with_h0 else None
    return dict(x=x, dt_raw=dt_raw, dt_bias=dt_bias, A=A, B=B, C=C, D=D, h0=h0)


def _rel(a, b):
    a = torch.as_tensor(a, dtype=torch.float64)
    b = torch.as_tensor(b, dtype=torch.float64)
    den = b.abs().max().item()
    return (a - b).abs().max().item() / (den if den > 0 else 1.0)


# ----------------------------------------------------------------------------- pins
# Each pin returns True when the oracle agrees with the independent expectation.

def pin_closed_form():
    ok = True
    cases = [(1, 1, 1, 1, 1, False), (7, 2, 3, 1, 4, True), (33, 4, 8, 2, 8, True),
             (48, 4, 4, 2, 5, False), (19, 2, 2, 2, 3, True)]
    for i, (L, H, P, G, N, h0) in enumerate(cases):
        for dtype in (torch.float32, torch.bfloat16):
            d = _rand_problem(10 + i, L, H, P, G, N, dtype, h0)
            y, fin = O.ssd_scan(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                                init_state=d["h0"])
            yc, hc = O.closed_form(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"],
                                   d["D"], h0=None if d["h0"] is None else d["h0"][0])
            ok &= _rel(y, yc) < 1e-12 and _rel(fin[0], hc) < 1e-12
    return ok


def pin_cumsum():
    """A = 0, D = 0: y_t = C_t . (h0 + sum_{s<=t} dt_s x_s B_s^T)."""
    L, H, P, G, N = 40, 2, 3, 1, 4
    d = _rand_problem(3, L, H, P, G, N, torch.float32, True)
    A = torch.zeros(H)
    D = torch.zeros(H)
    y, fin = O.ssd_scan(d["x"], d["dt_raw"], d["dt_bias"], A, d["B"], d["C"], D, init_state=d["h0"])
    z = (d["dt_raw"].double() + d["dt_bias"].double())
    dt = np.log1p(np.exp(z.numpy()))                                    # [L,H]
    x = d["x"].double().numpy()
    Bm = d["B"].double().numpy()[:, 0, :]
    Cm = d["C"].double().numpy()[:, 0, :]
    terms = dt[:, :, None, None] * x[:, :, :, None] * Bm[:, None, None, :]   # [L,H,P,N]
    h = np.cumsum(terms, axis=0) + d["h0"].numpy()[0][None]
    y_ref = np.einsum("tn,thpn->thp", Cm, h)
    return _rel(y, y_ref) < 1e-12 and _rel(fin[0], h[-1]) < 1e-12


def pin_prefix_sum():
    """N = 1, B = C = 1, A = 0, D = 0, constant dt: y = dt * cumsum(x)."""
    L, H, P = 50, 1, 2
    g = torch.Generator().manual_seed(5)
    x = torch.randn(L, H, P, generator=g)
    dt_raw = torch.zeros(L, H)
    dt_bias = torch.tensor([0.25])
    ones = torch.ones(L, 1, 1)
    y, _ = O.ssd_scan(x, dt_raw, dt_bias, torch.zeros(1), ones, ones, torch.zeros(1))
    dt = math.log1p(math.exp(0.25))
    return _rel(y[:, 0, :], dt * np.cumsum(x[:, 0, :].double().numpy(), axis=0)) < 1e-13


def _golden_case(name):
    with open(os.path.join(GOLDEN, name)) as f:
        gd = json.load(f)
    inp = gd["inputs"]
    T = len(inp["x"])
    x = torch.tensor(inp["x"], dtype=torch.float32).view(T, 1, 1)
    B = torch.tensor(inp["B"], dtype=torch.float32).view(T, 1, 1)
    C = torch.tensor(inp["C"], dtype=torch.float32).view(T, 1, 1)
    dt_raw = torch.tensor(inp["dt_raw"], dtype=torch.float32).view(T, 1)
    f = lambda k: torch.tensor(inp[k], dtype=torch.float32)
    cu = np.concatenate([[0], np.cumsum(inp["seqlens"])]).astype(np.int32)
    h0 = None
    if inp["h0"] is not None:
        h0 = torch.tensor(inp["h0"], dtype=torch.float64).view(-1, 1, 1, 1)
    y, fin = O.ssd_scan(x, dt_raw, f("dt_bias"), f("A"), B, C, f("D"), init_state=h0,
                        cu_seqlens=torch.from_numpy(cu))
    ey = np.array([a * LN2 + b for a, b in gd["expected"]["y_ln2_coeff_and_const"]])
    ef = np.array([a * LN2 + b for a, b in gd["expected"]["final_ln2_coeff_and_const"]])
    return (np.abs(y.numpy().reshape(-1) - ey).max() < 1e-14 and
            np.abs(fin.numpy().reshape(-1) - ef).max() < 1e-14)


def pin_golden_scalar():
    return _golden_case("scalar_three_tokens.json")


def pin_golden_varlen():
    return _golden_case("varlen_reset_init.json")


def pin_group_map():
    """H=4, G=2: heads 0,1 read group 0 and heads 2,3 read group 1 (GQA-style blocks).
    Group 1 has B = 0, so heads 2,3 keep a zero state and output exactly D*x."""
    L, H, P, G, N = 9, 4, 2, 2, 3
    d = _rand_problem(7, L, H, P, G, N)
    B = d["B"].clone()
    B[:, 1, :] = 0
    y, fin = O.ssd_scan(d["x"], d["dt_raw"], d["dt_bias"], d["A"], B, d["C"], d["D"])
    dx = d["D"].double()[None, :, None] * d["x"].double()
    zero_heads = torch.equal(y[:, 2:], dx[:, 2:]) and float(fin[0, 2:].abs().max()) == 0.0
    live_heads = float(fin[0, :2].abs().min()) > 0.0 and float((y[:, :2] - dx[:, :2]).abs().max()) > 1e-3
    return zero_heads and live_heads


def pin_degenerate():
    L, H, P, G, N = 12, 2, 3, 1, 4
    d = _rand_problem(8, L, H, P, G, N, torch.float32, True)
    dx = d["D"].double()[None, :, None] * d["x"].double()
    y, _ = O.ssd_scan(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], torch.zeros_like(d["C"]),
                      d["D"], init_state=d["h0"])
    c0 = torch.equal(y, dx)
    y, fin = O.ssd_scan(d["x"], d["dt_raw"], d["dt_bias"], d["A"], torch.zeros_like(d["B"]), d["C"],
                        d["D"])
    b0 = torch.equal(y, dx) and float(fin.abs().max()) == 0.0
    # memoryless: dt ~ 20, A = -16 -> exp(dt*A) ~ e^-320, y_t = dt_t (C_t.B_t) x_t + D x_t
    dt_bias = torch.full((H,), 20.0)
    A = torch.full((H,), -16.0)
    y, _ = O.ssd_scan(d["x"], torch.zeros(L, H), dt_bias, A, d["B"], d["C"], d["D"])
    dt = 20.0 + math.log1p(math.exp(-20.0))
    cb = (d["C"].double()[:, 0, :] * d["B"].double()[:, 0, :]).sum(-1)      # [L]
    y_ref = dt * cb[:, None, None] * d["x"].double() + dx
    mem = _rel(y, y_ref) < 1e-13
    return c0 and b0 and mem


def pin_linearity():
    L, H, P, G, N = 15, 2, 2, 1, 3
    d = _rand_problem(9, L, H, P, G, N, torch.float32, True)
    g = torch.Generator().manual_seed(99)
    x1 = torch.randint(-8, 8, (L, H, P), generator=g).float()
    x2 = torch.randint(-8, 8, (L, H, P), generator=g).float()
    h1 = torch.randint(-8, 8, (1, H, P, N), generator=g).double()
    h2 = torch.randint(-8, 8, (1, H, P, N), generator=g).double()
    args = lambda x: (x, d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"])
    ya, fa = O.ssd_scan(*args(x1), init_state=h1)
    yb, fb = O.ssd_scan(*args(x2), init_state=h2)
    ys, fs = O.ssd_scan(*args(x1 + x2), init_state=h1 + h2)
    return _rel(ys, ya + yb) < 1e-12 and _rel(fs, fa + fb) < 1e-12


def pin_split_invariance():
    """Prefill [0, L1), continue from its final state over [L1, L2) as a second
    prefill, then over [L2, L) as single-token decode steps == one-shot prefill."""
    L, L1, L2, H, P, G, N = 30, 11, 23, 4, 3, 2, 4
    d = _rand_problem(4, L, H, P, G, N, torch.bfloat16, True)
    sl = lambda a, b: {k: (v[a:b] if k in ("x", "dt_raw", "B", "C") else v) for k, v in d.items()}
    full_y, full_f = O.ssd_scan(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                                init_state=d["h0"])
    p1 = sl(0, L1)
    y1, f1 = O.ssd_scan(p1["x"], p1["dt_raw"], d["dt_bias"], d["A"], p1["B"], p1["C"], d["D"],
                        init_state=d["h0"])
    p2 = sl(L1, L2)
    y2, f2 = O.ssd_scan(p2["x"], p2["dt_raw"], d["dt_bias"], d["A"], p2["B"], p2["C"], d["D"],
                        init_state=f1)
    st = f2
    ys = [y1, y2]
    for t in range(L2, L):
        st, yt = O.state_update(st, d["x"][t:t + 1], d["dt_raw"][t:t + 1], d["dt_bias"], d["A"],
                                d["B"][t:t + 1], d["C"][t:t + 1], d["D"])
        ys.append(yt)
    return _rel(torch.cat(ys), full_y) < 1e-12 and _rel(st, full_f) < 1e-12


def pin_varlen_equals_separate():
    lens = [5, 1, 0, 9]
    H, P, G, N = 2, 2, 1, 3
    T = sum(lens)
    d = _rand_problem(12, T, H, P, G, N, torch.float32, False)
    h0 = torch.randn(len(lens), H, P, N, generator=torch.Generator().manual_seed(1), dtype=torch.float64)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    y, fin = O.ssd_scan(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                        init_state=h0, cu_seqlens=cu)
    ok = True
    for s, (a, b) in enumerate(zip(cu[:-1].tolist(), cu[1:].tolist())):
        ys, fs = O.ssd_scan(d["x"][a:b], d["dt_raw"][a:b], d["dt_bias"], d["A"], d["B"][a:b],
                            d["C"][a:b], d["D"], init_state=h0[s:s + 1])
        ok &= torch.equal(y[a:b], ys) and torch.equal(fin[s], fs[0])
    ok &= torch.equal(fin[2], h0[2])        # an empty sequence keeps its initial state
    return ok


def pin_softplus():
    vals = [(0.0, LN2), (1.0, math.log(1 + math.e)), (-3.0, math.log1p(math.exp(-3.0))),
            (40.0, 40.0 + math.exp(-40.0)), (-40.0, math.exp(-40.0))]
    return all(abs(O.softplus(z) - v) <= 1e-15 * max(1.0, abs(v)) for z, v in vals)


PINS = [pin_closed_form, pin_cumsum, pin_prefix_sum, pin_golden_scalar, pin_golden_varlen,
        pin_group_map, pin_degenerate, pin_linearity, pin_split_invariance,
        pin_varlen_equals_separate, pin_softplus]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin_holds(pin):
    O.set_mutation(0)
    assert pin()


MUTATIONS = {1: "drop D skip", 2: "head->group h % G", 3: "no softplus", 4: "decay exp(A)",
             5: "input term without dt", 6: "y from h_{t-1}", 7: "C used for B",
             8: "initial state ignored"}


@pytest.mark.parametrize("code", sorted(MUTATIONS), ids=lambda c: MUTATIONS[c])
def test_planted_mistake_is_caught(code):
    try:
        O.set_mutation(code)
        failed = [p.__name__ for p in PINS if not p()]
    finally:
        O.set_mutation(0)
    assert failed, f"mutation '{MUTATIONS[code]}' passed every pin"


def test_oracle_rejects_bad_dims():
    d = _rand_problem(1, 4, 3, 2, 1, 2)
    with pytest.raises(ValueError):
        O.ssd_scan(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"].expand(4, 2, 2).contiguous(),
                   d["C"].expand(4, 2, 2).contiguous(), d["D"])   # H=3 not divisible by G=2


def test_snapshots_equal_prefix_final_states():
    """A snapshot (state after the first m*I tokens of a sequence) is, by definition, the
    final state of the same sequence cut after m*I tokens; the last one of a sequence
    whose length is a multiple of I is its final state."""
    w = W.Workload("snap", nheads=4, headdim=8, ngroups=2, dstate=8, chunk=64, dtype=torch.float32,
                   seqlens=[300, 17, 256], varlen=True, init="normal", seed=5)
    d = W.make_all(w)
    I = 64
    y, fin, sn = O.ssd_scan(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                            init_state=d["init_state"], cu_seqlens=d["cu_seqlens"], snapshot_tokens=I)
    per = [300 // I, 17 // I, 256 // I]
    assert sn.shape == (sum(per), 4, 8, 8)
    cu = d["cu_seqlens"].tolist()
    first = [0, per[0], per[0] + per[1]]
    for s in range(3):
        for m in range(1, per[s] + 1):
            sl = slice(cu[s], cu[s] + m * I)
            _, f2 = O.ssd_scan(d["x"][sl], d["dt_raw"][sl], d["dt_bias"], d["A"], d["B"][sl], d["C"][sl],
                               d["D"], init_state=d["init_state"][s:s + 1], batch=1)
            assert torch.equal(sn[first[s] + m - 1], f2[0])
    assert torch.equal(sn[-1], fin[2])                       # 256 = 4 * 64: the final state
    # Without snapshots the results are unchanged.
    y0, fin0 = O.ssd_scan(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                          init_state=d["init_state"], cu_seqlens=d["cu_seqlens"])
    assert torch.equal(y0, y) and torch.equal(fin0, fin)
