"""GPU parity of ssd_state_update (decode) against the FP64 oracle.

Decode is checked the way the SSD contract states it: a prefix prefill on the GPU
produces the state, single-token decode steps continue it, and the oracle runs one
sequential recurrence over the concatenated tokens (RL-Kernel issue page, §4.1:
the same token's output must agree whether it came from prefill or decode).
"""
import pytest
import torch

from mamba_ssd_state_02_b200 import workloads as W
from oracle import oracle as O
from parity_util import TOL_STATE, TOL_Y, rel_err

pytestmark = pytest.mark.gpu


def _decode_run(ssd, dev, w, prefix, steps, pairs, chunk):
    """Prefill `prefix` tokens of every sequence, then `steps` decode steps.
    Token row of (sequence b, position t) is b*(prefix+steps)+t."""
    Ltot = prefix + steps
    nseq, H, P, G, N = w.nseq, w.nheads, w.headdim, w.ngroups, w.dstate
    par = W.make_params(w, device=dev)
    b_idx = torch.arange(nseq, device=dev, dtype=torch.int64)
    pre_rows = (b_idx[:, None] * Ltot + torch.arange(prefix, device=dev)[None, :]).reshape(-1)
    pre = W.make_tokens(w, 0, 0, rows=pre_rows)
    rs = lambda t: t.reshape(nseq, prefix, *t.shape[1:])
    _, state = ssd.scan_fwd(rs(pre["x"]), rs(pre["dt_raw"]), par["dt_bias"], par["A"], rs(pre["B"]),
                            rs(pre["C"]), par["D"], chunk=chunk)
    del pre
    step_rows = (torch.arange(steps, device=dev)[:, None] + prefix + b_idx[None, :] * Ltot).reshape(-1)
    stp = W.make_tokens(w, 0, 0, rows=step_rows)
    xs = stp["x"].view(steps, nseq, H, P)
    dts = stp["dt_raw"].view(steps, nseq, H)
    Bs = stp["B"].view(steps, nseq, G, N)
    Cs = stp["C"].view(steps, nseq, G, N)
    ys = torch.empty(steps, nseq, H, P, dtype=w.dtype, device=dev)
    for k in range(steps):
        ssd.state_update(state, xs[k], dts[k], par["dt_bias"], par["A"], Bs[k], Cs[k], par["D"], y=ys[k])
    ssd.device_status()
    # Oracle: one recurrence over all Ltot tokens of each sampled sequence.
    got_y, ref_y, got_f, ref_f = [], [], [], []
    for b, h in pairs:
        rows = b * Ltot + torch.arange(Ltot, device=dev)
        tok = {k: v.cpu() for k, v in W.make_tokens(w, 0, 0, rows=rows).items()}
        yb, fb = O.ssd_scan(tok["x"], tok["dt_raw"], par["dt_bias"].cpu(), par["A"].cpu(), tok["B"],
                            tok["C"], par["D"].cpu(), pairs=[(0, h)])
        ref_y.append(torch.from_numpy(yb[0][prefix:]).reshape(-1))
        got_y.append(ys[:, b, h, :].cpu().double().reshape(-1))
        ref_f.append(fb[0])
        got_f.append(state[b, h].cpu().double())
    return rel_err(torch.cat(got_y), torch.cat(ref_y)), rel_err(torch.stack(got_f), torch.stack(ref_f))


@pytest.mark.parametrize("dtype,P,N,G", [(torch.bfloat16, 64, 128, 2), (torch.float32, 16, 16, 1),
                                         (torch.float32, 128, 32, 4), (torch.bfloat16, 32, 64, 8)])
def test_decode_small(ssd, cuda_dev, dtype, P, N, G):
    w = W.Workload("decode_small", nheads=8, headdim=P, ngroups=G, dstate=N, chunk=64, dtype=dtype,
                   seqlens=[100] * 5, varlen=False, seed=31)
    pairs = [(b, h) for b in range(5) for h in (0, 3, 7)]
    ey, ef = _decode_run(ssd, cuda_dev, w, 100, 24, pairs, 64)
    assert ey <= TOL_Y[dtype], ey
    assert ef <= TOL_STATE, ef


def test_decode_equals_scan_of_one_token(ssd, cuda_dev):
    """ssd_state_update == ssd_scan_fwd with L=1 continuing from the same state."""
    w = W.Workload("one", nheads=8, headdim=64, ngroups=2, dstate=128, chunk=64, dtype=torch.bfloat16,
                   seqlens=[1] * 6, varlen=False, init="normal", seed=5)
    inp = W.make_all(w, device=cuda_dev)
    st = inp["init_state"].clone()
    y1 = ssd.state_update(st, inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"])
    r = lambda t: t.unsqueeze(1)
    y2, f2 = ssd.scan_fwd(r(inp["x"]), r(inp["dt_raw"]), inp["dt_bias"], inp["A"], r(inp["B"]), r(inp["C"]),
                          inp["D"], init_state=inp["init_state"], chunk=64)
    assert rel_err(y1, y2[:, 0]) <= 1e-2
    assert rel_err(st, f2) <= 1e-5


@pytest.mark.slow
def test_config4_decode_full(ssd, cuda_dev):
    w = W.config(4)
    pairs = [(0, 0), (37, 9), (101, 18), (128, 27), (170, 36), (200, 45), (233, 54), (255, 63)]
    ey, ef = _decode_run(ssd, cuda_dev, w, 2048, w.decode_steps, pairs, w.chunk)
    assert ey <= 1e-2, ey
    assert ef <= TOL_STATE, ef
