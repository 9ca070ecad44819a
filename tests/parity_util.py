"""Helpers shared by the GPU parity tests: run the CUDA path and the FP64 oracle on
the same seeded inputs and compare them with the error metric of the SSD contract:
max|y - y_ref| / max|y_ref| over the compared elements (y), and the same for the
final state. Tolerances: y <= 1e-2 for bf16 inputs, <= 1e-4 for float32 inputs;
final state <= 1e-3."""
from __future__ import annotations

import torch

from mamba_ssd_state_02_b200 import workloads as W
from oracle import oracle as O

TOL_Y = {torch.bfloat16: 1e-2, torch.float32: 1e-4}
TOL_STATE = 1e-3


def rel_err(got, ref) -> float:
    got = torch.as_tensor(got).to("cpu", torch.float64)
    ref = torch.as_tensor(ref).to("cpu", torch.float64)
    den = ref.abs().max().item()
    err = (got - ref).abs().max().item()
    if den == 0.0:
        return err
    return err / den


def seq_bounds(w: W.Workload):
    off = [0]
    for L in w.seqlens:
        off.append(off[-1] + int(L))
    return off


def run_gpu_scan(ssd, w: W.Workload, inp: dict, dev, chunk=None, workspace=None):
    """Call ssd.scan_fwd on packed [T,...] inputs (moved to dev). Returns (y [T,H,P], final)."""
    g = lambda t: None if t is None else t.to(dev)
    x, dt_raw, B, C = g(inp["x"]), g(inp["dt_raw"]), g(inp["B"]), g(inp["C"])
    q = w.chunk if chunk is None else chunk
    if w.varlen:
        y, fin = ssd.scan_fwd(x, dt_raw, g(inp["dt_bias"]), g(inp["A"]), B, C, g(inp["D"]),
                              init_state=g(inp["init_state"]), cu_seqlens=g(inp["cu_seqlens"]),
                              chunk=q, workspace=workspace)
        return y, fin
    b, L = w.nseq, w.seqlens[0]
    rs = lambda t: t.reshape(b, L, *t.shape[1:])
    y, fin = ssd.scan_fwd(rs(x), rs(dt_raw), g(inp["dt_bias"]), g(inp["A"]), rs(B), rs(C),
                          g(inp["D"]), init_state=g(inp["init_state"]), chunk=q, workspace=workspace)
    return y.reshape(b * L, *y.shape[2:]), fin


def oracle_scan(w: W.Workload, inp: dict, pairs=None):
    cpu = {k: (None if v is None else v.to("cpu")) for k, v in inp.items()}
    cu = cpu["cu_seqlens"]
    return O.ssd_scan(cpu["x"], cpu["dt_raw"], cpu["dt_bias"], cpu["A"], cpu["B"], cpu["C"],
                      cpu["D"], init_state=cpu["init_state"], cu_seqlens=cu,
                      batch=None if w.varlen else w.nseq, pairs=pairs)


def compare_pairs(w, y_gpu, fin_gpu, y_blocks, fin_ref, pairs):
    """Errors over the sampled (sequence, head) pairs."""
    off = seq_bounds(w)
    got_y, ref_y, got_f = [], [], []
    yc = y_gpu.to("cpu", torch.float64)
    fc = fin_gpu.to("cpu", torch.float64)
    for (s, h), blk in zip(pairs, y_blocks):
        got_y.append(yc[off[s]:off[s + 1], h, :].reshape(-1))
        ref_y.append(torch.from_numpy(blk).reshape(-1))
        got_f.append(fc[s, h])
    ey = rel_err(torch.cat(got_y), torch.cat(ref_y))
    ef = rel_err(torch.stack(got_f), fin_ref)
    return ey, ef
