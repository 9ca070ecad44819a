"""ctypes wrapper of the FP64 SSD oracle (``ssd_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg may call this module; the product path never does.

It takes CPU tensors exactly as the CUDA path receives them (float32, or bf16,
whose bit patterns the C code widens to double) and returns float64 results.
It imports nothing from the CUDA library's package.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with plain gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-pthread", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        p, i64, i32, d = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.oracle_ssd_scan.argtypes = [i64, p, i32, i32, i32, i32, i32, p, p, p, p, p, p, p, p,
                                      i64, p, p, p, p, i32]
        L.oracle_ssd_scan.restype = i32
        L.oracle_ssd_scan_snapshots.argtypes = [i64, p, i32, i32, i32, i32, i32, p, p, p, p, p, p, p, p,
                                                i64, p, p, p, p, i64, p, p, i32]
        L.oracle_ssd_scan_snapshots.restype = i32
        L.oracle_state_update.argtypes = [i64, i32, i32, i32, i32, i32, p, p, p, p, p, p, p, p, p]
        L.oracle_state_update.restype = i32
        L.oracle_closed_form.argtypes = [i32, i32, i32, i32, i32, i32, p, p, p, p, p, p, p, p, p, p]
        L.oracle_closed_form.restype = i32
        L.oracle_softplus.argtypes = [d]
        L.oracle_softplus.restype = d
        L.oracle_set_mutation.argtypes = [i32]
        L.oracle_set_mutation.restype = None
        _lib = L
    return _lib


def set_mutation(code: int) -> None:
    """Plant a deliberate mistake (code > 0) for the pin tests; 0 restores the oracle."""
    lib().oracle_set_mutation(int(code))


def softplus(z: float) -> float:
    return lib().oracle_softplus(float(z))


def _cpu(t, dtype=None):
    if t is None:
        return None
    t = t.detach().to("cpu")
    if dtype is not None:
        t = t.to(dtype)
    return t.contiguous()


def _dtype_code(x: torch.Tensor) -> int:
    if x.dtype == torch.float32:
        return 0
    if x.dtype == torch.bfloat16:
        return 1
    raise TypeError(f"oracle takes float32 or bf16 x/B/C, got {x.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def seq_offsets(T: int, cu_seqlens=None, batch: int | None = None) -> np.ndarray:
    if cu_seqlens is not None:
        return np.asarray(_cpu(cu_seqlens).numpy(), dtype=np.int64)
    b = 1 if batch is None else int(batch)
    L = T // b if b > 0 else 0
    return np.arange(b + 1, dtype=np.int64) * L


def ssd_scan(x, dt_raw, dt_bias, A, B, C, D, init_state=None, cu_seqlens=None, batch=None,
             pairs=None, want_y=True, nthreads=None, snapshot_tokens=None):
    """Run the recurrence.

    x [T,H,P], dt_raw [T,H], B/C [T,G,N] (packed tokens), dt_bias/A/D [H];
    init_state [nseq,H,P,N] or None; cu_seqlens [nseq+1] or None (dense: ``batch``
    rows of T/batch tokens).

    pairs=None: returns (y [T,H,P] float64, final [nseq,H,P,N] float64).
    pairs=[(s,h), ...]: returns (list of y blocks [len_s,P], final [npairs,P,N]).
    snapshot_tokens=I adds a third result, the state after every I tokens of each
    sequence: [n_snap,H,P,N] ordered by sequence, then position (pairs=None), or a list
    of [len_s // I, P, N] blocks (pairs given).
    """
    x, B, C = _cpu(x), _cpu(B), _cpu(C)
    dtype = _dtype_code(x)
    if B.dtype != x.dtype or C.dtype != x.dtype:
        raise TypeError("x, B and C must share a dtype")
    T, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    dt_raw = _cpu(dt_raw, torch.float32)
    dt_bias, A_, D_ = (_cpu(v, torch.float32) for v in (dt_bias, A, D))
    off = seq_offsets(T, cu_seqlens, batch)
    nseq = len(off) - 1
    init = _cpu(init_state, torch.float64)
    all_pairs = pairs is None
    if all_pairs:
        pairs = [(s, h) for s in range(nseq) for h in range(H)]
    pr = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
    lens = (off[pr[:, 0] + 1] - off[pr[:, 0]]) if len(pr) else np.zeros(0, np.int64)
    yoff = np.zeros(len(pr), dtype=np.int64)
    if len(pr) > 1:
        yoff[1:] = np.cumsum(lens[:-1] * P)
    ybuf = np.zeros(int(lens.sum()) * P if want_y else 1, dtype=np.float64)
    fin = np.zeros((len(pr), P, N), dtype=np.float64)
    I = int(snapshot_tokens or 0)
    nsn = lens // I if I > 0 else np.zeros(len(pr), np.int64)
    soff = np.zeros(len(pr), dtype=np.int64)
    if len(pr) > 1:
        soff[1:] = np.cumsum(nsn[:-1] * P * N)
    sbuf = np.zeros(max(1, int(nsn.sum()) * P * N), dtype=np.float64)
    rc = lib().oracle_ssd_scan_snapshots(
        nseq, off.ctypes.data_as(ctypes.c_void_p), H, P, G, N, dtype, _ptr(x), _ptr(dt_raw),
        _ptr(dt_bias), _ptr(A_), _ptr(B), _ptr(C), _ptr(D_), _ptr(init), len(pr),
        pr.ctypes.data_as(ctypes.c_void_p), yoff.ctypes.data_as(ctypes.c_void_p),
        ybuf.ctypes.data_as(ctypes.c_void_p) if want_y else None,
        fin.ctypes.data_as(ctypes.c_void_p), I, soff.ctypes.data_as(ctypes.c_void_p),
        sbuf.ctypes.data_as(ctypes.c_void_p), nthreads or _threads())
    if rc != 0:
        raise ValueError("oracle_ssd_scan rejected its arguments")
    blocks = [ybuf[o:o + l * P].reshape(l, P) for o, l in zip(yoff, lens)] if want_y else None
    sblocks = [sbuf[o:o + n * P * N].reshape(n, P, N) for o, n in zip(soff, nsn)] if I > 0 else None
    if not all_pairs:
        if I > 0:
            return blocks, torch.from_numpy(fin), [torch.from_numpy(b) for b in sblocks]
        return blocks, torch.from_numpy(fin)
    y = None
    if want_y:
        y = np.zeros((T, H, P), dtype=np.float64)
        for (s, h), blk in zip(pr, blocks):
            y[off[s]:off[s + 1], h, :] = blk
        y = torch.from_numpy(y)
    fin_t = torch.from_numpy(fin.reshape(nseq, H, P, N))
    if I > 0:
        per_seq = (off[1:] - off[:-1]) // I
        snaps = np.zeros((int(per_seq.sum()), H, P, N), dtype=np.float64)
        first = np.concatenate([[0], np.cumsum(per_seq)])
        for (s, h), blk in zip(pr, sblocks):
            snaps[first[s]:first[s + 1], h] = blk
        return y, fin_t, torch.from_numpy(snaps)
    return y, fin_t


def state_update(state, x, dt_raw, dt_bias, A, B, C, D):
    """One decode step. state [nseq,H,P,N] (any float dtype, not modified);
    x [nseq,H,P], dt_raw [nseq,H], B/C [nseq,G,N]. Returns (new_state, y) float64."""
    x, B, C = _cpu(x), _cpu(B), _cpu(C)
    dtype = _dtype_code(x)
    nseq, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    st = _cpu(state, torch.float64).clone()
    y = torch.zeros(nseq, H, P, dtype=torch.float64)
    dt_raw = _cpu(dt_raw, torch.float32)
    dt_bias, A_, D_ = (_cpu(v, torch.float32) for v in (dt_bias, A, D))
    rc = lib().oracle_state_update(nseq, H, P, G, N, dtype, _ptr(st), _ptr(x), _ptr(dt_raw),
                                   _ptr(dt_bias), _ptr(A_), _ptr(B), _ptr(C), _ptr(D_), _ptr(y))
    if rc != 0:
        raise ValueError("oracle_state_update rejected its arguments")
    return st, y


def closed_form(x, dt_raw, dt_bias, A, B, C, D, h0=None):
    """Brute-force quadratic form for ONE dense sequence: x [L,H,P], B/C [L,G,N],
    h0 [H,P,N] or None. Returns (y [L,H,P], h_L [H,P,N]) float64."""
    x, B, C = _cpu(x), _cpu(B), _cpu(C)
    dtype = _dtype_code(x)
    L, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    y = torch.zeros(L, H, P, dtype=torch.float64)
    hL = torch.zeros(H, P, N, dtype=torch.float64)
    dt_raw = _cpu(dt_raw, torch.float32)
    dt_bias, A_, D_ = (_cpu(v, torch.float32) for v in (dt_bias, A, D))
    h0 = _cpu(h0, torch.float64)
    rc = lib().oracle_closed_form(L, H, P, G, N, dtype, _ptr(x), _ptr(dt_raw), _ptr(dt_bias),
                                  _ptr(A_), _ptr(B), _ptr(C), _ptr(D_), _ptr(h0), _ptr(y), _ptr(hL))
    if rc != 0:
        raise ValueError("oracle_closed_form rejected its arguments")
    return y, hL
