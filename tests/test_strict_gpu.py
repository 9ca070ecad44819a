"""Strict mode on the GPU: ssd_strict_scan_fwd and the chunk-emulating decode
ssd_strict_state_update.

Two kinds of check (RL-Kernel issue page, §7: parity between two strict paths is
bitwise, correctness is a tolerance against an independent FP64 reference):

* correctness: the strict prefill's y, final state and cached state, and the decode's
  y, against the FP64 oracle within the SSD contract's tolerances;
* invariance (§4.1), bitwise on the raw bit patterns: a sequence split into a strict
  prefill of any length followed by decode steps, into strict prefills at chunk
  boundaries, or into prefill -> decode -> prefill, gives the same y bits and the same
  cache as one strict prefill over the whole sequence; batch composition, packing and
  dense layout change no bit.
"""
import pytest
import torch

from mamba_ssd_state_02_b200 import workloads as W
from oracle import oracle as O
from parity_util import TOL_STATE, TOL_Y, rel_err

pytestmark = pytest.mark.gpu


def _w(seqlens, dtype=torch.bfloat16, H=8, P=64, G=2, N=128, chunk=128, seed=61, dt_range=(1e-3, 0.1)):
    return W.Workload("strict", nheads=H, headdim=P, ngroups=G, dstate=N, chunk=chunk, dtype=dtype,
                      seqlens=list(seqlens), varlen=True, init="normal", seed=seed, dt_range=dt_range)


def _bits(t):
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


def assert_same_bits(a, b, what):
    assert a.shape == b.shape, what
    eq = _bits(a.contiguous()) == _bits(b.contiguous())
    assert bool(eq.all()), f"{what}: {int((~eq).sum())} of {eq.numel()} elements differ in bits"


def _cache(ssd, w, dev, init=None):
    c = ssd.ChunkCache.empty(w.nseq, w.nheads, w.headdim, w.ngroups, w.dstate, w.chunk, w.dtype, dev)
    if init is not None:
        c.set_state(init)
    return c


def _rows(inp, idx):
    return {k: inp[k][idx].contiguous() for k in ("x", "dt_raw", "B", "C")}


def _prefill(ssd, w, inp, rows, lens, cache, resume=True):
    """Strict prefill of the packed token rows `rows` (sequence s owns lens[s] of them)."""
    cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()), dtype=torch.int32,
                      device=inp["x"].device)
    t = _rows(inp, rows)
    return ssd.strict_scan_fwd(t["x"], t["dt_raw"], inp["dt_bias"], inp["A"], t["B"], t["C"], inp["D"],
                               cache, resume=resume, cu_seqlens=cu)


def _seq_rows(cu, s, a, b, dev):
    return torch.arange(cu[s] + a, cu[s] + b, device=dev)


def _assert_cache_equal(c1, c2, G, H):
    assert torch.equal(c1.len, c2.len)
    assert_same_bits(c1.state, c2.state, "cache.state")
    for s in range(c1.len.shape[0]):
        n = int(c1.len[s, 0])
        assert_same_bits(c1.x[s, :, :n], c2.x[s, :, :n], "cache.x")
        assert_same_bits(c1.dt[s, :, :n], c2.dt[s, :, :n], "cache.dt")
        assert_same_bits(c1.acum[s, :, :n], c2.acum[s, :, :n], "cache.acum")
        assert_same_bits(c1.B[s, :, :n], c2.B[s, :, :n], "cache.B")


# --------------------------------------------------------------------------------------
# Correctness against the FP64 oracle.
@pytest.mark.parametrize("dtype,chunk,P,N", [
    (torch.bfloat16, 128, 64, 128), (torch.float32, 128, 64, 128), (torch.bfloat16, 64, 32, 64),
    (torch.float32, 256, 16, 16), (torch.bfloat16, 256, 128, 128),
])
def test_strict_prefill_matches_oracle(ssd, cuda_dev, dtype, chunk, P, N):
    w = _w([1, 127, 128, 129, 300, 0, 517], dtype=dtype, P=P, N=N, chunk=chunk, dt_range=(1e-4, 0.5))
    inp = W.make_all(w, device=cuda_dev)
    cache = _cache(ssd, w, cuda_dev, inp["init_state"])
    y, fin = ssd.strict_scan_fwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"],
                                 inp["D"], cache, resume=True, cu_seqlens=inp["cu_seqlens"])
    ssd.device_status()
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    y_ref, fin_ref, snaps = O.ssd_scan(cpu["x"], cpu["dt_raw"], cpu["dt_bias"], cpu["A"], cpu["B"], cpu["C"],
                                       cpu["D"], init_state=cpu["init_state"], cu_seqlens=cpu["cu_seqlens"],
                                       snapshot_tokens=chunk)
    assert rel_err(y, y_ref) <= TOL_Y[dtype]
    assert rel_err(fin, fin_ref) <= TOL_STATE
    # The cached state is the state after each sequence's last full chunk.
    k = 0
    ref_state = []
    for s, L in enumerate(w.seqlens):
        full = L // chunk
        ref_state.append(snaps[k + full - 1] if full > 0 else cpu["init_state"][s].double())
        k += full
    assert rel_err(cache.state_pn(), torch.stack(ref_state)) <= TOL_STATE
    assert cache.len[:, 0].tolist() == [L % chunk for L in w.seqlens]
    assert bool((cache.len == cache.len[:, :1]).all())


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_strict_decode_matches_oracle(ssd, cuda_dev, dtype):
    # Prefill 100 tokens, then 200 decode steps (crossing chunk boundaries at 128 and 256).
    K, L1 = 200, 100
    w = _w([L1 + K] * 3, dtype=dtype, seed=62)
    inp = W.make_all(w, device=cuda_dev)
    cu = inp["cu_seqlens"].tolist()
    cache = _cache(ssd, w, cuda_dev, inp["init_state"])
    rows = torch.cat([_seq_rows(cu, s, 0, L1, cuda_dev) for s in range(w.nseq)])
    _prefill(ssd, w, inp, rows, [L1] * w.nseq, cache)
    ys = []
    for k in range(K):
        t = _rows(inp, torch.tensor([cu[s] + L1 + k for s in range(w.nseq)], device=cuda_dev))
        ys.append(ssd.strict_state_update(cache, t["x"], t["dt_raw"], inp["dt_bias"], inp["A"], t["B"], t["C"],
                                          inp["D"]))
    ssd.device_status()
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    y_ref, fin_ref = O.ssd_scan(cpu["x"], cpu["dt_raw"], cpu["dt_bias"], cpu["A"], cpu["B"], cpu["C"], cpu["D"],
                                init_state=cpu["init_state"], cu_seqlens=cpu["cu_seqlens"])
    got = torch.stack(ys, 1)                                   # [nseq, K, H, P]
    ref = torch.stack([y_ref[cu[s] + L1:cu[s + 1]] for s in range(w.nseq)])
    assert rel_err(got, ref) <= TOL_Y[dtype]
    # 300 tokens: two full chunks folded, 44 tokens open.
    assert cache.len[:, 0].tolist() == [(L1 + K) % 128] * w.nseq
    _, _, snaps = O.ssd_scan(cpu["x"], cpu["dt_raw"], cpu["dt_bias"], cpu["A"], cpu["B"], cpu["C"], cpu["D"],
                             init_state=cpu["init_state"], cu_seqlens=cpu["cu_seqlens"], snapshot_tokens=128)
    assert rel_err(cache.state_pn(), snaps.view(w.nseq, 2, *snaps.shape[1:])[:, 1]) <= TOL_STATE


# --------------------------------------------------------------------------------------
# Bitwise invariance.
@pytest.mark.parametrize("dtype,chunk", [(torch.bfloat16, 128), (torch.float32, 128), (torch.bfloat16, 64)])
def test_prefill_then_decode_is_bitwise_one_shot(ssd, cuda_dev, dtype, chunk):
    """Split each sequence at a different token (0, 1, 77, chunk, chunk+5, 2 chunks, 300)
    into a strict prefill and 150 chunk-emulating decode steps."""
    K = 150
    L1 = [0, 1, 77, chunk, chunk + 5, 2 * chunk, 300]
    w = _w([a + K for a in L1], dtype=dtype, chunk=chunk, seed=63, dt_range=(1e-4, 0.5))
    inp = W.make_all(w, device=cuda_dev)
    cu = inp["cu_seqlens"].tolist()
    full = _cache(ssd, w, cuda_dev, inp["init_state"])
    y_full, fin_full = ssd.strict_scan_fwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"],
                                           inp["D"], full, resume=True, cu_seqlens=inp["cu_seqlens"])
    split = _cache(ssd, w, cuda_dev, inp["init_state"])
    rows = torch.cat([_seq_rows(cu, s, 0, L1[s], cuda_dev) for s in range(w.nseq)])
    y_pre, _ = _prefill(ssd, w, inp, rows, L1, split)
    ys = []
    for k in range(K):
        t = _rows(inp, torch.tensor([cu[s] + L1[s] + k for s in range(w.nseq)], device=cuda_dev))
        ys.append(ssd.strict_state_update(split, t["x"], t["dt_raw"], inp["dt_bias"], inp["A"], t["B"], t["C"],
                                          inp["D"]))
    ssd.device_status()
    assert_same_bits(y_pre, y_full[rows], "prefill part")
    dec_rows = torch.tensor([[cu[s] + L1[s] + k for s in range(w.nseq)] for k in range(K)], device=cuda_dev)
    assert_same_bits(torch.stack(ys), y_full[dec_rows], "decode part")
    _assert_cache_equal(split, full, w.ngroups, w.nheads)


@pytest.mark.parametrize("H,G,P,N", [(8, 1, 128, 32), (16, 1, 64, 64), (4, 1, 16, 16)])
def test_decode_geometries_bitwise_and_against_oracle(ssd, cuda_dev, H, G, P, N):
    """The decode step streams each group's state rows (heads per group x P of them) through
    shared memory in batches of 512 rows and slices of 16 columns: 1024 rows in two batches
    (P = 128 or 16 heads per group), a single slice (N = 16), two slices (N = 32). Split each
    sequence into a strict prefill and 80 decode steps (crossing chunk ends at 64 tokens);
    the decode must give the one-shot prefill's bits and match the oracle."""
    K, chunk = 80, 64
    L1 = [0, 5, 64, 70]
    w = _w([a + K for a in L1], H=H, G=G, P=P, N=N, chunk=chunk, seed=66)
    inp = W.make_all(w, device=cuda_dev)
    cu = inp["cu_seqlens"].tolist()
    full = _cache(ssd, w, cuda_dev, inp["init_state"])
    y_full, _ = ssd.strict_scan_fwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                                    full, resume=True, cu_seqlens=inp["cu_seqlens"])
    split = _cache(ssd, w, cuda_dev, inp["init_state"])
    rows = torch.cat([_seq_rows(cu, s, 0, L1[s], cuda_dev) for s in range(w.nseq)])
    y_pre, _ = _prefill(ssd, w, inp, rows, L1, split)
    ys = []
    for k in range(K):
        t = _rows(inp, torch.tensor([cu[s] + L1[s] + k for s in range(w.nseq)], device=cuda_dev))
        ys.append(ssd.strict_state_update(split, t["x"], t["dt_raw"], inp["dt_bias"], inp["A"], t["B"], t["C"],
                                          inp["D"]))
    ssd.device_status()
    dec_rows = torch.tensor([[cu[s] + L1[s] + k for s in range(w.nseq)] for k in range(K)], device=cuda_dev)
    assert_same_bits(torch.stack(ys), y_full[dec_rows], "decode part")
    _assert_cache_equal(split, full, w.ngroups, w.nheads)
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    y_ref, _ = O.ssd_scan(cpu["x"], cpu["dt_raw"], cpu["dt_bias"], cpu["A"], cpu["B"], cpu["C"], cpu["D"],
                          init_state=cpu["init_state"], cu_seqlens=cpu["cu_seqlens"])
    assert rel_err(torch.stack(ys), y_ref[dec_rows.cpu()]) <= TOL_Y[w.dtype]


def test_prefill_split_at_chunk_boundaries_is_bitwise(ssd, cuda_dev):
    chunk = 128
    L1, L2 = [256, 128, 0, 384], [300, 5, 129, 0]
    w = _w([a + b for a, b in zip(L1, L2)], seed=64)
    inp = W.make_all(w, device=cuda_dev)
    cu = inp["cu_seqlens"].tolist()
    full = _cache(ssd, w, cuda_dev, inp["init_state"])
    y_full, fin_full = ssd.strict_scan_fwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"],
                                           inp["D"], full, resume=True, cu_seqlens=inp["cu_seqlens"])
    split = _cache(ssd, w, cuda_dev, inp["init_state"])
    r1 = torch.cat([_seq_rows(cu, s, 0, L1[s], cuda_dev) for s in range(w.nseq)])
    r2 = torch.cat([_seq_rows(cu, s, L1[s], L1[s] + L2[s], cuda_dev) for s in range(w.nseq)])
    y1, _ = _prefill(ssd, w, inp, r1, L1, split)
    y2, fin2 = _prefill(ssd, w, inp, r2, L2, split)
    ssd.device_status()
    assert_same_bits(y1, y_full[r1], "first prefill")
    assert_same_bits(y2, y_full[r2], "second prefill")
    assert_same_bits(fin2, fin_full, "final state")
    _assert_cache_equal(split, full, w.ngroups, w.nheads)
    assert chunk == w.chunk


def test_prefill_decode_prefill_is_bitwise(ssd, cuda_dev):
    """Prefill 100 / 228 tokens, decode 28 steps (both sequences reach a chunk boundary),
    then resume with a strict prefill of 50 / 300 more."""
    L1, K, L3 = [100, 228], 28, [50, 300]
    w = _w([a + K + b for a, b in zip(L1, L3)], seed=65)
    inp = W.make_all(w, device=cuda_dev)
    cu = inp["cu_seqlens"].tolist()
    full = _cache(ssd, w, cuda_dev, inp["init_state"])
    y_full, _ = ssd.strict_scan_fwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"],
                                    inp["D"], full, resume=True, cu_seqlens=inp["cu_seqlens"])
    split = _cache(ssd, w, cuda_dev, inp["init_state"])
    r1 = torch.cat([_seq_rows(cu, s, 0, L1[s], cuda_dev) for s in range(2)])
    y1, _ = _prefill(ssd, w, inp, r1, L1, split)
    ys = []
    for k in range(K):
        t = _rows(inp, torch.tensor([cu[s] + L1[s] + k for s in range(2)], device=cuda_dev))
        ys.append(ssd.strict_state_update(split, t["x"], t["dt_raw"], inp["dt_bias"], inp["A"], t["B"], t["C"],
                                          inp["D"]))
    assert split.len.sum().item() == 0
    r3 = torch.cat([_seq_rows(cu, s, L1[s] + K, L1[s] + K + L3[s], cuda_dev) for s in range(2)])
    y3, _ = _prefill(ssd, w, inp, r3, L3, split)
    ssd.device_status()
    assert_same_bits(y1, y_full[r1], "prefill 1")
    dec_rows = torch.tensor([[cu[s] + L1[s] + k for s in range(2)] for k in range(K)], device=cuda_dev)
    assert_same_bits(torch.stack(ys), y_full[dec_rows], "decode")
    assert_same_bits(y3, y_full[r3], "prefill 2")
    _assert_cache_equal(split, full, w.ngroups, w.nheads)


def test_batch_position_and_layout_are_bitwise(ssd, cuda_dev):
    w = _w([50, 333, 7, 333], seed=66)
    inp = W.make_all(w, device=cuda_dev)
    cu = inp["cu_seqlens"].tolist()
    c4 = _cache(ssd, w, cuda_dev, inp["init_state"])
    y4, f4 = ssd.strict_scan_fwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                                 c4, resume=True, cu_seqlens=inp["cu_seqlens"])
    # Sequence 1 alone.
    w1 = _w([333], seed=66)
    c1 = _cache(ssd, w1, cuda_dev, inp["init_state"][1:2])
    r = _seq_rows(cu, 1, 0, 333, cuda_dev)
    y1, f1 = _prefill(ssd, w1, inp, r, [333], c1)
    # Sequences 1 and 3 as a dense batch of two (sequence 3 gets sequence 1's tokens).
    w2 = _w([333, 333], seed=66)
    c2 = _cache(ssd, w2, cuda_dev, inp["init_state"][[1, 1]])
    t = _rows(inp, torch.cat([r, r]))
    rs = lambda v: v.view(2, 333, *v.shape[1:])
    y2, f2 = ssd.strict_scan_fwd(rs(t["x"]), rs(t["dt_raw"]), inp["dt_bias"], inp["A"], rs(t["B"]), rs(t["C"]),
                                 inp["D"], c2, resume=True)
    ssd.device_status()
    assert_same_bits(y1, y4[r], "alone vs in a batch of 4")
    assert_same_bits(f1[0], f4[1], "final state")
    assert_same_bits(y2[0], y4[r], "dense batch position 0")
    assert_same_bits(y2[1], y4[r], "dense batch position 1")
    assert_same_bits(c2.state[1], c4.state[1], "cache state")


def test_resume_with_open_chunk_fails_closed(ssd, cuda_dev):
    w = _w([130, 256], seed=67)
    inp = W.make_all(w, device=cuda_dev)
    cache = _cache(ssd, w, cuda_dev)
    ssd.strict_scan_fwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"], cache,
                        cu_seqlens=inp["cu_seqlens"])
    ssd.device_status()
    assert cache.len[:, 0].tolist() == [2, 0]
    ssd.strict_scan_fwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"], cache,
                        resume=True, cu_seqlens=inp["cu_seqlens"])
    with pytest.raises(ssd.SSDError, match="UNSUPPORTED"):
        ssd.device_status()
    ssd.device_status()                      # the error word was read and cleared


def test_strict_is_within_tolerance_of_fast_path(ssd, cuda_dev):
    """Strict and default prefill agree to rounding (not bitwise)."""
    w = _w([700, 1500], seed=68)
    inp = W.make_all(w, device=cuda_dev)
    cache = _cache(ssd, w, cuda_dev, inp["init_state"])
    ys, fs = ssd.strict_scan_fwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                                 cache, resume=True, cu_seqlens=inp["cu_seqlens"])
    yf, ff = ssd.scan_fwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                          init_state=inp["init_state"], cu_seqlens=inp["cu_seqlens"])
    ssd.device_status()
    assert rel_err(ys, yf) <= 1e-2
    assert rel_err(fs, ff) <= 1e-3


# --------------------------------------------------------------------------------------
# Full size: the long-context workload (1 x 65536 tokens, 64 heads, chunk 256) in strict
# mode against the oracle on one head of every group; its cache ends on a chunk boundary.
GROUP_HEADS = [0, 9, 18, 27, 36, 45, 54, 63]


@pytest.mark.slow
def test_strict_long_context_full_size(ssd, cuda_dev):
    w = W.config(2)
    inp = W.make_all(w, device=cuda_dev)
    L = w.seqlens[0]
    r4 = lambda t: t.view(w.nseq, L, *t.shape[1:])
    cache = _cache(ssd, w, cuda_dev, inp["init_state"])
    y, fin = ssd.strict_scan_fwd(r4(inp["x"]), r4(inp["dt_raw"]), inp["dt_bias"], inp["A"], r4(inp["B"]),
                                 r4(inp["C"]), inp["D"], cache, resume=inp["init_state"] is not None)
    ssd.device_status()
    pairs = [(0, h) for h in GROUP_HEADS]
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    blocks, fin_ref = O.ssd_scan(cpu["x"], cpu["dt_raw"], cpu["dt_bias"], cpu["A"], cpu["B"], cpu["C"], cpu["D"],
                                 init_state=cpu["init_state"], batch=1, pairs=pairs)
    yc = y.view(L, w.nheads, w.headdim)
    got = torch.stack([yc[:, h, :] for _, h in pairs])
    ref = torch.stack([torch.from_numpy(b) for b in blocks])
    assert rel_err(got, ref) <= TOL_Y[w.dtype]
    assert rel_err(torch.stack([fin[0, h] for _, h in pairs]), fin_ref) <= TOL_STATE
    assert int(cache.len.max()) == 0                      # 65536 is a multiple of the chunk
    assert_same_bits(cache.state, fin, "cache state = final state on a chunk boundary")


def test_strict_decode_full_batch_bitwise(ssd, cuda_dev):
    """The chunk-emulating decode at the shape the benchmark times it: 256 sequences, 64
    heads (8 groups), headdim 64, dstate 128, chunk 128 (2048 blocks). Each sequence is
    split after 100 to 227 tokens (all different open-chunk lengths) into a strict prefill
    and 60 decode steps, so that most sequences cross a chunk end and are folded mid-batch.
    The decode must give the one-shot prefill's bits; three sequences also go through the
    oracle."""
    w0 = W.config(4)
    K, nseq = 60, 256
    L1 = [100 + (s * 37) % 128 for s in range(nseq)]
    w = W.Workload("strict_decode_full", nheads=w0.nheads, headdim=w0.headdim, ngroups=w0.ngroups,
                   dstate=w0.dstate, chunk=w0.chunk, dtype=w0.dtype, seqlens=[a + K for a in L1], varlen=True,
                   init="normal", seed=67)
    inp = W.make_all(w, device=cuda_dev)
    cu = inp["cu_seqlens"].tolist()
    full = _cache(ssd, w, cuda_dev, inp["init_state"])
    y_full, _ = ssd.strict_scan_fwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                                    full, resume=True, cu_seqlens=inp["cu_seqlens"])
    split = _cache(ssd, w, cuda_dev, inp["init_state"])
    rows = torch.cat([_seq_rows(cu, s, 0, L1[s], cuda_dev) for s in range(nseq)])
    _prefill(ssd, w, inp, rows, L1, split)
    ys = []
    for k in range(K):
        t = _rows(inp, torch.tensor([cu[s] + L1[s] + k for s in range(nseq)], device=cuda_dev))
        ys.append(ssd.strict_state_update(split, t["x"], t["dt_raw"], inp["dt_bias"], inp["A"], t["B"], t["C"],
                                          inp["D"]))
    ssd.device_status()
    dec_rows = torch.tensor([[cu[s] + L1[s] + k for s in range(nseq)] for k in range(K)], device=cuda_dev)
    got = torch.stack(ys)
    assert_same_bits(got, y_full[dec_rows], "decode part")
    _assert_cache_equal(split, full, w.ngroups, w.nheads)
    for s in (0, 97, 255):
        sub = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
        a, b = cu[s], cu[s + 1]
        y_ref, _ = O.ssd_scan(sub["x"][a:b], sub["dt_raw"][a:b], sub["dt_bias"], sub["A"], sub["B"][a:b],
                              sub["C"][a:b], sub["D"], init_state=sub["init_state"][s:s + 1],
                              cu_seqlens=torch.tensor([0, b - a], dtype=torch.int32))
        assert rel_err(got[:, s].cpu(), y_ref[L1[s]:L1[s] + K]) <= TOL_Y[w.dtype]

