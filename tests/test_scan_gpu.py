"""GPU parity of ssd_scan_fwd (through the C ABI) against the FP64 oracle.

Small cases compare every output element; they span several chunks, ragged last
chunks, every supported chunk size, the smallest and largest head/state dims,
dense and packed layouts, zero and random initial states. The full-size cases
(the five named workloads) compare sampled (sequence, head) pairs that cover
every B/C group, over all tokens of those pairs.

Tolerances (SSD contract): max|y - y_ref| / max|y_ref| <= 1e-2 for bf16 inputs,
<= 1e-4 for float32 inputs; final state <= 1e-3.
"""
import pytest
import torch

from mamba_ssd_state_02_b200 import workloads as W
from parity_util import TOL_STATE, TOL_Y, compare_pairs, oracle_scan, rel_err, run_gpu_scan

pytestmark = pytest.mark.gpu


def _wl(name, H, P, G, N, Q, dtype, seqlens, varlen, init="zero", seed=7, dt_range=(1e-3, 0.1)):
    return W.Workload(name, nheads=H, headdim=P, ngroups=G, dstate=N, chunk=Q, dtype=dtype,
                      seqlens=seqlens, varlen=varlen, init=init, seed=seed, dt_range=dt_range)


SMALL = [
    _wl("bf16_dense_ragged", 8, 64, 2, 128, 128, torch.bfloat16, [300, 300], False, "normal"),
    _wl("f32_P128_N128_Q256", 4, 128, 1, 128, 256, torch.float32, [520], False),
    _wl("f32_P16_N16_varlen", 4, 16, 4, 16, 64, torch.float32, [1, 63, 64, 65, 200], True, "normal"),
    _wl("bf16_varlen_empty_seq", 8, 32, 2, 64, 64, torch.bfloat16, [0, 129, 7], True, "normal"),
    _wl("bf16_P128_N32_G8", 16, 128, 8, 32, 128, torch.bfloat16, [257], False, "normal"),
    _wl("bf16_P16_N128_wide_dt", 8, 16, 1, 128, 256, torch.bfloat16, [700], False, "zero", 11, (1e-4, 0.5)),
    _wl("f32_L1", 4, 32, 2, 32, 64, torch.float32, [1, 1, 1], False, "normal"),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_scan_matches_oracle_small(ssd, cuda_dev, w):
    inp = W.make_all(w)
    y, fin = run_gpu_scan(ssd, w, inp, cuda_dev)
    ssd.device_status()
    y_ref, fin_ref = oracle_scan(w, inp)
    assert rel_err(y, y_ref) <= TOL_Y[w.dtype]
    assert rel_err(fin, fin_ref) <= TOL_STATE


@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_config0_tiny_fp32_every_chunk(ssd, cuda_dev, chunk):
    w = W.config(0)
    inp = W.make_all(w)
    y, fin = run_gpu_scan(ssd, w, inp, cuda_dev, chunk=chunk)
    y_ref, fin_ref = oracle_scan(w, inp)
    assert rel_err(y, y_ref) <= 1e-4
    assert rel_err(fin, fin_ref) <= TOL_STATE


def _sampled(ssd, cuda_dev, k, heads, per_seq=None):
    w = W.config(k)
    inp = W.make_all(w, device=cuda_dev)
    y, fin = run_gpu_scan(ssd, w, inp, cuda_dev)
    ssd.device_status()
    if per_seq is None:
        pairs = [(s, h) for s in range(w.nseq) for h in heads]
    else:
        pairs = [(s, heads[(s * per_seq + j) % len(heads)]) for s in range(w.nseq) for j in range(per_seq)]
    y_blocks, fin_ref = oracle_scan(w, inp, pairs=pairs)
    return compare_pairs(w, y, fin, y_blocks, fin_ref, pairs)


GROUP_HEADS = [0, 9, 18, 27, 36, 45, 54, 63]   # one head in each of the 8 groups


@pytest.mark.slow
def test_config1_batched_prefill(ssd, cuda_dev):
    ey, ef = _sampled(ssd, cuda_dev, 1, GROUP_HEADS, per_seq=4)
    assert ey <= 1e-2 and ef <= TOL_STATE, (ey, ef)


@pytest.mark.slow
def test_config2_long_context(ssd, cuda_dev):
    ey, ef = _sampled(ssd, cuda_dev, 2, GROUP_HEADS)
    assert ey <= 1e-2 and ef <= TOL_STATE, (ey, ef)


@pytest.mark.slow
def test_config3_packed_varlen(ssd, cuda_dev):
    ey, ef = _sampled(ssd, cuda_dev, 3, GROUP_HEADS, per_seq=2)
    assert ey <= 1e-2 and ef <= TOL_STATE, (ey, ef)
