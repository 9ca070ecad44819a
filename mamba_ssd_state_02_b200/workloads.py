"""Seeded synthetic inputs for the Mamba-2 SSD scan and decode step.

This module draws input tensors only. It holds none of the SSD arithmetic: no
softplus, no decay, no contraction. Both the CUDA path (through the tests and the
benchmark) and the FP64 oracle receive tensors made here, so it imports nothing
from either of them.

Generator (counter-based, so any element can be drawn independently and the same
stream is reproduced on the CPU or on a CUDA device):

* ``u64(seed, stream, i) = splitmix64(seed XOR (stream << 56) XOR i)``, where
  splitmix64 is Vigna's 64-bit finaliser (add 0x9E3779B97F4A7C15, then two
  xor-shift-multiply rounds and a final xor-shift).
* ``uniform = (u64 >> 11) * 2**-53`` in [0, 1).
* ``normal_i = sqrt(-2 ln(1 - U_{2i})) * cos(2 pi U_{2i+1})`` (Box-Muller, cosine
  branch only, two uniforms per normal).
* Values are drawn in float64 and rounded to float32 (round to nearest even); bf16
  inputs are then rounded float32 -> bf16 (round to nearest even).

Value recipe, per the Nemotron-H Mamba-2 block on the RL-Kernel issue page
(Figure 2: ``softplus(dt + dt_bias)``, ``A = -exp(A_log)``, B/C groups) and the
SSD layer's D skip on the JAX Nemotron 3 Nano page ("Key Components"):

* x ~ N(0, 1); B, C ~ N(0, 1) / sqrt(N); dt_raw ~ N(0, 1).
* dt_bias: per head, dt0 = exp(U(ln lo, ln hi)) and dt_bias = inverse softplus of
  dt0, so softplus(dt_raw + dt_bias) spreads around dt0. (lo, hi) = (1e-3, 0.1),
  widened to (1e-4, 0.5) for the long-context workload.
* A = -exp(U(0, ln 16)), so A lies in [-16, -1]; D ~ U(0, 1).
* Initial states: zero, or N(0, 0.1) (standard deviation 0.1).
* Packed variable-length workload: lengths uniform integers in [512, 8192].
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

_GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB


def _as_i64(v: int) -> int:
    v &= (1 << 64) - 1
    return v - (1 << 64) if v >= (1 << 63) else v


def _lsr(z: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of an int64 tensor holding uint64 bit patterns."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def _splitmix64(z: torch.Tensor) -> torch.Tensor:
    z = z + _as_i64(_GOLDEN)
    z = (z ^ _lsr(z, 30)) * _as_i64(_M1)
    z = (z ^ _lsr(z, 27)) * _as_i64(_M2)
    return z ^ _lsr(z, 31)


# Stream identifiers: one per tensor role, so tensors never share random numbers.
STREAM = {
    "x": 1, "dt_raw": 2, "dt0": 3, "A": 4, "B": 5, "C": 6, "D": 7, "init_state": 8,
    "lengths": 15,
    "xbc": 20, "conv_w": 21, "conv_b": 22, "conv_state": 23,
}

_CHUNK = 1 << 22


def _key(seed: int, stream: int) -> int:
    return _as_i64((seed & ((1 << 56) - 1)) ^ (stream << 56))


def uniform_at(seed: int, stream: int, ctr: torch.Tensor) -> torch.Tensor:
    """Uniform float64 draws in [0, 1) at the given int64 counters."""
    u = _splitmix64(ctr ^ _key(seed, stream))
    return _lsr(u, 11).to(torch.float64) * (2.0 ** -53)


def normal_at(seed: int, stream: int, ctr: torch.Tensor) -> torch.Tensor:
    """Standard normal float64 draws at the given counters (Box-Muller on 2c, 2c+1)."""
    u1 = uniform_at(seed, stream, 2 * ctr)
    u2 = uniform_at(seed, stream, 2 * ctr + 1)
    return torch.sqrt(-2.0 * torch.log1p(-u1)) * torch.cos((2.0 * math.pi) * u2)


def _draw(fn, seed, stream, n, offset, device):
    out = torch.empty(n, dtype=torch.float64, device=device)
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        ctr = torch.arange(offset + lo, offset + hi, dtype=torch.int64, device=device)
        out[lo:hi] = fn(seed, stream, ctr)
    return out


def uniform(seed: int, stream: int, n: int, offset: int = 0, device="cpu") -> torch.Tensor:
    """Uniform float64 draws for counters offset .. offset+n-1."""
    return _draw(uniform_at, seed, stream, n, offset, device)


def normal(seed: int, stream: int, n: int, offset: int = 0, device="cpu") -> torch.Tensor:
    """Standard normal float64 draws for counters offset .. offset+n-1."""
    return _draw(normal_at, seed, stream, n, offset, device)


def normal_rows(seed: int, stream: int, rows: torch.Tensor, width: int) -> torch.Tensor:
    """Normal draws for the given packed rows of a [T, width] tensor -> [len(rows), width]."""
    out = torch.empty(rows.numel(), width, dtype=torch.float64, device=rows.device)
    step = max(1, _CHUNK // width)
    col = torch.arange(width, dtype=torch.int64, device=rows.device)
    for lo in range(0, rows.numel(), step):
        r = rows[lo:lo + step].to(torch.int64)
        out[lo:lo + r.numel()] = normal_at(seed, stream, r[:, None] * width + col[None, :])
    return out


def to_input_dtype(v: torch.Tensor, dtype: torch.dtype) -> torch.Tensor:
    """float64 -> float32 (RNE) -> dtype (RNE when dtype is bf16)."""
    v32 = v.to(torch.float32)
    return v32 if dtype == torch.float32 else v32.to(dtype)


@dataclass
class Workload:
    """One synthetic SSD problem: dims, dtype, chunk and the value recipe."""
    name: str
    nheads: int
    headdim: int
    ngroups: int
    dstate: int
    chunk: int
    dtype: torch.dtype
    seqlens: list            # one entry per sequence
    varlen: bool             # packed with cu_seqlens (True) or dense batch x L (False)
    dt_range: tuple = (1e-3, 0.1)
    init: str = "zero"       # "zero" or "normal" (std 0.1)
    seed: int = 1000
    decode_steps: int = 0    # decode workload: steps after the prefix
    extra: dict = field(default_factory=dict)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def nseq(self) -> int:
        return len(self.seqlens)


def varlen_lengths(seed: int, nseq: int, lo: int = 512, hi: int = 8192) -> list:
    u = uniform(seed, STREAM["lengths"], nseq)
    return [lo + int(math.floor(float(v) * (hi - lo + 1))) for v in u]


def config(k: int, seed: int | None = None) -> Workload:
    """The five named workloads (dims from the Nemotron-H SSD shapes)."""
    s = 1000 + k if seed is None else seed
    common = dict(nheads=64, headdim=64, ngroups=8, dstate=128, dtype=torch.bfloat16, seed=s)
    if k == 0:
        return Workload("tiny_fp32_L256_H4_P16_N16_Q64", nheads=4, headdim=16, ngroups=1,
                        dstate=16, chunk=64, dtype=torch.float32, seqlens=[256],
                        varlen=False, seed=s)
    if k == 1:
        return Workload("prefill_bf16_B4_L4096_H64_P64_G8_N128_Q128", chunk=128,
                        seqlens=[4096] * 4, varlen=False, init="normal", **common)
    if k == 2:
        return Workload("prefill_bf16_B1_L65536_H64_P64_G8_N128_Q256", chunk=256,
                        seqlens=[65536], varlen=False, dt_range=(1e-4, 0.5), **common)
    if k == 3:
        return Workload("varlen_bf16_16seq_U512_8192_H64_P64_G8_N128_Q128", chunk=128,
                        seqlens=varlen_lengths(s, 16), varlen=True, init="normal", **common)
    if k == 4:
        return Workload("decode_bf16_256seq_prefix2048_steps1024_H64_P64_G8_N128", chunk=128,
                        seqlens=[2048] * 256, varlen=False, decode_steps=1024, **common)
    raise ValueError(f"no workload {k}")


def make_params(w: Workload, device="cpu") -> dict:
    """Per-head parameters dt_bias, A, D (float32, [H])."""
    H = w.nheads
    lo, hi = w.dt_range
    u = uniform(w.seed, STREAM["dt0"], H, device=device)
    dt0 = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))
    dt_bias = dt0 + torch.log(-torch.expm1(-dt0))  # inverse softplus of dt0
    A = -torch.exp(uniform(w.seed, STREAM["A"], H, device=device) * math.log(16.0))
    D = uniform(w.seed, STREAM["D"], H, device=device)
    f32 = torch.float32
    return {"dt_bias": dt_bias.to(f32), "A": A.to(f32), "D": D.to(f32)}


def make_tokens(w: Workload, t0: int, t1: int, device="cpu", rows=None) -> dict:
    """Per-token tensors for packed token rows t0..t1-1 of the workload.

    Token row t of the packed [T, ...] layout always draws the same counters, so
    any row set can be regenerated on its own (pass ``rows``, an int64 tensor of
    row indices, to draw exactly those rows; t0/t1 are then ignored).
    """
    H, P, G, N = w.nheads, w.headdim, w.ngroups, w.dstate
    if rows is None:
        rows = torch.arange(t0, t1, dtype=torch.int64, device=device)
    n = rows.numel()
    s = w.seed
    x = normal_rows(s, STREAM["x"], rows, H * P).view(n, H, P)
    dt_raw = normal_rows(s, STREAM["dt_raw"], rows, H).view(n, H)
    sc = 1.0 / math.sqrt(N)
    B = (normal_rows(s, STREAM["B"], rows, G * N) * sc).view(n, G, N)
    C = (normal_rows(s, STREAM["C"], rows, G * N) * sc).view(n, G, N)
    return {
        "x": to_input_dtype(x, w.dtype),
        "dt_raw": dt_raw.to(torch.float32),
        "B": to_input_dtype(B, w.dtype),
        "C": to_input_dtype(C, w.dtype),
    }


def make_init_state(w: Workload, device="cpu"):
    """[nseq, H, P, N] float32 initial states, or None for zero initial states."""
    if w.init == "zero":
        return None
    n = w.nseq * w.nheads * w.headdim * w.dstate
    v = normal(w.seed, STREAM["init_state"], n, 0, device) * 0.1
    return v.to(torch.float32).view(w.nseq, w.nheads, w.headdim, w.dstate)


def cu_seqlens(w: Workload, device="cpu") -> torch.Tensor:
    c = [0]
    for L in w.seqlens:
        c.append(c[-1] + int(L))
    return torch.tensor(c, dtype=torch.int32, device=device)


def make_all(w: Workload, device="cpu") -> dict:
    """Every input of one scan call: token tensors, parameters and initial state."""
    d = make_tokens(w, 0, w.total_tokens, device)
    d.update(make_params(w, device))
    d["init_state"] = make_init_state(w, device)
    d["cu_seqlens"] = cu_seqlens(w, device) if w.varlen else None
    return d


def conv_channels(w: Workload) -> int:
    """Channels of the conv1d prologue's input: x, B and C side by side."""
    return w.nheads * w.headdim + 2 * w.ngroups * w.dstate


def make_conv_inputs(w: Workload, width: int = 4, init: bool = True, device="cpu") -> dict:
    """Inputs of the conv1d prologue for workload w: xbc [T, D] ~ N(0,1) (w.dtype),
    weight [D, width] ~ U(-1, 1)/sqrt(width) and bias [D] ~ U(-0.5, 0.5) (float32), and a
    conv state [nseq, D, width-1] ~ N(0,1) (w.dtype) or None."""
    Dc = conv_channels(w)
    T = w.total_tokens
    xbc = to_input_dtype(normal(w.seed, STREAM["xbc"], T * Dc, device=device), w.dtype).view(T, Dc)
    weight = ((uniform(w.seed, STREAM["conv_w"], Dc * width, device=device) * 2 - 1) / math.sqrt(width))
    bias = uniform(w.seed, STREAM["conv_b"], Dc, device=device) - 0.5
    st = None
    if init:
        st = to_input_dtype(normal(w.seed, STREAM["conv_state"], w.nseq * Dc * (width - 1), device=device),
                            w.dtype).view(w.nseq, Dc, width - 1)
    return {"xbc": xbc, "weight": weight.to(torch.float32).view(Dc, width), "bias": bias.to(torch.float32),
            "conv_state": st, "cu_seqlens": cu_seqlens(w, device) if w.varlen else None}
