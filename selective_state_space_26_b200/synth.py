"""Seeded synthetic inputs for the S6 scan and the decode update.

This module only draws numbers; it contains none of the scan's arithmetic.  It
is the one piece shared by the tests' oracle side and the CUDA side: both read
the very same tensors it returns (the oracle gets them copied to the host).

Recipe (the S6 layer of the Jamba pages: d_state = 16, expansion 2, so
d_model 4096 -> d_inner 8192):
  x, z, B, C, raw delta  ~ N(0, 1), drawn in fp32 and rounded (RNE) to the I/O
                           dtype (bf16, or fp32 for the tiny case);
  delta_bias[d]          = softplus^-1(dt0[d]) with dt0[d] log-uniform in
                           [1e-3, 1e-1], so Delta = softplus(delta + delta_bias)
                           is centred on dt0 (fp32 parameter);
  A[d, n]                = -(n + 1) (fp32), or -exp(N(0,1)) for the
                           "random" kind the tests use so no kernel can lean on
                           the integer structure;
  D[d]                   = 1 (fp32);
  h0                     = 0 for prefill; for decode the cached state is
                           N(0, 0.1^2) (std 0.1), fp32.
Every tensor is drawn from its own torch.Generator whose seed is a SplitMix64
hash of (workload seed, tensor id, sequence index, chunk/step index), so a
sequence or a decode step can be regenerated on its own, and the draws do not
depend on how many sequences are generated together.  Values depend on the
device they are drawn on (torch's CPU and CUDA generators differ); tests always
copy the device tensors to the host for the oracle.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

_MASK = (1 << 64) - 1
# tensor ids of the counter
T_X, T_DT, T_Z, T_B, T_C, T_H0, T_DT0, T_A, T_DTLOW, T_WDT, T_WX, T_NORMW = range(12)
_ROWS_PER_DRAW = 8192  # rows of [seqlen, width] drawn per generator call


def _splitmix64(v: int) -> int:
    v = (v + 0x9E3779B97F4A7C15) & _MASK
    v = ((v ^ (v >> 30)) * 0xBF58476D1CE4E5B9) & _MASK
    v = ((v ^ (v >> 27)) * 0x94D049BB133111EB) & _MASK
    return v ^ (v >> 31)


def counter_seed(seed: int, tensor: int, seq: int, chunk: int) -> int:
    """63-bit generator seed for one (workload seed, tensor, sequence, chunk)."""
    v = _splitmix64(seed & _MASK)
    for part in (tensor, seq, chunk):
        v = _splitmix64(v ^ (part & _MASK))
    return v & ((1 << 63) - 1)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(shape, seed: int, tensor: int, seq: int, chunk: int, device,
           std: float = 1.0) -> torch.Tensor:
    """fp32 N(0, std^2) tensor from one counter-derived generator."""
    g = _gen(device, counter_seed(seed, tensor, seq, chunk))
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def _fill_sequence(dst: torch.Tensor, seed: int, tensor: int, seq: int):
    """Fill dst [seqlen, width] (any dtype) with N(0,1), drawn in row chunks."""
    seqlen = dst.shape[0]
    for c, r0 in enumerate(range(0, seqlen, _ROWS_PER_DRAW)):
        r1 = min(seqlen, r0 + _ROWS_PER_DRAW)
        dst[r0:r1].copy_(normal((r1 - r0, dst.shape[1]), seed, tensor, seq, c, dst.device))


def dt_bias_for(d_inner: int, seed: int, dt_min: float = 1e-3, dt_max: float = 1e-1):
    """Per-channel bias so that softplus(0 + bias) = dt0, dt0 log-uniform."""
    rng = np.random.Generator(np.random.PCG64(counter_seed(seed, T_DT0, 0, 0)))
    u = rng.random(d_inner)
    dt0 = np.exp(np.log(dt_min) + u * (np.log(dt_max) - np.log(dt_min)))
    bias = dt0 + np.log(-np.expm1(-dt0))  # inverse of log(1 + e^v)
    return torch.from_numpy(bias.astype(np.float32))


def make_A(d_inner: int, d_state: int, kind: str = "mamba", seed: int = 0) -> torch.Tensor:
    if kind == "mamba":
        row = -torch.arange(1, d_state + 1, dtype=torch.float32)
        return row.repeat(d_inner, 1).contiguous()
    if kind == "random":
        g = _gen("cpu", counter_seed(seed, T_A, 0, 0))
        return (-torch.exp(torch.randn(d_inner, d_state, generator=g))).contiguous()
    raise ValueError(f"unknown A kind {kind!r}")


@dataclasses.dataclass
class ScanInputs:
    x: torch.Tensor
    delta: torch.Tensor
    z: torch.Tensor
    B: torch.Tensor
    C: torch.Tensor
    A: torch.Tensor
    D: torch.Tensor
    delta_bias: torch.Tensor
    h0: torch.Tensor | None
    delta_softplus: bool = True

    @property
    def shape(self):
        b, l, d = self.x.shape
        return b, l, d, self.A.shape[1]


def scan_inputs(batch: int, seqlen: int, d_inner: int, d_state: int,
                dtype=torch.bfloat16, seed: int = 0, device="cpu",
                h0_std: float = 0.0, A_kind: str = "mamba",
                seq_offset: int = 0) -> ScanInputs:
    """Prefill inputs; sequence b uses counter index seq_offset + b."""
    dev = torch.device(device)
    def act(width, tensor):
        t = torch.empty(batch, seqlen, width, dtype=dtype, device=dev)
        for b in range(batch):
            _fill_sequence(t[b], seed, tensor, seq_offset + b)
        return t
    x, dt, z = act(d_inner, T_X), act(d_inner, T_DT), act(d_inner, T_Z)
    Bm, Cm = act(d_state, T_B), act(d_state, T_C)
    h0 = None
    if h0_std > 0:
        h0 = torch.stack([normal((d_inner, d_state), seed, T_H0, seq_offset + b, 0, dev,
                                 std=h0_std) for b in range(batch)]) if batch else \
            torch.empty(0, d_inner, d_state, device=dev)
    return ScanInputs(x=x, delta=dt, z=z, B=Bm, C=Cm,
                      A=make_A(d_inner, d_state, A_kind, seed).to(dev),
                      D=torch.ones(d_inner, dtype=torch.float32, device=dev),
                      delta_bias=dt_bias_for(d_inner, seed).to(dev), h0=h0)


@dataclasses.dataclass
class DecodeStep:
    x: torch.Tensor      # [batch, d_inner]
    delta: torch.Tensor  # [batch, d_inner]
    z: torch.Tensor      # [batch, d_inner]
    B: torch.Tensor      # [batch, d_state]
    C: torch.Tensor      # [batch, d_state]


def decode_state(batch: int, d_inner: int, d_state: int, seed: int, device="cpu",
                 std: float = 0.1) -> torch.Tensor:
    """Cached fp32 state [batch, d_inner, d_state] ~ N(0, std^2)."""
    dev = torch.device(device)
    st = torch.empty(batch, d_inner, d_state, dtype=torch.float32, device=dev)
    for b in range(batch):
        st[b].copy_(normal((d_inner, d_state), seed, T_H0, b, 0, dev, std=std))
    return st


def decode_step(batch: int, d_inner: int, d_state: int, step: int, seed: int,
                dtype=torch.bfloat16, device="cpu") -> DecodeStep:
    """Inputs of one decode step (counter chunk index = step)."""
    dev = torch.device(device)
    def draw(width, tensor):
        return normal((batch, width), seed, tensor, 0, step, dev).to(dtype)
    return DecodeStep(x=draw(d_inner, T_X), delta=draw(d_inner, T_DT), z=draw(d_inner, T_Z),
                      B=draw(d_state, T_B), C=draw(d_state, T_C))


@dataclasses.dataclass
class SsdInputs:
    x: torch.Tensor           # [batch, seqlen, nheads * headdim]
    delta: torch.Tensor       # [batch, seqlen, nheads]
    z: torch.Tensor
    B: torch.Tensor           # [batch, seqlen, d_state]
    C: torch.Tensor
    A: torch.Tensor           # [nheads] fp32
    D: torch.Tensor           # [nheads * headdim] fp32
    delta_bias: torch.Tensor  # [nheads] fp32
    h0: torch.Tensor | None
    delta_softplus: bool = True


def ssd_inputs(batch: int, seqlen: int, nheads: int, headdim: int, d_state: int,
               dtype=torch.bfloat16, seed: int = 0, device="cpu", h0_std: float = 0.0,
               seq_offset: int = 0) -> SsdInputs:
    """Inputs of the scalar-identity (Mamba-2) scan, drawn like the diagonal
    scan's: x, z, delta, B, C ~ N(0, 1) rounded to the I/O dtype (delta one
    column per head), a per-head bias that centres Delta on a log-uniform dt0,
    A[head] = -U(1, 16) (a head's decay rate; Mamba-2 draws its A in that
    range), D = 1."""
    dev = torch.device(device)
    d_inner = nheads * headdim

    def act(width, tensor):
        t = torch.empty(batch, seqlen, width, dtype=dtype, device=dev)
        for b in range(batch):
            _fill_sequence(t[b], seed, tensor, seq_offset + b)
        return t
    x, dt, z = act(d_inner, T_X), act(nheads, T_DT), act(d_inner, T_Z)
    Bm, Cm = act(d_state, T_B), act(d_state, T_C)
    g = _gen("cpu", counter_seed(seed, T_A, 1, 0))
    A = -(1.0 + 15.0 * torch.rand(nheads, generator=g, dtype=torch.float32))
    h0 = None
    if h0_std > 0:
        h0 = torch.stack([normal((d_inner, d_state), seed, T_H0, seq_offset + b, 0, dev,
                                 std=h0_std) for b in range(batch)])
    return SsdInputs(x=x, delta=dt, z=z, B=Bm, C=Cm, A=A.to(dev),
                     D=torch.ones(d_inner, dtype=torch.float32, device=dev),
                     delta_bias=dt_bias_for(nheads, seed).to(dev), h0=h0)


# Named workloads (the S6 layer at Jamba's sizes, plus a tiny fp32 case).
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str          # "prefill" or "decode"
    batch: int
    seqlen: int        # prefill length, or decode steps for kind == "decode"
    d_inner: int
    d_state: int
    dtype: torch.dtype
    seed: int


WORKLOADS = {
    w.name: w for w in [
        Workload("s6_tiny_fp32_b1_l64_d16_n4", "prefill", 1, 64, 16, 4, torch.float32, 0),
        Workload("s6_prefill_bf16_b1_l4096_d8192_n16", "prefill", 1, 4096, 8192, 16,
                 torch.bfloat16, 1),
        Workload("s6_prefill_bf16_b1_l262144_d8192_n16", "prefill", 1, 262144, 8192, 16,
                 torch.bfloat16, 2),
        Workload("s6_prefill_bf16_b16_l16384_d8192_n16", "prefill", 16, 16384, 8192, 16,
                 torch.bfloat16, 3),
        Workload("s6_decode_bf16_b256_d8192_n16_x128", "decode", 256, 128, 8192, 16,
                 torch.bfloat16, 4),
    ]
}


def workload_inputs(w: Workload, device="cpu", seq_offset: int = 0) -> ScanInputs:
    assert w.kind == "prefill"
    return scan_inputs(w.batch, w.seqlen, w.d_inner, w.d_state, w.dtype, w.seed, device,
                       seq_offset=seq_offset)


@dataclasses.dataclass
class DtProjInputs:
    dt_low: torch.Tensor  # [ntok, dt_rank] fp32
    hi: torch.Tensor      # [ntok, dt_rank] bf16, bf16(dt_low)
    lo: torch.Tensor      # [ntok, dt_rank] bf16, bf16(dt_low - hi)
    W_dt: torch.Tensor    # [d_inner, dt_rank] bf16


def dt_proj_inputs(ntok: int, d_inner: int, dt_rank: int, seed: int, device) -> DtProjInputs:
    """Inputs of the low-rank product that produces the scan's raw Delta.

    dt_low ~ N(0, 1) in fp32 (unit RMS, as it leaves an RMSNorm with unit
    weights), handed over as the two bf16 planes the library takes;
    W_dt ~ U(-R^-1/2, R^-1/2) rounded to bf16 (R = dt_rank; the scale of
    Mamba's dt_proj initialisation), so that delta has variance ~1/3.
    """
    dt_low = normal((ntok, dt_rank), seed, T_DTLOW, 0, 0, device)
    hi = dt_low.to(torch.bfloat16)
    lo = (dt_low - hi.float()).to(torch.bfloat16)
    g = _gen(device, counter_seed(seed, T_WDT, 0, 0))
    u = torch.rand((d_inner, dt_rank), generator=g, device=device, dtype=torch.float32)
    W_dt = ((2.0 * u - 1.0) * dt_rank ** -0.5).to(torch.bfloat16)
    return DtProjInputs(dt_low, hi, lo, W_dt)


@dataclasses.dataclass
class XProjInputs:
    u: torch.Tensor      # [ntok, d_inner] bf16 (the scan's x)
    W_x: torch.Tensor    # [dt_rank + 2 d_state, d_inner] bf16
    w_dt: torch.Tensor   # [dt_rank] fp32 RMSNorm weights
    w_B: torch.Tensor    # [d_state] fp32
    w_C: torch.Tensor    # [d_state] fp32


def x_proj_inputs(ntok: int, d_inner: int, dt_rank: int, d_state: int, seed: int,
                  device) -> XProjInputs:
    """Inputs of the projection before the scan.

    u ~ N(0, 1) rounded to bf16 (the scan's x recipe); W_x ~ N(0, 1/d_inner)
    rounded to bf16, so each projected entry is ~N(0, 1) before its norm; the
    three RMSNorm weights ~ U(0.5, 1.5) in fp32 (a trained norm's weights sit
    near 1; the spread makes a swapped or ignored weight visible).
    """
    u = normal((ntok, d_inner), seed, T_X, 0, 0, device).to(torch.bfloat16)
    W_x = normal((dt_rank + 2 * d_state, d_inner), seed, T_WX, 0, 0, device,
                 std=d_inner ** -0.5).to(torch.bfloat16)
    g = _gen(device, counter_seed(seed, T_NORMW, 0, 0))
    w = 0.5 + torch.rand(dt_rank + 2 * d_state, generator=g, device=device, dtype=torch.float32)
    return XProjInputs(u, W_x, w[:dt_rank].contiguous(), w[dt_rank:dt_rank + d_state].contiguous(),
                       w[dt_rank + d_state:].contiguous())
