"""Seeded synthetic inputs for the Sketch&Walk hot path.

This module is shared by the tests, the benchmark and the oracle's callers.
It draws random tensors and holds none of the method's arithmetic: no block
pooling, no projection, no walk, no selection and no attention.

Recipe (one stream per (sequence, layer, tensor kind, head)):

* Q and K rows follow a stationary AR(1) process along the sequence,
  x_0 ~ N(0, I), x_t = rho * x_{t-1} + sqrt(1 - rho^2) * eps_t, eps_t ~ N(0, I).
* "Hub" blocks: per (layer, KV head) ``hubs`` distinct block indices are drawn
  uniformly without replacement from 1..b-1 (b = number of blocks of the
  prompt). Each hub gets one offset vector ~ N(0, 0.5 I) (variance 0.5) that is
  added to every row of that block in K of the KV head and in Q of every query
  head of its GQA group.
* "Sink": +1.0 on every coordinate of block 0, in Q and in K.
* V ~ N(0, I) i.i.d.
* Decode: the KV cache holds ``n0`` prompt tokens followed by the tokens that
  the decode steps append (the same processes, continued); the query tokens
  are a fresh AR(1) stream of length ``steps`` per (sequence, layer, head).

The random engine is torch's: Philox on CUDA devices, mt19937 on the CPU, so
values depend on the device they were drawn on. Both sides of every parity
check consume the very same tensors, which makes this parity-neutral.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass
from typing import Tuple

import torch

_M64 = (1 << 64) - 1

KIND_Q, KIND_K, KIND_V, KIND_HUB_POS, KIND_HUB_OFF, KIND_QDEC, KIND_QSEQ = range(7)


def _mix64(x: int) -> int:
    """Scrambles a stream id into a generator seed (splitmix64 finaliser)."""
    x = (x + 0x9E3779B97F4A7C15) & _M64
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & _M64
    return x ^ (x >> 31)


def stream_seed(seed: int, layer: int, kind: int, head: int, seq: int = 0) -> int:
    sid = (seed << 40) ^ (seq << 24) ^ (layer << 16) ^ (kind << 12) ^ head
    return _mix64(sid & _M64) & ((1 << 63) - 1)


def _gen(device, s: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


@dataclass(frozen=True)
class PrefillWorkload:
    name: str
    layers: int
    hq: int
    hkv: int
    d: int
    n: int
    B: int
    k: int
    density: Tuple[int, int]
    dtype: str  # "fp32" or "bf16"
    rho: float
    hubs: int
    seed: int
    s: int = 8

    @property
    def b(self) -> int:
        return -(-self.n // self.B)

    def scaled(self, **kw) -> "PrefillWorkload":
        return dataclasses.replace(self, **kw)


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    batch: int
    layers: int
    hq: int
    hkv: int
    d: int
    n0: int  # cached prompt tokens per sequence
    steps: int
    B: int
    k: int
    density: Tuple[int, int]
    rho: float
    hubs: int
    seed: int
    s: int = 8
    dtype: str = "bf16"

    @property
    def max_len(self) -> int:
        return self.n0 + self.steps

    def scaled(self, **kw) -> "DecodeWorkload":
        return dataclasses.replace(self, **kw)


# The five workloads the hot path is specified on (shapes of the GQA models the
# pages evaluate: 32 query / 8 KV heads, head dim 128, 16K-128K context).
TINY = PrefillWorkload("tiny_n1024_d64_B64_k16", 2, 1, 1, 64, 1024, 64, 16, (1, 5), "fp32", 0.9, 2, 0)
PREFILL_16K = PrefillWorkload("prefill_n16384_B64_k32_L4", 4, 32, 8, 128, 16384, 64, 32, (1, 5), "bf16", 0.9, 8, 1)
PREFILL_64K = PrefillWorkload("prefill_n65536_B128_k32_L8", 8, 32, 8, 128, 65536, 128, 32, (1, 5), "bf16", 0.95, 16, 2)
PREFILL_128K = PrefillWorkload("prefill_n131072_B128_k32_L4", 4, 32, 8, 128, 131072, 128, 32, (1, 5), "bf16", 0.95, 32, 3)
PREFILL_128K_D10 = PREFILL_128K.scaled(name="prefill_n131072_B128_k32_L4_d10", density=(1, 10))
DECODE_128K = DecodeWorkload("decode_b16_n131072_B64_k32_L8", 16, 8, 32, 8, 128, 131072, 64, 64, 32, (1, 5), 0.95, 32, 4)


def _dtype(name: str) -> torch.dtype:
    return {"fp32": torch.float32, "bf16": torch.bfloat16, "fp64": torch.float64}[name]


def _linear_scan(e: torch.Tensor, a: float, chunk: int = 256) -> torch.Tensor:
    """x_t = a * x_{t-1} + e_t along dim -2 (x_{-1} = 0), chunked and recursive."""
    n, d = e.shape[-2], e.shape[-1]
    lead = e.shape[:-2]
    dev, dt = e.device, e.dtype
    c = min(chunk, n)
    t = torch.arange(c, device=dev, dtype=torch.float64)
    expo = t[:, None] - t[None, :]
    T = torch.where(expo >= 0, torch.tensor(a, dtype=torch.float64, device=dev) ** expo.clamp(min=0),
                    torch.zeros((), dtype=torch.float64, device=dev)).to(dt)
    if n <= c:
        return torch.matmul(T, e)
    nc = -(-n // c)
    pad = nc * c - n
    if pad:
        e = torch.cat([e, torch.zeros(*lead, pad, d, device=dev, dtype=dt)], dim=-2)
    ec = e.reshape(*lead, nc, c, d)
    xl = torch.matmul(T, ec)  # local scans of each chunk
    ends = _linear_scan(xl[..., :, c - 1, :], a ** c, chunk)  # true chunk-end values
    prev = torch.cat([torch.zeros(*lead, 1, d, device=dev, dtype=dt), ends[..., :-1, :]], dim=-2)
    powers = (torch.tensor(a, dtype=torch.float64, device=dev) ** (t + 1)).to(dt)
    x = xl + powers[:, None] * prev[..., :, None, :]
    return x.reshape(*lead, nc * c, d)[..., :n, :]


def ar1(n: int, d: int, rho: float, gen: torch.Generator, device) -> torch.Tensor:
    """One stationary AR(1) stream of n rows of dimension d (unit variance)."""
    work = torch.float64 if torch.device(device).type == "cpu" else torch.float32
    eps = torch.randn(n, d, generator=gen, device=device, dtype=work)
    eps[1:] *= math.sqrt(1.0 - rho * rho)
    return _linear_scan(eps, rho, chunk=256 if work == torch.float64 else 16)


def hub_layout(b: int, hubs: int, d: int, seed: int, layer: int, g: int, device, seq: int = 0):
    """Hub block indices (from 1..b-1, without replacement) and their offsets."""
    h = min(hubs, max(b - 1, 0))
    gp = _gen(device, stream_seed(seed, layer, KIND_HUB_POS, g, seq))
    pos = (torch.randperm(b - 1, generator=gp, device=device)[:h] + 1) if h > 0 else torch.zeros(0, dtype=torch.long, device=device)
    go = _gen(device, stream_seed(seed, layer, KIND_HUB_OFF, g, seq))
    work = torch.float64 if torch.device(device).type == "cpu" else torch.float32
    off = torch.randn(h, d, generator=go, device=device, dtype=work) * math.sqrt(0.5)
    return pos, off


def _add_structure(x: torch.Tensor, B: int, pos: torch.Tensor, off: torch.Tensor) -> None:
    """Adds the sink shift on block 0 and the hub offsets, in place, to x [n, d]."""
    x[: min(B, x.shape[0])] += 1.0
    for j in range(pos.shape[0]):
        p = int(pos[j])
        x[p * B:(p + 1) * B] += off[j]


def prefill_layer_inputs(w: PrefillWorkload, layer: int, device="cpu"):
    """Q [hq, n, d], K [hkv, n, d], V [hkv, n, d] in the workload's dtype."""
    out_dt = _dtype(w.dtype)
    group = w.hq // w.hkv
    Q = torch.empty(w.hq, w.n, w.d, dtype=out_dt, device=device)
    K = torch.empty(w.hkv, w.n, w.d, dtype=out_dt, device=device)
    V = torch.empty(w.hkv, w.n, w.d, dtype=out_dt, device=device)
    for g in range(w.hkv):
        pos, off = hub_layout(w.b, w.hubs, w.d, w.seed, layer, g, device)
        kx = ar1(w.n, w.d, w.rho, _gen(device, stream_seed(w.seed, layer, KIND_K, g)), device)
        _add_structure(kx, w.B, pos, off)
        K[g] = kx.to(out_dt)
        del kx
        gv = _gen(device, stream_seed(w.seed, layer, KIND_V, g))
        work = torch.float64 if torch.device(device).type == "cpu" else torch.float32
        V[g] = torch.randn(w.n, w.d, generator=gv, device=device, dtype=work).to(out_dt)
        for h in range(g * group, (g + 1) * group):
            qx = ar1(w.n, w.d, w.rho, _gen(device, stream_seed(w.seed, layer, KIND_Q, h)), device)
            _add_structure(qx, w.B, pos, off)
            Q[h] = qx.to(out_dt)
            del qx
    return Q, K, V


def prefill_head_inputs(w: PrefillWorkload, layer: int, h: int, device="cpu"):
    """Q[h] [n, d] and K[g], V[g] [n, d] of query head h (g = its KV head): the
    same streams as prefill_layer_inputs, for callers that need one head only."""
    out_dt = _dtype(w.dtype)
    g = h // (w.hq // w.hkv)
    work = torch.float64 if torch.device(device).type == "cpu" else torch.float32
    pos, off = hub_layout(w.b, w.hubs, w.d, w.seed, layer, g, device)
    kx = ar1(w.n, w.d, w.rho, _gen(device, stream_seed(w.seed, layer, KIND_K, g)), device)
    _add_structure(kx, w.B, pos, off)
    gv = _gen(device, stream_seed(w.seed, layer, KIND_V, g))
    v = torch.randn(w.n, w.d, generator=gv, device=device, dtype=work)
    qx = ar1(w.n, w.d, w.rho, _gen(device, stream_seed(w.seed, layer, KIND_Q, h)), device)
    _add_structure(qx, w.B, pos, off)
    return qx.to(out_dt), kx.to(out_dt), v.to(out_dt)


def decode_cache_inputs(w: DecodeWorkload, seq: int, layer: int, device="cpu"):
    """K, V [hkv, n0 + steps, d] for one sequence and layer (prompt + appended)."""
    out_dt = _dtype(w.dtype)
    L = w.max_len
    b0 = -(-w.n0 // w.B)
    K = torch.empty(w.hkv, L, w.d, dtype=out_dt, device=device)
    V = torch.empty(w.hkv, L, w.d, dtype=out_dt, device=device)
    work = torch.float64 if torch.device(device).type == "cpu" else torch.float32
    for g in range(w.hkv):
        pos, off = hub_layout(b0, w.hubs, w.d, w.seed, layer, g, device, seq)
        kx = ar1(L, w.d, w.rho, _gen(device, stream_seed(w.seed, layer, KIND_K, g, seq)), device)
        _add_structure(kx, w.B, pos, off)
        K[g] = kx.to(out_dt)
        del kx
        gv = _gen(device, stream_seed(w.seed, layer, KIND_V, g, seq))
        V[g] = torch.randn(L, w.d, generator=gv, device=device, dtype=work).to(out_dt)
    return K, V


def decode_queries(w: DecodeWorkload, seq: int, layer: int, device="cpu"):
    """Q [hq, steps, d]: the query token of every decode step for one sequence and layer."""
    out_dt = _dtype(w.dtype)
    Q = torch.empty(w.hq, w.steps, w.d, dtype=out_dt, device=device)
    for h in range(w.hq):
        Q[h] = ar1(w.steps, w.d, w.rho, _gen(device, stream_seed(w.seed, layer, KIND_QDEC, h, seq)), device).to(out_dt)
    return Q


def decode_sequence_queries(w: DecodeWorkload, seq: int, layer: int, device="cpu"):
    """Q [hq, n0 + steps, d]: the queries of every position of one sequence and
    layer, prompt and decoded tokens alike (for a decode that needs the prompt's
    queries too); the same AR(1), sink and hub structure as the keys of the
    query head's group."""
    out_dt = _dtype(w.dtype)
    L = w.max_len
    b0 = -(-w.n0 // w.B)
    group = w.hq // w.hkv
    Q = torch.empty(w.hq, L, w.d, dtype=out_dt, device=device)
    for g in range(w.hkv):
        pos, off = hub_layout(b0, w.hubs, w.d, w.seed, layer, g, device, seq)
        for h in range(g * group, (g + 1) * group):
            qx = ar1(L, w.d, w.rho, _gen(device, stream_seed(w.seed, layer, KIND_QSEQ, h, seq)), device)
            _add_structure(qx, w.B, pos, off)
            Q[h] = qx.to(out_dt)
            del qx
    return Q
