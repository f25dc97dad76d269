"""Seeded synthetic inputs for the seed-matmul path.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no LFSR, no basis, no unpacking).  Both the oracle-based
tests and the CUDA path take their inputs from here.

The generator is SplitMix64 (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014) used as a counter-based hash:
value i of stream ``key`` is mix64(key + (i + 1) * 0x9E3779B97F4A7C15).
It is written with int64 torch ops (wrapping multiply, masked logical shifts),
so it produces the same bits on the CPU and on a GPU; the 21.9 GB expert stack
is drawn directly in device memory, and any slice of it can be drawn again on
the host.

Packed-field recipe (uniform fields, as the synthetic workloads state):
* seeds: 1 + (u32 mod 65535), two per 64-bit draw -> uniform on [1, 65535]
  (bias below 1e-5).
* coefs: one uniform u16 per block (four per draw).  For P=4 that is four
  uniform int4 nibbles; for P=3 three uniform int4 nibbles and a uniform
  4-bit exponent code in the top nibble.
* codes (P=4): one uniform byte per two blocks (eight per draw): two uniform
  4-bit exponent codes.
* exp_bias: constant (-12 by default) per row.
* x: bf16(N(0,1)) by Box-Muller on two 53-bit uniforms, drawn on the CPU.
* router logits: N(0,1) float32; Zipf variant: log p_e + Gumbel(0,1) with
  p_e proportional to (rank_e + 1)^-s over a seeded permutation of ranks.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

BASE_SEED = 0x5EED

_GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1

# stream tags
FIELD_SEEDS, FIELD_COEFS, FIELD_CODES, FIELD_X, FIELD_LOGITS, FIELD_PERM = 1, 2, 3, 4, 5, 6
MAT_GATE, MAT_UP, MAT_DOWN, MAT_SINGLE = 0, 1, 2, 3


def _s64(v: int) -> int:
    """Python int (mod 2^64) -> the signed int64 with the same bits."""
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def mix64_int(z: int) -> int:
    """SplitMix64 finaliser on a Python int (mod 2^64)."""
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def stream_key(*parts: int) -> int:
    """Key of one stream, from the base seed and a tuple of small integers."""
    h = BASE_SEED
    for p in parts:
        h = mix64_int(h ^ mix64_int((int(p) + _GOLDEN) & _MASK64))
    return h


def _lsr(z: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def splitmix64(key: int, start: int, n: int, device="cpu") -> torch.Tensor:
    """Values start .. start+n-1 of stream ``key`` as int64 bit patterns."""
    idx = torch.arange(start + 1, start + n + 1, dtype=torch.int64, device=device)
    z = idx * _s64(_GOLDEN) + _s64(key)
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    return z ^ _lsr(z, 31)


def uniform01(key: int, n: int, start: int = 0) -> torch.Tensor:
    """n float64 uniforms in (0, 1] from the top 53 bits (CPU)."""
    z = splitmix64(key, start, n, "cpu")
    return (_lsr(z, 11).to(torch.float64) + 1.0) * (2.0 ** -53)


def normal_f64(key: int, n: int) -> torch.Tensor:
    """n standard normals by Box-Muller (CPU, float64)."""
    m = (n + 1) // 2
    u = uniform01(key, 2 * m)
    u1, u2 = u[0::2], u[1::2]
    r = torch.sqrt(-2.0 * torch.log(u1))
    z = torch.cat([r * torch.cos(2 * math.pi * u2), r * torch.sin(2 * math.pi * u2)])
    return z[:n]


def bf16_bits(t: torch.Tensor) -> torch.Tensor:
    """bfloat16 tensor -> its bit patterns as int16 (same storage size)."""
    return t.contiguous().view(torch.int16)


def normal_bf16(key: int, shape) -> torch.Tensor:
    """bf16(N(0,1)) values, as a bfloat16 CPU tensor of the given shape."""
    n = int(math.prod(shape))
    return normal_f64(key, n).to(torch.float32).to(torch.bfloat16).reshape(shape)


@dataclasses.dataclass
class SeedMatrix:
    """Packed seed matrix fields (a stack of ``n_experts`` experts when > 1).

    seeds int16 [R][K/8], coefs int16 [R][K/8], codes uint8 [R][K/16] (P=4)
    or None (P=3), exp_bias int32 [R]; R = n_experts * rows."""

    seeds: torch.Tensor
    coefs: torch.Tensor
    codes: Optional[torch.Tensor]
    exp_bias: torch.Tensor
    rows: int
    K: int
    P: int
    n_experts: int = 1

    @property
    def N(self) -> int:
        return self.rows * self.n_experts

    def packed_bytes(self) -> int:
        n = self.seeds.numel() * 2 + self.coefs.numel() * 2 + self.exp_bias.numel() * 4
        if self.codes is not None:
            n += self.codes.numel()
        return n

    def to(self, device) -> "SeedMatrix":
        return dataclasses.replace(
            self, seeds=self.seeds.to(device), coefs=self.coefs.to(device),
            codes=None if self.codes is None else self.codes.to(device),
            exp_bias=self.exp_bias.to(device))

    def expert(self, e: int) -> "SeedMatrix":
        """View of expert e of a stack, as a single matrix."""
        r0, r1 = e * self.rows, (e + 1) * self.rows
        return dataclasses.replace(
            self, seeds=self.seeds[r0:r1], coefs=self.coefs[r0:r1],
            codes=None if self.codes is None else self.codes[r0:r1],
            exp_bias=self.exp_bias[r0:r1], n_experts=1)

    def numpy(self):
        """A host copy with NumPy arrays (uint16 / uint8 / int32), for the oracle."""
        import numpy as np

        class _Host:
            pass

        h = _Host()
        h.seeds = self.seeds.cpu().numpy().view(np.uint16)
        h.coefs = self.coefs.cpu().numpy().view(np.uint16)
        h.codes = None if self.codes is None else self.codes.cpu().numpy().view(np.uint8)
        h.exp_bias = self.exp_bias.cpu().numpy().astype(np.int32)
        h.P = self.P
        return h


def _u16_stream(key: int, n: int, device) -> torch.Tensor:
    """n uniform 16-bit values (as int16 bit patterns)."""
    z = splitmix64(key, 0, (n + 3) // 4, device)
    return z.view(torch.int16)[:n]


def _u8_stream(key: int, n: int, device) -> torch.Tensor:
    z = splitmix64(key, 0, (n + 7) // 8, device)
    return z.view(torch.uint8)[:n]


def _seed_stream(key: int, n: int, device) -> torch.Tensor:
    """n seeds uniform on [1, 65535] (int16 bit patterns)."""
    z = splitmix64(key, 0, (n + 1) // 2, device)
    u32 = z.view(torch.int32)[:n].to(torch.int64) & 0xFFFFFFFF
    s = (u32 % 65535) + 1
    return s.to(torch.int32).to(torch.int16)  # wraps 32768..65535 to the same bits


def seed_matrix(rows: int, K: int, P: int, tag=(0,), n_experts: int = 1,
                exp_bias: int = -12, device="cpu") -> SeedMatrix:
    """Uniform random packed fields for a (stack of) rows x K seed matrix.

    P = 35 is P = 3 with 5-bit coefficients: a uniform coefs word is three
    uniform 5-bit fields and one uniform code bit, and the codes stream holds
    3 uniform code bits per block (3K/64 bytes per row)."""
    if K % {4: 16, 3: 8, 35: 64}[P] != 0:
        raise ValueError("K must be a multiple of 16 (P=4), 8 (P=3) or 64 (P=35)")
    R = rows * n_experts
    nb = K // 8
    seeds = _seed_stream(stream_key(*tag, FIELD_SEEDS), R * nb, device).reshape(R, nb)
    coefs = _u16_stream(stream_key(*tag, FIELD_COEFS), R * nb, device).reshape(R, nb)
    codes = None
    if P == 4:
        codes = _u8_stream(stream_key(*tag, FIELD_CODES), R * nb // 2, device).reshape(R, nb // 2)
    elif P == 35:
        codes = _u8_stream(stream_key(*tag, FIELD_CODES), R * 3 * nb // 8, device).reshape(R, 3 * nb // 8)
    eb = torch.full((R,), exp_bias, dtype=torch.int32, device=device)
    return SeedMatrix(seeds.contiguous(), coefs.contiguous(),
                      None if codes is None else codes.contiguous(), eb, rows, K, P, n_experts)


def activations(tag, T: int, K: int) -> torch.Tensor:
    """x: [T][K] bf16(N(0,1)) on the CPU."""
    return normal_bf16(stream_key(*tag, FIELD_X), (T, K))


def router_logits(tag, T: int, E: int, zipf_s: Optional[float] = None) -> torch.Tensor:
    """[T][E] float32 router logits: N(0,1), or the Zipf(s) variant."""
    if zipf_s is None:
        return normal_f64(stream_key(*tag, FIELD_LOGITS), T * E).to(torch.float32).reshape(T, E)
    perm_keys = splitmix64(stream_key(*tag, FIELD_PERM), 0, E, "cpu")
    rank = torch.argsort(torch.argsort(perm_keys))          # a seeded permutation of 0..E-1
    logp = -zipf_s * torch.log(rank.to(torch.float64) + 1.0)
    logp = logp - torch.logsumexp(logp, 0)
    u = uniform01(stream_key(*tag, FIELD_LOGITS), T * E).reshape(T, E)
    u = torch.clamp(u, max=1.0 - 2.0 ** -53)
    gumbel = -torch.log(-torch.log(u))
    return (logp[None, :] + gumbel).to(torch.float32)


# ------------------------------------------------------------ workloads

@dataclasses.dataclass
class MoELayer:
    gate: SeedMatrix
    up: SeedMatrix
    down: SeedMatrix


def moe_layer(layer: int, E: int, hidden: int, inter: int, P: int, device="cpu",
              config: int = 2) -> MoELayer:
    """One layer of E stacked experts: gate/up [E*inter][hidden], down [E*hidden][inter]."""
    g = seed_matrix(inter, hidden, P, (config, layer, MAT_GATE), E, device=device)
    u = seed_matrix(inter, hidden, P, (config, layer, MAT_UP), E, device=device)
    d = seed_matrix(hidden, inter, P, (config, layer, MAT_DOWN), E, device=device)
    return MoELayer(g, u, d)


def expert_slice(layer: int, e: int, E: int, hidden: int, inter: int, P: int,
                 config: int = 2) -> MoELayer:
    """Expert e of a layer drawn again on the host (the same bits as moe_layer)."""
    def one(rows, K, mat):
        nb = K // 8
        tag = (config, layer, mat)
        start_blk = e * rows * nb
        n = rows * nb
        # seeds: two per draw; coefs: four per draw; codes: eight per draw
        z = splitmix64(stream_key(*tag, FIELD_SEEDS), start_blk // 2, (n + 1) // 2 + 1)
        u32 = z.view(torch.int32).to(torch.int64) & 0xFFFFFFFF
        off = start_blk % 2
        seeds = ((u32[off:off + n] % 65535) + 1).to(torch.int32).to(torch.int16)
        z = splitmix64(stream_key(*tag, FIELD_COEFS), start_blk // 4, n // 4 + 2)
        off = start_blk % 4
        coefs = z.view(torch.int16)[off:off + n]
        codes = None
        if P == 4:
            nc = n // 2
            st = start_blk // 2
            z = splitmix64(stream_key(*tag, FIELD_CODES), st // 8, nc // 8 + 2)
            codes = z.view(torch.uint8)[st % 8: st % 8 + nc].reshape(rows, nb // 2).contiguous()
        eb = torch.full((rows,), -12, dtype=torch.int32)
        return SeedMatrix(seeds.reshape(rows, nb).contiguous(), coefs.reshape(rows, nb).contiguous(),
                          codes, eb, rows, K, P, 1)

    return MoELayer(one(inter, hidden, MAT_GATE), one(inter, hidden, MAT_UP), one(hidden, inter, MAT_DOWN))
