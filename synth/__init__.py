"""Seeded synthetic inputs for the Gated DeltaNet recurrence.

This module is shared by the tests, the benchmark and the package smoke check,
and serves both the CUDA path and the fp64 oracle with the same bytes.  It holds
none of the method's arithmetic: it draws random numbers, casts them to the
storage types, and applies the input recipe of each workload (for example
"q and k L2-normalised per head in fp32, then cast to bf16").

The five workloads (sizes of the Qwen3.8-27B linear-attention layers: 16 key
heads, 48 value heads, head width 128, conv width 4):

  0  prefill, 1 sequence, T = 256, zero initial state
  1  front end (conv1d + SiLU + L2) then prefill, 1 sequence, T = 8192
  2  prefill, 1 sequence, T = 262144, initial state ~ N(0, 0.02^2)
  3  varlen prefill, 16 sequences of lengths U[1024, 32768], per-sequence S0
  4  decode, one token through 48 layers for 128 sequences, state in place

Distributions: q, k, v ~ N(0, 1); a, b ~ N(0, 1); A_log = ln U(1, 16) per value
head; dt = exp(U(ln 1e-3, ln 0.1)) and dt_bias = ln(expm1(dt)) (the inverse of
softplus, so that softplus(dt_bias) = dt); conv weights ~ N(0, 0.5^2); initial
states ~ N(0, 0.02^2).  Every array is drawn from numpy's PCG64 seeded with a
list [seed, stream, block], so a block can be regenerated on its own.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

HQK, HV, D, CONV_K = 16, 48, 128, 4

# stream ids: one per kind of array, so that changing one size leaves the others
_S_Q, _S_K, _S_V, _S_A, _S_B, _S_ALOG, _S_DT, _S_S0, _S_QKV, _S_W, _S_LEN, _S_SLOT, _S_CS = range(13)

_BLOCK_ROWS = 4096          # rows per independently seeded block


def _rng(seed: int, stream: int, block: int = 0) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(stream), int(block)])


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even) and return the bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _normal_rows(seed, stream, rows, cols, std=1.0, dtype=np.float32):
    """[rows, cols] ~ N(0, std^2), generated in independently seeded row blocks."""
    out = np.empty((rows, cols), dtype=dtype)
    nblk = (rows + _BLOCK_ROWS - 1) // _BLOCK_ROWS

    def fill(bi):
        r0 = bi * _BLOCK_ROWS
        r1 = min(rows, r0 + _BLOCK_ROWS)
        blk = _rng(seed, stream, bi).standard_normal((r1 - r0, cols), dtype=np.float32)
        if std != 1.0:
            blk *= np.float32(std)
        out[r0:r1] = blk

    if nblk <= 1:
        for bi in range(nblk):
            fill(bi)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nblk)))
    return out


def _unit_rows_bf16(seed, stream, rows, heads, d, normalize):
    """[rows, heads, d] bf16 bits of N(0,1) draws; optionally each head vector is
    divided by sqrt(sum x^2 + 1e-6) in float32 before the cast (the input recipe
    "L2-normalised per head in fp32")."""
    out = np.empty((rows, heads, d), dtype=np.uint16)
    nblk = (rows + _BLOCK_ROWS - 1) // _BLOCK_ROWS

    def fill(bi):
        r0 = bi * _BLOCK_ROWS
        r1 = min(rows, r0 + _BLOCK_ROWS)
        x = _rng(seed, stream, bi).standard_normal((r1 - r0, heads, d), dtype=np.float32)
        if normalize:
            n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True, dtype=np.float32) + np.float32(1e-6))
            x = x / n
        out[r0:r1] = f32_to_bf16_bits(x)

    if nblk <= 1:
        for bi in range(nblk):
            fill(bi)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nblk)))
    return out


def gate_params(seed: int, Hv: int = HV, layers: int | None = None):
    """A_log = ln U(1,16); dt_bias = ln(expm1(dt)), dt log-uniform in [1e-3, 0.1].
    Shape [Hv], or [layers, Hv] when layers is given."""
    shape = (Hv,) if layers is None else (layers, Hv)
    A = _rng(seed, _S_ALOG).uniform(1.0, 16.0, size=shape)
    A_log = np.log(A).astype(np.float32)
    dt = np.exp(_rng(seed, _S_DT).uniform(math.log(1e-3), math.log(0.1), size=shape))
    dt_bias = np.log(np.expm1(dt)).astype(np.float32)
    return A_log, dt_bias


@dataclass
class PrefillInputs:
    q: np.ndarray            # uint16 bf16 bits [T, Hqk, d]
    k: np.ndarray            # uint16 bf16 bits [T, Hqk, d]
    v: np.ndarray            # uint16 bf16 bits [T, Hv, d]
    a: np.ndarray            # float32 [T, Hv]
    b: np.ndarray            # float32 [T, Hv]
    A_log: np.ndarray        # float32 [Hv]
    dt_bias: np.ndarray      # float32 [Hv]
    cu_seqlens: np.ndarray   # int32 [N+1]
    initial_state: np.ndarray | None   # float32 [N, Hv, d, d] or None
    scale: float
    Hqk: int = HQK
    Hv: int = HV
    d: int = D

    @property
    def T(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def N(self) -> int:
        return len(self.cu_seqlens) - 1


@dataclass
class FrontEndInputs:
    qkv: np.ndarray          # uint16 bf16 bits [T, (2 Hqk + Hv) d]
    conv_w: np.ndarray       # float32 [(2 Hqk + Hv) d, 4]
    cu_seqlens: np.ndarray   # int32 [N+1]
    conv_state: np.ndarray | None   # float32 [N, Ctot, 3] or None
    gates: PrefillInputs     # a, b, A_log, dt_bias, initial_state (q/k/v unused: empty)
    Hqk: int = HQK
    Hv: int = HV
    d: int = D


def make_prefill(lengths, seed: int, *, init_state: bool, init_std: float = 0.02,
                 Hqk: int = HQK, Hv: int = HV, d: int = D, normalize_qk: bool = True,
                 qkv: bool = True) -> PrefillInputs:
    """Packed (varlen) prefill inputs for the given sequence lengths."""
    lengths = [int(x) for x in lengths]
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    T = int(cu[-1])
    if qkv:
        q = _unit_rows_bf16(seed, _S_Q, T, Hqk, d, normalize_qk)
        k = _unit_rows_bf16(seed, _S_K, T, Hqk, d, normalize_qk)
        v = _unit_rows_bf16(seed, _S_V, T, Hv, d, False)
    else:
        q = k = np.zeros((0, Hqk, d), np.uint16)
        v = np.zeros((0, Hv, d), np.uint16)
    a = _normal_rows(seed, _S_A, T, Hv)
    b = _normal_rows(seed, _S_B, T, Hv)
    A_log, dt_bias = gate_params(seed, Hv)
    s0 = None
    if init_state:
        s0 = _normal_rows(seed, _S_S0, len(lengths) * Hv * d, d, std=init_std)
        s0 = s0.reshape(len(lengths), Hv, d, d)
    return PrefillInputs(q, k, v, a, b, A_log, dt_bias, cu, s0, 1.0 / math.sqrt(d), Hqk, Hv, d)


def make_frontend(lengths, seed: int, *, w_std: float = 0.5, conv_state: bool = False,
                  init_state: bool = False, Hqk: int = HQK, Hv: int = HV, d: int = D) -> FrontEndInputs:
    """Packed q|k|v channels ~ N(0,1) in bf16 and conv weights ~ N(0, w_std^2)."""
    lengths = [int(x) for x in lengths]
    ctot = (2 * Hqk + Hv) * d
    gates = make_prefill(lengths, seed, init_state=init_state, Hqk=Hqk, Hv=Hv, d=d, qkv=False)
    T = gates.T
    x = _normal_rows(seed, _S_QKV, T, ctot)
    qkv = f32_to_bf16_bits(x)
    w = _rng(seed, _S_W).standard_normal((ctot, CONV_K), dtype=np.float32) * np.float32(w_std)
    cs = None
    if conv_state:
        cs = bf16_bits_to_f32(f32_to_bf16_bits(
            _rng(seed, _S_QKV, 1 << 30).standard_normal((len(lengths), ctot, 3), dtype=np.float32)))
    return FrontEndInputs(qkv, w, gates.cu_seqlens, cs, gates, Hqk, Hv, d)


def varlen_lengths(seed: int, n: int = 16, lo: int = 1024, hi: int = 32768):
    """n integer lengths uniform in [lo, hi] inclusive."""
    return [int(x) for x in _rng(seed, _S_LEN).integers(lo, hi + 1, size=n)]


@dataclass
class DecodeInputs:
    q: np.ndarray            # uint16 [U, Hqk, d]   (U = n_seq * layers, unit u = s*layers + l)
    k: np.ndarray
    v: np.ndarray            # uint16 [U, Hv, d]
    a: np.ndarray            # float32 [U, Hv]
    b: np.ndarray
    A_log: np.ndarray        # float32 [layers, Hv]
    dt_bias: np.ndarray
    n_seq: int
    layers: int
    seed: int
    state_std: float
    scale: float
    Hqk: int = HQK
    Hv: int = HV
    d: int = D
    units_per_block: int = 16
    extra: dict = field(default_factory=dict)

    @property
    def U(self) -> int:
        return self.n_seq * self.layers

    def state_block(self, blk: int) -> np.ndarray:
        """float32 [units_per_block', Hv, d, d] initial states of units
        [blk*upb, min(U, (blk+1)*upb)), drawn from their own seed."""
        u0 = blk * self.units_per_block
        u1 = min(self.U, u0 + self.units_per_block)
        g = _rng(self.seed, _S_S0, blk)
        x = g.standard_normal((u1 - u0, self.Hv, self.d, self.d), dtype=np.float32)
        x *= np.float32(self.state_std)
        return x

    def n_state_blocks(self) -> int:
        return (self.U + self.units_per_block - 1) // self.units_per_block

    def state_of_units(self, units) -> np.ndarray:
        """float32 [len(units), Hv, d, d] initial states of the listed units."""
        out = np.empty((len(units), self.Hv, self.d, self.d), dtype=np.float32)
        cache = {}
        for i, u in enumerate(units):
            blk = int(u) // self.units_per_block
            if blk not in cache:
                cache[blk] = self.state_block(blk)
            out[i] = cache[blk][int(u) - blk * self.units_per_block]
        return out

    def full_state(self) -> np.ndarray:
        out = np.empty((self.U, self.Hv, self.d, self.d), dtype=np.float32)
        for blk in range(self.n_state_blocks()):
            s = self.state_block(blk)
            out[blk * self.units_per_block: blk * self.units_per_block + len(s)] = s
        return out


def make_decode(n_seq: int, layers: int, seed: int, *, state_std: float = 0.02,
                Hqk: int = HQK, Hv: int = HV, d: int = D) -> DecodeInputs:
    U = n_seq * layers
    q = _unit_rows_bf16(seed, _S_Q, U, Hqk, d, True)
    k = _unit_rows_bf16(seed, _S_K, U, Hqk, d, True)
    v = _unit_rows_bf16(seed, _S_V, U, Hv, d, False)
    a = _normal_rows(seed, _S_A, U, Hv)
    b = _normal_rows(seed, _S_B, U, Hv)
    A_log, dt_bias = gate_params(seed, Hv, layers)
    return DecodeInputs(q, k, v, a, b, A_log, dt_bias, n_seq, layers, seed, state_std,
                        1.0 / math.sqrt(d), Hqk, Hv, d)


@dataclass
class FusedDecodeInputs:
    """One decode step with the front end fused in: n_seq sequences x `layers`
    layers (unit u = n * layers + l), states held in n_slots slots."""
    qkv: np.ndarray          # uint16 [U, Ctot] packed q|k|v channels of the token
    conv_w: np.ndarray       # float32 [layers, Ctot, 4]
    conv_state: np.ndarray   # float32 [n_slots * layers, Ctot, 3], oldest input first
    a: np.ndarray            # float32 [U, Hv]
    b: np.ndarray
    A_log: np.ndarray        # float32 [layers, Hv]
    dt_bias: np.ndarray
    state: np.ndarray        # float32 [n_slots * layers, Hv, d, d]
    slot: np.ndarray         # int32 [n_seq], distinct slots
    n_seq: int
    layers: int
    n_slots: int
    scale: float
    Hqk: int = HQK
    Hv: int = HV
    d: int = D

    @property
    def U(self) -> int:
        return self.n_seq * self.layers


def make_decode_fused(n_seq: int, layers: int, n_slots: int, seed: int, *, w_std: float = 0.5,
                      state_std: float = 0.02, Hqk: int = HQK, Hv: int = HV,
                      d: int = D) -> FusedDecodeInputs:
    """Packed channels ~ N(0,1) in bf16, conv weights ~ N(0, w_std^2), conv
    histories ~ N(0,1) rounded to bf16 values, states ~ N(0, state_std^2), gates
    as for decode, and the sequences placed in a random choice of distinct
    slots."""
    U = n_seq * layers
    ctot = (2 * Hqk + Hv) * d
    qkv = f32_to_bf16_bits(_normal_rows(seed, _S_QKV, U, ctot))
    conv_w = _rng(seed, _S_W).standard_normal((layers, ctot, CONV_K), dtype=np.float32)
    conv_w *= np.float32(w_std)
    cs = _rng(seed, _S_CS).standard_normal((n_slots * layers, ctot, 3), dtype=np.float32)
    cs = bf16_bits_to_f32(f32_to_bf16_bits(cs))
    a = _normal_rows(seed, _S_A, U, Hv)
    b = _normal_rows(seed, _S_B, U, Hv)
    A_log, dt_bias = gate_params(seed, Hv, layers)
    st = _rng(seed, _S_S0).standard_normal((n_slots * layers, Hv, d, d), dtype=np.float32)
    st *= np.float32(state_std)
    slot = _rng(seed, _S_SLOT).permutation(n_slots)[:n_seq].astype(np.int32)
    return FusedDecodeInputs(qkv, conv_w, cs, a, b, A_log, dt_bias, st, slot, n_seq, layers,
                             n_slots, 1.0 / math.sqrt(d), Hqk, Hv, d)


# ---- the five workloads --------------------------------------------------------

WORKLOADS = {
    0: "gdn_prefill T=256 N=1 Hqk=16 Hv=48 d=128 zero S0",
    1: "gdn_conv1d_silu+gdn_prefill T=8192 N=1 Hqk=16 Hv=48 d=128 zero S0",
    2: "gdn_prefill T=262144 N=1 Hqk=16 Hv=48 d=128 S0~N(0,0.02^2)",
    3: "gdn_prefill varlen N=16 lengths U[1024,32768] Hqk=16 Hv=48 d=128 S0~N(0,0.02^2)",
    4: "gdn_decode_step 128 seq x 48 layers Hqk=16 Hv=48 d=128 fp32 state in place",
}


def workload(i: int):
    """Inputs of workload i (seed = i)."""
    if i == 0:
        return make_prefill([256], 0, init_state=False)
    if i == 1:
        return make_frontend([8192], 1)
    if i == 2:
        return make_prefill([262144], 2, init_state=True)
    if i == 3:
        return make_prefill(varlen_lengths(3), 3, init_state=True)
    if i == 4:
        return make_decode(128, 48, 4)
    raise ValueError(i)
