"""Seeded synthetic inputs for the gated delta-rule layer.

This module is shared by the tests, the benchmark and the oracle harness.  It
holds no arithmetic of the method itself: it draws random numbers, rounds them
to bf16 and lays them out.  Every tensor it returns is a numpy array:

* bf16 tensors are ``uint16`` arrays holding the raw bf16 bit patterns,
* fp32 tensors are ``float32`` arrays,
* ``cu_seqlens`` is ``int32``.

Distributions follow the workloads the layer is exercised on (16 key heads,
48 value heads, head dim 128; see the recipe in the repository's design
notes):

* q, k, v, x, a, b, z  ~ N(0, 1)
* A_log   = log U(1, 16)                  (one per value head)
* dt_bias = log(expm1(U(1e-3, 0.1)))     (one per value head)
* conv weights ~ N(0, 0.5) (std 0.5)
* initial recurrent states ~ N(0, 0.02) (std 0.02)

The generator is numpy's PCG64 seeded with the workload's seed; draws happen
in a fixed documented order so that a workload is reproducible bit for bit.
A normal tensor of more than 2^24 elements is drawn in blocks of 2^22
elements, block i from its own PCG64 whose seed is the i-th of a list of
63-bit integers drawn from the workload's generator at that point of the
order; the blocks are filled on all host cores.  Smaller tensors come straight
from the workload's generator.
"""

from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np

HK = 16          # key heads
HV = 48          # value heads
DK = 128         # key head dim
DV = 128         # value head dim
CONV_K = 4       # causal conv width
CHUNK = 64       # chunk length of the prefill


# ---------------------------------------------------------------------------
# bf16 bit handling (input preparation only)
# ---------------------------------------------------------------------------

_PAR_MIN = 1 << 24      # tensors above this many elements are processed in blocks
_PAR_BLOCK = 1 << 22    # elements per block


def _blocks(n):
    return [slice(i, min(n, i + _PAR_BLOCK)) for i in range(0, n, _PAR_BLOCK)]


def _each_block(fn, n):
    """fn(slice) over the blocks of n elements on all host cores (numpy releases the GIL)."""
    with ThreadPoolExecutor(max(1, os.cpu_count() or 1)) as ex:
        list(ex.map(fn, _blocks(n)))


def _f32_to_bf16_flat(u, out):
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    out[...] = ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even).

    Returns the bf16 bit patterns as uint16.  Inputs are finite.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.reshape(-1).view(np.uint32)
    out = np.empty(u.shape, dtype=np.uint16)
    if u.size <= _PAR_MIN:
        _f32_to_bf16_flat(u, out)
    else:
        _each_block(lambda s: _f32_to_bf16_flat(u[s], out[s]), u.size)
    return out.reshape(x.shape)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


# ---------------------------------------------------------------------------
# primitive draws
# ---------------------------------------------------------------------------

def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _standard_normal_f32(rng, shape) -> np.ndarray:
    """N(0, 1) float32 draws of the given shape (large tensors in seeded blocks, see above)."""
    n = int(np.prod(shape))
    if n <= _PAR_MIN:
        return rng.standard_normal(size=shape, dtype=np.float32)
    blocks = _blocks(n)
    seeds = rng.integers(0, 2 ** 63, size=len(blocks), dtype=np.int64)
    out = np.empty(n, dtype=np.float32)
    index = {b.start: i for i, b in enumerate(blocks)}

    def fill(s):
        g = np.random.Generator(np.random.PCG64(int(seeds[index[s.start]])))
        g.standard_normal(dtype=np.float32, out=out[s])

    _each_block(fill, n)
    return out.reshape(shape)


def _normal_bf16(rng, shape, std=1.0) -> np.ndarray:
    x = _standard_normal_f32(rng, shape)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x)


def _unit_rows_bf16(rng, shape) -> np.ndarray:
    """N(0,1) rows rescaled to unit L2 length along the last axis, then bf16.

    This is the input recipe "q and k L2-normalised per head".
    """
    x = _standard_normal_f32(rng, shape)
    d = shape[-1]
    flat = x.reshape(-1, d)
    out = np.empty_like(flat)

    def unit(s):
        rows = slice(s.start // d, s.stop // d)
        n = np.sqrt(np.sum(flat[rows].astype(np.float64) ** 2, axis=-1, keepdims=True))
        out[rows] = (flat[rows] / n).astype(np.float32)

    if x.size <= _PAR_MIN or _PAR_BLOCK % d:
        unit(slice(0, x.size))
    else:
        _each_block(unit, x.size)
    return f32_to_bf16_bits(out.reshape(shape))


def _head_params(rng, hv):
    """A_log = log U(1,16), dt_bias = log(expm1(U(1e-3, 0.1))), float32."""
    A_log = np.log(rng.uniform(1.0, 16.0, size=hv)).astype(np.float32)
    dt = rng.uniform(1e-3, 0.1, size=hv)
    dt_bias = np.log(np.expm1(dt)).astype(np.float32)
    return A_log, dt_bias


def varlen_lengths(seed: int, n: int, lo: int, hi: int) -> np.ndarray:
    """n sequence lengths drawn uniformly from the integers [lo, hi]."""
    rng = _rng(seed)
    return rng.integers(lo, hi + 1, size=n).astype(np.int64)


def cu_seqlens_from_lengths(lengths) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    assert cu[-1] < 2 ** 31
    return cu.astype(np.int32)


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class CoreInputs:
    """Inputs of the recurrence alone (already convolved / no conv)."""
    q: np.ndarray            # [T, hk, dk]  bf16 bits
    k: np.ndarray            # [T, hk, dk]  bf16 bits
    v: np.ndarray            # [T, hv, dv]  bf16 bits
    a: np.ndarray            # [T, hv]      bf16 bits
    b: np.ndarray            # [T, hv]      bf16 bits
    A_log: np.ndarray        # [hv] f32
    dt_bias: np.ndarray      # [hv] f32
    cu_seqlens: np.ndarray   # [N+1] int32
    h0: Optional[np.ndarray] # [N, hv, dk, dv] f32 or None
    scale: float = 1.0

    @property
    def T(self):
        return int(self.q.shape[0])

    @property
    def n_seqs(self):
        return int(self.cu_seqlens.shape[0] - 1)


def make_core_inputs(seed: int, lengths, hk=HK, hv=HV, dk=DK, dv=DV,
                     prenorm_qk=True, h0_std: Optional[float] = None,
                     scale: float = 1.0) -> CoreInputs:
    """Draw order: q, k, v, a, b, A_log/dt_bias, h0."""
    rng = _rng(seed)
    cu = cu_seqlens_from_lengths(lengths)
    T = int(cu[-1])
    if prenorm_qk:
        q = _unit_rows_bf16(rng, (T, hk, dk))
        k = _unit_rows_bf16(rng, (T, hk, dk))
    else:
        q = _normal_bf16(rng, (T, hk, dk))
        k = _normal_bf16(rng, (T, hk, dk))
    v = _normal_bf16(rng, (T, hv, dv))
    a = _normal_bf16(rng, (T, hv))
    b = _normal_bf16(rng, (T, hv))
    A_log, dt_bias = _head_params(rng, hv)
    h0 = None
    if h0_std is not None:
        h0 = (rng.standard_normal(size=(len(lengths), hv, dk, dv), dtype=np.float32)
              * np.float32(h0_std))
    return CoreInputs(q, k, v, a, b, A_log, dt_bias, cu, h0, scale)


@dataclasses.dataclass
class FullInputs:
    """Inputs of the whole prefill path: conv -> recurrence -> gated norm."""
    x: np.ndarray            # [T, C] bf16 bits, C = hk*dk + hk*dk + hv*dv ([q | k | v])
    conv_w: np.ndarray       # [C, 4] bf16 bits
    conv_state: Optional[np.ndarray]  # [N, 3, C] bf16 bits or None (zeros)
    a: np.ndarray            # [T, hv] bf16 bits
    b: np.ndarray            # [T, hv] bf16 bits
    z: np.ndarray            # [T, hv, dv] bf16 bits
    norm_w: Optional[np.ndarray]  # [dv] f32 or None (ones)
    A_log: np.ndarray
    dt_bias: np.ndarray
    cu_seqlens: np.ndarray
    h0: Optional[np.ndarray]
    hk: int = HK
    hv: int = HV
    dk: int = DK
    dv: int = DV
    scale: float = 1.0
    eps: float = 1e-6

    @property
    def T(self):
        return int(self.x.shape[0])

    @property
    def n_seqs(self):
        return int(self.cu_seqlens.shape[0] - 1)

    @property
    def channels(self):
        return int(self.x.shape[1])


def make_full_inputs(seed: int, lengths, hk=HK, hv=HV, dk=DK, dv=DV,
                     h0_std: Optional[float] = None, conv_state_std: Optional[float] = None,
                     norm_w_std: Optional[float] = None, scale: float = 1.0,
                     eps: float = 1e-6) -> FullInputs:
    """Draw order: x, conv_w, a, b, z, A_log/dt_bias, h0, conv_state, norm_w."""
    rng = _rng(seed)
    cu = cu_seqlens_from_lengths(lengths)
    T = int(cu[-1])
    C = hk * dk * 2 + hv * dv
    x = _normal_bf16(rng, (T, C))
    conv_w = _normal_bf16(rng, (C, CONV_K), std=0.5)
    a = _normal_bf16(rng, (T, hv))
    b = _normal_bf16(rng, (T, hv))
    z = _normal_bf16(rng, (T, hv, dv))
    A_log, dt_bias = _head_params(rng, hv)
    h0 = None
    if h0_std is not None:
        h0 = (rng.standard_normal(size=(len(lengths), hv, dk, dv), dtype=np.float32)
              * np.float32(h0_std))
    conv_state = None
    if conv_state_std is not None:
        conv_state = _normal_bf16(rng, (len(lengths), CONV_K - 1, C), std=conv_state_std)
    norm_w = None
    if norm_w_std is not None:
        norm_w = (1.0 + rng.standard_normal(size=(dv,), dtype=np.float32)
                  * np.float32(norm_w_std)).astype(np.float32)
    return FullInputs(x, conv_w, conv_state, a, b, z, norm_w, A_log, dt_bias, cu, h0,
                      hk, hv, dk, dv, scale, eps)


@dataclasses.dataclass
class DecodeInputs:
    """B independent sequences advanced by `steps` single-token steps."""
    x: np.ndarray            # [steps, B, C] bf16 bits (pre-conv)
    a: np.ndarray            # [steps, B, hv] bf16 bits
    b: np.ndarray            # [steps, B, hv] bf16 bits
    conv_w: np.ndarray       # [C, 4] bf16 bits
    conv_state: np.ndarray   # [B, 3, C] bf16 bits
    state: np.ndarray        # [B, hv, dk, dv] f32
    A_log: np.ndarray
    dt_bias: np.ndarray
    hk: int = HK
    hv: int = HV
    dk: int = DK
    dv: int = DV
    scale: float = 1.0

    @property
    def B(self):
        return int(self.x.shape[1])

    @property
    def steps(self):
        return int(self.x.shape[0])


def make_decode_inputs(seed: int, batch: int, steps: int, hk=HK, hv=HV, dk=DK, dv=DV,
                       state_std=0.02, conv_state_std=1.0, scale: float = 1.0) -> DecodeInputs:
    """Draw order: state, conv_state, conv_w, A_log/dt_bias, then x, a, b of every step
    (each one tensor [steps, batch, ...])."""
    rng = _rng(seed)
    C = hk * dk * 2 + hv * dv
    state = (rng.standard_normal(size=(batch, hv, dk, dv), dtype=np.float32)
             * np.float32(state_std))
    conv_state = _normal_bf16(rng, (batch, CONV_K - 1, C), std=conv_state_std)
    conv_w = _normal_bf16(rng, (C, CONV_K), std=0.5)
    A_log, dt_bias = _head_params(rng, hv)
    x = _normal_bf16(rng, (steps, batch, C))
    a = _normal_bf16(rng, (steps, batch, hv))
    b = _normal_bf16(rng, (steps, batch, hv))
    return DecodeInputs(x, a, b, conv_w, conv_state, state, A_log, dt_bias,
                        hk, hv, dk, dv, scale)


def make_slot_table(seed: int, batch: int, n_slots: int, n_padding: int = 0) -> np.ndarray:
    """Distinct pool entries for `batch` rows drawn from `n_slots`, int32; the last
    `n_padding` rows get -1 (padding).  Indices only: no arithmetic of the layer."""
    if batch - n_padding > n_slots:
        raise ValueError("more live rows than pool entries")
    slot = np.full(batch, -1, dtype=np.int32)
    slot[: batch - n_padding] = _rng(seed).permutation(n_slots)[: batch - n_padding]
    return slot


# ---------------------------------------------------------------------------
# the five workloads of the layer (sizes and seeds)
# ---------------------------------------------------------------------------

def workload_core_T128(seed=0):
    """B=1, T=128, pre-normalised q/k, zero initial state, no conv."""
    return make_core_inputs(seed, [128], prenorm_qk=True)


def workload_full_T4096(seed=1):
    """B=1, T=4096, conv4+SiLU -> recurrence -> gated RMSNorm, zero state."""
    return make_full_inputs(seed, [4096])


def workload_decode_B64(seed=2, steps=1000):
    """64 sequences, one token per step, fp32 states ~ N(0, 0.02)."""
    return make_decode_inputs(seed, 64, steps)


def workload_core_T262144(seed=3):
    """B=1, T=262144, pre-normalised q/k, zero initial state, no conv."""
    return make_core_inputs(seed, [262144], prenorm_qk=True)


def varlen8_lengths(seed=4):
    return varlen_lengths(seed, 8, 1024, 32768)


def workload_full_varlen8(seed=4):
    """8 packed sequences, lengths U{1024..32768}, h0 ~ N(0,0.02), full path."""
    return make_full_inputs(seed + 1000, varlen8_lengths(seed), h0_std=0.02)


@dataclasses.dataclass
class MixedServing:
    """One mixed serving step on a pool of cached states: new requests prefilled into free
    entries of the pool, running requests decoding one token from theirs."""
    prefill: CoreInputs       # the new requests' recurrence inputs (packed, varlen)
    new_slot: np.ndarray      # [n_new] int32 entries the new requests fill
    decode_slot: np.ndarray   # [rows] int32 entries of the running requests
    n_slots: int


def workload_mixed_serving(seed=5, n_new=4, rows=64, n_slots=128):
    """4 new requests of U{256..4096} tokens (recurrence inputs, q/k not normalised) into free
    entries of a 128-entry pool, beside the 64 running rows of decode_B64 (their entries: the
    same seeded half of the pool as make_slot_table(7, 64, 128))."""
    decode_slot = make_slot_table(7, rows, n_slots)
    free = np.setdiff1d(np.arange(n_slots, dtype=np.int32), decode_slot)
    new_slot = _rng(seed).permutation(free)[:n_new].astype(np.int32)
    lengths = varlen_lengths(seed, n_new, 256, 4096)
    return MixedServing(make_core_inputs(seed + 1000, lengths, prenorm_qk=False), new_slot,
                        decode_slot, n_slots)


# ---------------------------------------------------------------------------
# the layer's projections (hidden 5120 -> q|k|v 10 240, z 6144, a, b 48 each; 6144 -> 5120)
# ---------------------------------------------------------------------------

HIDDEN = 5120
IN_PROJ_N = 2 * HK * DK + HV * DV + HV * DV + 2 * HV   # q|k|v, z, a, b: 16 480 outputs
OUT_PROJ_K = HV * DV                                    # the gated norm's output, 6144


def make_linear_inputs(seed: int, M: int, N: int, K: int):
    """Activations x [M, K] ~ N(0, 1) and a weight w [N, K] ~ N(0, 1/K) (a projection at
    initialisation scale), both bf16 bits.  Draw order: x, w."""
    rng = _rng(seed)
    x = _normal_bf16(rng, (M, K))
    w = _normal_bf16(rng, (N, K), std=1.0 / np.sqrt(K))
    return x, w


def workload_in_proj_T4096(seed=6):
    """The input projection of the T = 4096 prefill: 4096 tokens x 5120 -> 16 480."""
    return make_linear_inputs(seed, 4096, IN_PROJ_N, HIDDEN)


def workload_out_proj_T4096(seed=7):
    """The output projection of the T = 4096 prefill: 4096 tokens x 6144 -> 5120."""
    return make_linear_inputs(seed, 4096, HIDDEN, OUT_PROJ_K)
