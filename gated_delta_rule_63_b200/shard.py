"""Head sharding of the layer over GPUs (host logic only: index arrays).

The layer's heads never exchange data: value head h reads key head h // (hv / hk), and
the conv, the recurrence and the gated norm are per channel, per head or per 128-wide
row.  So n GPUs can each hold hk / n key heads and hv / n value heads ("33B 只做 18 层
...", mhpq.cn §6: the optional two-way tensor parallel run): each computes its heads'
columns of the input projection (q, k, v, z, a, b), runs the layer's entry points on
them with hk / n and hv / n heads, and multiplies its slice of the normed output by its
columns of the output projection's weight.  The n partial outputs are summed by one
all-reduce; nothing else crosses GPUs.

Layouts are those of the entry points: the input projection's 2 hk dk + 2 hv dv + 2 hv
outputs in the order [q | k | v | z | a | b] (conv channels [q | k | v] first), the
output projection's weight [hidden][hv dv].
"""
from dataclasses import dataclass

import numpy as np


@dataclass
class HeadShard:
    in_rows: np.ndarray     # rows of the input projection's weight (its outputs) this shard computes
    conv_channels: np.ndarray   # conv channels ([q | k | v] order) of those outputs: in_rows[:n_conv]
    n_conv: int             # outputs that go through the conv (q, k, v), then z, a, b
    n_z: int
    n_gate: int             # outputs in each of a and b
    heads: slice            # value heads (A_log, dt_bias, states, o and the norm's rows)
    key_heads: slice
    out_cols: np.ndarray    # columns of the output projection's weight (the normed output's channels)
    hk: int
    hv: int


def head_shard(shard: int, n_shards: int, hk: int = 16, hv: int = 48, dk: int = 128, dv: int = 128) -> HeadShard:
    """The part of the layer that shard `shard` of `n_shards` holds (contiguous head groups)."""
    if n_shards < 1 or not 0 <= shard < n_shards or hk % n_shards or hv % n_shards or hv % hk:
        raise ValueError("heads must split evenly over the shards and value heads group over key heads")
    ks, vs = hk // n_shards, hv // n_shards
    kq = np.arange(shard * ks * dk, (shard + 1) * ks * dk)
    v = np.arange(shard * vs * dv, (shard + 1) * vs * dv)
    g = np.arange(shard * vs, (shard + 1) * vs)
    q_off, k_off, v_off = 0, hk * dk, 2 * hk * dk
    z_off = v_off + hv * dv
    a_off = z_off + hv * dv
    b_off = a_off + hv
    conv = np.concatenate([q_off + kq, k_off + kq, v_off + v])
    rows = np.concatenate([conv, z_off + v, a_off + g, b_off + g])
    return HeadShard(in_rows=rows, conv_channels=conv, n_conv=conv.size, n_z=v.size, n_gate=g.size,
                     heads=slice(shard * vs, (shard + 1) * vs), key_heads=slice(shard * ks, (shard + 1) * ks),
                     out_cols=v, hk=ks, hv=vs)
